// plan_harness.cu -- a host build of the CUDA library's work decomposition,
// for CPU tests of its tile lists against the KSA mask.
//
// The library's sources are compiled into this program whole, so the
// functions under test are the kernels' own, marked __host__ __device__:
//   pf::unit_of           the forward's work items and their K/V tiles
//                         (plain prefill and chunk mode),
//   bt::key_tile, bt::key_queries, bt::share_blocks, bt::q_tile
//                         the backward's key tiles with the text query range
//                         that sees each (dk/dv), and its query tiles with
//                         their key tiles (dq),
//   bt_step_shape, bt_max_tiles, bt_dkv_grid, bt_dq_grid
//                         the backward's step shape and launch bounds,
//   ck::chunk_state_code, ck::chunk_ranges, ck::layout, ck::key_rows
//                         the chunked prefill's state checks, gathered
//                         chunk ranges, buffer sizes and the cache slot or
//                         block row each key is read from,
//   decode_slice          the live cache slots of a decode query.
// Only the prefix sums that the plan kernels compute on the device (one
// scan per array) are written out here, as plain loops, together with the
// per-call constants the launch functions set (Gp, Tc, Tk).
//
// Input: one query per line on stdin.  Output: integer lines, each query's
// block closed by a line "end".
//   fwd   k w Hq Hkv B n_0 .. n_{B-1}
//         "W Gp HP Tc Tk", then per work item
//         "hkv h0 b nb mb ncb qbase kvbase sbase c0 cend cw_lo n_win T"
//   chunk k w Hq Hkv B (n0 m0 T)_0 .. (n0 m0 T)_{B-1}
//         per sequence "code cbeg kvb ncb qoff kvoff"; then
//         "sum_q sum_kv units L.q_chunks L.kv_chunks L.max_units sum_slot0";
//         then the work items as for fwd
//   bwd   k w Hq Hkv B n_0 .. n_{B-1}
//         "ns nt nqs split max_tiles dkv_grid dq_grid dkv_ctas", then per key
//         tile "b sum j0 kcnt n m c0 qlo qhi nq lead nsh" followed by each
//         share's query blocks "r_lo r_hi", then "ntt" and per dq CTA
//         "b n m c0 q0 qn c_first ns n_sum t_lo n_win"
//   bwdt  k w n t_0 .. t_{j-1}
//         one sequence of n tokens (n up to INT32_MAX: only the listed key
//         tiles are built); per tile "b sum j0 kcnt n m c0 qlo qhi nq lead
//         nsh", then
//         "lo hi" of key rows 0, 1 and kcnt - 1 (bt::key_queries)
//   slice k w kind n m
//         "ok lo hi"
//   keys  k w n0 m0 T
//         per text key p < n0 + T "0 p src at", then per summary
//         j < m0 + S "1 j src at": src 0 = cache slot at, 1 = row at of the
//         block's input (one sequence, one kv head)
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "../kv_cache_compression_ksa_b200/csrc/prefill_sm100.cu"
#include "../kv_cache_compression_ksa_b200/csrc/prefill_bwd_sm100.cu"
#include "../kv_cache_compression_ksa_b200/csrc/prefill_chunk.cu"

namespace ksa {
int sm_count() { return 148; }   // the launch functions are not called here
}

using namespace ksa;

static ksa_params params(int k, int w, int Hq, int Hkv)
{
    ksa_params p;
    std::memset(&p, 0, sizeof(p));
    p.k = k; p.w = w; p.num_q_heads = Hq; p.num_kv_heads = Hkv; p.head_dim = 128;
    return p;
}

// Per-call constants of the forward, as the launch functions set them.
static bool fwd_consts(const ksa_params &p, pf::Params &P)
{
    std::memset(&P, 0, sizeof(P));
    const int G = p.num_q_heads / p.num_kv_heads;
    P.k = p.k; P.w = p.w; P.G = G; P.Hq = p.num_q_heads; P.Hkv = p.num_kv_heads;
    P.Gp = prefill_heads_per_tile(&p);
    if (P.Gp < 1) return false;
    P.HP = G / P.Gp;
    P.Tc = pf::BM / (P.Gp * p.k);
    P.Tk = pf::BN / p.k;
    if (P.Tc < 1 || P.Tk < 1) return false;
    P.unit_chunks = P.Tc;
    return true;
}

static void print_items(const pf::Params &P, int n_units)
{
    const int W = n_units * P.Hkv * P.HP;
    std::printf("%d %d %d %d %d\n", W, P.Gp, P.HP, P.Tc, P.Tk);
    for (int item = 0; item < W; ++item) {
        const pf::Unit U = pf::unit_of(P, item, n_units);
        std::printf("%d %d %d %d %d %d %d %d %d %d %d %d %d %d\n", U.hkv, U.h0, U.b, U.nb, U.mb, U.ncb, U.qbase,
                    U.kvbase, U.sbase, U.c0, U.cend, U.cw_lo, U.n_win, U.T);
    }
}

static void run_fwd(int k, int w, int Hq, int Hkv, const std::vector<int> &n)
{
    const ksa_params p = params(k, w, Hq, Hkv);
    pf::Params P;
    if (!fwd_consts(p, P)) { std::printf("unsupported\n"); return; }
    const int B = (int)n.size();
    std::vector<int32_t> cu(B + 1, 0), chunk_off(B + 1, 0), tile_off(B + 1, 0);
    for (int b = 0; b < B; ++b) {
        const int c = (n[b] + k - 1) / k;
        cu[b + 1] = cu[b] + n[b];
        chunk_off[b + 1] = chunk_off[b] + c;
        tile_off[b + 1] = tile_off[b] + (c + P.unit_chunks - 1) / P.unit_chunks;
    }
    P.batch = B;
    P.cu = cu.data();
    P.pl.chunk_off = chunk_off.data();
    P.pl.tile_off = tile_off.data();
    print_items(P, tile_off[B]);
}

static void run_chunk(int k, int w, int Hq, int Hkv, const std::vector<int> &trip)
{
    const ksa_params p = params(k, w, Hq, Hkv);
    const int B = (int)trip.size() / 3;
    const int64_t cap = 1 << 20;
    ck::Args a;
    std::memset(&a, 0, sizeof(a));
    a.k = k; a.w = w; a.Hq = Hq; a.Hkv = Hkv; a.G = Hq / Hkv; a.batch = B; a.d = 128;
    a.cap = cap;
    a.S = 1 + (int64_t)k + (int64_t)w * k + cap;
    a.uc = ck::tc_unit_chunks(&p);
    std::vector<int32_t> state(4 * B, 0);
    int64_t total_t = 0, total_s = 0;
    std::vector<int> T(B), S(B);
    for (int b = 0; b < B; ++b) {
        const int n0 = trip[3 * b], m0 = trip[3 * b + 1];
        T[b] = trip[3 * b + 2];
        state[4 * b] = n0;
        state[4 * b + 1] = m0;
        const int64_t f0 = (int64_t)n0 - (int64_t)m0 * k;
        S[b] = f0 >= 0 ? (int)((f0 + T[b]) / k) : 0;   // the summaries the block completes
        total_t += T[b];
        total_s += S[b];
    }
    a.state = state.data();
    pf::Params P;
    if (a.uc < 1 || !fwd_consts(p, P)) { std::printf("unsupported\n"); return; }
    std::vector<int32_t> cbeg(B), ntot(B), qbase(B), kvbase(B), uoff(B + 1, 0);
    int32_t oq = 0, okv = 0;
    for (int b = 0; b < B; ++b) {
        int32_t n0, m0;
        const int code = ck::chunk_state_code(a, b, T[b], S[b], &n0, &m0);
        int cb = 0, kb = 0, nc = 0;
        if (code == KSA_OK && T[b] > 0) ck::chunk_ranges(a, n0, m0, T[b], &cb, &kb, &nc);
        std::printf("%d %d %d %d %d %d\n", code, cb, kb, nc, oq, okv);
        cbeg[b] = cb; ntot[b] = n0 + T[b];
        qbase[b] = oq - cb; kvbase[b] = okv - kb;
        uoff[b + 1] = uoff[b];
        if (code == KSA_OK && T[b] > 0) {
            uoff[b + 1] += (nc - cb + a.uc - 1) / a.uc;
            oq += nc - cb;
            okv += nc - kb;
        }
    }
    const ck::Layout L = ck::layout(&p, B, total_t, total_s);
    P.batch = B;
    P.ck_tile_off = uoff.data(); P.ck_cbeg = cbeg.data(); P.ck_ntot = ntot.data();
    P.ck_qbase = qbase.data(); P.ck_kvbase = kvbase.data();
    P.sum_slot0 = 1 + k + w * k;
    std::printf("%d %d %d %lld %lld %lld %d\n", oq, okv, uoff[B], (long long)L.q_chunks, (long long)L.kv_chunks,
                (long long)L.max_units, P.sum_slot0);
    print_items(P, uoff[B]);
}

static void run_bwd(int k, int w, int Hq, int Hkv, const std::vector<int> &n)
{
    const int B = (int)n.size();
    int nqs, split;
    bt_step_shape(k, &nqs, &split);
    std::vector<int32_t> cu(B + 1, 0), chunk_off(B + 1, 0), ks_off(B + 1, 0), kt_off(B + 1, 0);
    for (int b = 0; b < B; ++b) {
        cu[b + 1] = cu[b] + n[b];
        chunk_off[b + 1] = chunk_off[b] + (n[b] + k - 1) / k;
        ks_off[b + 1] = ks_off[b] + (n[b] / k + bt::BK - 1) / bt::BK;
        kt_off[b + 1] = kt_off[b] + (n[b] + bt::BK - 1) / bt::BK;
    }
    bt::TArgs a;
    std::memset(&a, 0, sizeof(a));
    a.k = k; a.w = w; a.G = Hq / Hkv; a.Hq = Hq; a.Hkv = Hkv; a.batch = B;
    a.cu = cu.data();
    a.pl.chunk_off = chunk_off.data();
    a.ks_off = ks_off.data();
    a.kt_off = kt_off.data();
    a.nqs = nqs;
    a.split = split;
    a.bpw = bt_bpw(a.G, split);
    const int ns = ks_off[B], nt = kt_off[B];
    const int64_t total_text = cu[B], aug_rows = (int64_t)chunk_off[B] * (k + 1);
    // the plan's CTA shares: nsh per key tile
    int64_t ctas = 0;
    std::vector<bt::KTile> tiles(ns + nt);
    for (int t = 0; t < ns + nt; ++t) {
        bt::key_tile(a, t, tiles[t]);
        ctas += tiles[t].nsh;
    }
    std::printf("%d %d %d %d %lld %lld %lld %lld\n", ns, nt, nqs, split, (long long)bt_max_tiles(B, aug_rows),
                (long long)bt_dkv_grid(total_text, B, k, w, a.G, nqs, split), (long long)bt_dq_grid(total_text, B),
                (long long)ctas);
    for (const bt::KTile &T : tiles) {
        std::printf("%d %d %d %d %d %d %d %d %d %d %d %d", T.b, T.sum, T.j0, T.kcnt, T.n, T.m, T.c0, T.qlo, T.qhi,
                    T.nq, T.lead, T.nsh);
        for (int sh = 0; sh < T.nsh; ++sh) {
            int r_lo, r_hi;
            bt::share_blocks(a, T, sh, r_lo, r_hi);
            std::printf(" %d %d", r_lo, r_hi);
        }
        std::printf("\n");
    }
    std::printf("%d\n", nt);
    for (int cta = 0;; ++cta) {
        bt::QTile Q;
        if (!bt::q_tile(a, cta, Q)) break;
        std::printf("%d %d %d %d %d %d %d %d %d %d %d\n", Q.b, Q.n, Q.m, Q.c0, Q.q0, Q.qn, Q.c_first, Q.ns, Q.n_sum,
                    Q.t_lo, Q.n_win);
    }
}

static void run_bwd_tiles(int k, int w, int64_t n, const std::vector<int> &tiles)
{
    int nqs, split;
    bt_step_shape(k, &nqs, &split);
    const int32_t cu[2] = {0, (int32_t)n};
    const int32_t chunk_off[2] = {0, (int32_t)((n + k - 1) / k)};
    const int32_t ks_off[2] = {0, (int32_t)((n / k + bt::BK - 1) / bt::BK)};
    const int32_t kt_off[2] = {0, (int32_t)((n + bt::BK - 1) / bt::BK)};
    bt::TArgs a;
    std::memset(&a, 0, sizeof(a));
    a.k = k; a.w = w; a.G = 1; a.Hq = 1; a.Hkv = 1; a.batch = 1;
    a.cu = cu;
    a.pl.chunk_off = const_cast<int32_t *>(chunk_off);
    a.ks_off = ks_off;
    a.kt_off = kt_off;
    a.nqs = nqs;
    a.split = split;
    a.bpw = bt_bpw(a.G, split);
    for (int t : tiles) {
        bt::KTile T;
        bt::key_tile(a, t, T);
        std::printf("%d %d %d %d %d %d %d %d %d %d %d %d\n", T.b, T.sum, T.j0, T.kcnt, T.n, T.m, T.c0, T.qlo, T.qhi,
                    T.nq, T.lead, T.nsh);
        const int rows[3] = {0, 1, T.kcnt - 1};
        for (int r : rows) {
            int lo, hi;
            bt::key_queries(a, T, r, lo, hi);
            std::printf("%d %d ", lo, hi);
        }
        std::printf("\n");
    }
}

static void run_keys(int k, int w, int n0, int m0, int T)
{
    constexpr int D = 64;
    const int64_t f0 = (int64_t)n0 - (int64_t)m0 * k;
    const int S_new = f0 >= 0 ? (int)((f0 + T) / k) : 0;
    const int64_t cap = m0 + S_new + 1;
    ck::Args a;
    std::memset(&a, 0, sizeof(a));
    a.k = k; a.w = w; a.Hkv = 1; a.Hq = 1; a.G = 1; a.batch = 1; a.d = D;
    a.cap = cap;
    a.S = 1 + (int64_t)k + (int64_t)w * k + cap;
    const int32_t cu_t[2] = {0, T}, cu_s[2] = {0, S_new};
    a.cu_t = cu_t; a.cu_s = cu_s;
    std::vector<__nv_bfloat16> ck_(a.S * D), cv_(a.S * D), kt_((size_t)T * D + D), vt_((size_t)T * D + D),
        ks_((size_t)S_new * D + D), vs_((size_t)S_new * D + D);
    a.ck = ck_.data(); a.cv = cv_.data();
    a.ktr = kt_.data(); a.vt = vt_.data();
    a.ksr = ks_.data(); a.vs = vs_.data();
    const ck::Snap sn{n0, m0, 1, 0};
    auto locate = [&](const __nv_bfloat16 *pk, const __nv_bfloat16 *pv, const __nv_bfloat16 *kb,
                      const __nv_bfloat16 *vb, size_t rows, int64_t *at) {
        if (pk < kb || pk >= kb + rows * D) return false;
        *at = (pk - kb) / D;
        return (pk - kb) % D == 0 && pv == vb + *at * D;   // K and V from the same row
    };
    for (int kind = 0; kind < 2; ++kind) {
        const int count = kind == 0 ? n0 + T : m0 + S_new;
        for (int idx = 0; idx < count; ++idx) {
            const __nv_bfloat16 *pk = nullptr, *pv = nullptr;
            ck::key_rows<D>(a, sn, 0, 0, kind == 0 ? ck::TEXT_ROWS : ck::SUM_ROWS, idx, pk, pv);
            int64_t at = -1;
            int src = -1;
            if (locate(pk, pv, a.ck, a.cv, (size_t)a.S, &at)) src = 0;
            else if (kind == 0 && locate(pk, pv, a.ktr, a.vt, (size_t)T, &at)) src = 1;
            else if (kind == 1 && locate(pk, pv, a.ksr, a.vs, (size_t)S_new, &at)) src = 1;
            std::printf("%d %d %d %lld\n", kind, idx, src, (long long)at);
        }
    }
}

int main()
{
    char line[1 << 16];
    while (std::fgets(line, sizeof(line), stdin)) {
        char mode[16] = {0};
        int off = 0;
        if (std::sscanf(line, "%15s%n", mode, &off) != 1) continue;
        std::vector<long long> v;
        const char *s = line + off;
        long long x;
        int used;
        while (std::sscanf(s, "%lld%n", &x, &used) == 1) { v.push_back(x); s += used; }
        const std::string m(mode);
        auto ints = [&](size_t from) { return std::vector<int>(v.begin() + from, v.end()); };
        if (m == "fwd" && v.size() >= 5 && v.size() == 5 + (size_t)v[4]) {
            run_fwd((int)v[0], (int)v[1], (int)v[2], (int)v[3], ints(5));
        } else if (m == "chunk" && v.size() >= 5 && v.size() == 5 + 3 * (size_t)v[4]) {
            run_chunk((int)v[0], (int)v[1], (int)v[2], (int)v[3], ints(5));
        } else if (m == "bwd" && v.size() >= 5 && v.size() == 5 + (size_t)v[4]) {
            run_bwd((int)v[0], (int)v[1], (int)v[2], (int)v[3], ints(5));
        } else if (m == "bwdt" && v.size() >= 3) {
            run_bwd_tiles((int)v[0], (int)v[1], v[2], ints(3));
        } else if (m == "keys" && v.size() == 5) {
            run_keys((int)v[0], (int)v[1], (int)v[2], (int)v[3], (int)v[4]);
        } else if (m == "slice" && v.size() == 5) {
            int64_t lo = 0, hi = 0;
            const bool ok = decode_slice((int)v[2], v[3], v[4], (int)v[0], (int)v[1], &lo, &hi);
            std::printf("%d %lld %lld\n", ok ? 1 : 0, (long long)lo, (long long)hi);
        } else {
            std::printf("bad query\n");
        }
        std::printf("end\n");
        std::fflush(stdout);
    }
    return 0;
}

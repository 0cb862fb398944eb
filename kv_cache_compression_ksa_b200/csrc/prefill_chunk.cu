// prefill_chunk.cu -- chunked prefill: a block of new text tokens per
// sequence (and the summaries of the chunks they complete) attended against
// the sequence's decode cache, after which the cache is extended by the block.
//
// Kwai Summary Attention Technical Report.  The rows computed are the
// prefill's, Eq. (10) under the rule of section 2.2: text t_i of chunk c sees
// the text of chunks c-w .. c causally and the summaries s_0 .. s_{c-w-1}
// (Eqs. (2)-(3)); summary s_j sees the k text tokens of chunk j and itself.
// They are the rows of text positions n0 .. n0+T-1 (and of summaries
// m0 .. m1-1) of a sequence whose first n0 tokens already sit in the cache
// of section 2.3.1 (Figure 4).  Older keys are read where that cache keeps
// them: a distant summary s_j at slot 1+k+w*k+j, a token of the open chunk at
// slot k-r, a token of one of the last w complete chunks in its ring block
// (chunk mod w).  The block's own keys come from the call's inputs (q and k
// rotated once into the workspace).  Then the block is written into the
// cache in the state that the token-by-token appends of Figure 4 reach.
//
//   chunk_plan_kernel    validate each sequence, snapshot (n0, m0), offsets
//   chunk_rope_kernel    rotate the block's q and k at their positions
// text rows, tensor-core path (shapes the prefill kernel takes):
//   chunk_sumwrite_kernel  the block's summaries into the cache's summary
//                        slots first (append-only slots no query reads yet),
//                        so all summary keys sit in one contiguous run
//   chunk_gather_kernel  the block's query rows and its window of text keys
//                        (cached ring / open-chunk tokens and new tokens)
//                        into small augmented buffers
//   prefill_kernel       (prefill_sm100.cu, chunk mode) summary tiles by TMA
//                        from the cache, window tiles from the gathered rows
//   chunk_scatter_kernel outputs of the new rows back to [T, Hq, d]
//   chunk_sum_kernel     the block's summary rows: k + 1 keys each, one warp
//                        per (summary, kv head)
// text and summary rows otherwise (q heads per kv head not 1, 2, 4 or 8):
//   chunk_attn_kernel    64 query rows of one q head against their visible keys
//                        (warp-level tensor-core MMA, online softmax)
//   chunk_append_kernel  write the block into the cache, advance the state
#include <math.h>

#include "ksa_internal.cuh"
#include "warp_mma.cuh"

namespace ksa {
namespace ck {

constexpr int RB = 64;          // query rows per block, keys per key block
constexpr int kThreads = 128;   // 4 warps x 16 query rows
constexpr int TEXT_ROWS = 0, SUM_ROWS = 1;

// Per sequence, taken before the call changes the cache state.
struct Snap {
    int32_t n0, m0, ok, pad;
};

struct Args {
    int k, w, Hq, Hkv, G, batch, d;
    int64_t S, cap;                     // cache slots per (sequence, kv head); summary capacity
    float scale_log2;
    double log2_theta;
    int rotate;
    const int32_t *cu_t, *cu_s;         // [B+1] new text tokens / new summaries
    int64_t total_t, total_s;
    Snap *snap;                         // [B]
    int32_t *tb_off, *sb_off;           // [B+1] first text / summary query block
    // tensor-core path (uc > 0: query chunks per prefill work unit)
    int uc;
    int32_t *cbeg, *kvbeg, *ntot, *qbase, *kvbase;   // [B]
    int32_t *qoff, *kvoff, *uoff;                    // [B+1] gathered q chunks, window chunks, work units
    int64_t q_chunks, kv_chunks;                     // buffer extents (chunks of k + 1 rows)
    __nv_bfloat16 *qa, *ka, *va, *oa;                // gathered buffers
    float *la;
    int32_t *state;                     // cache state [B, 4]
    int32_t *err;
    __nv_bfloat16 *ck, *cv;             // cache [B, Hkv, S, d]
    const __nv_bfloat16 *qt, *kt, *vt, *qs, *ks, *vs;   // block inputs, q / k not rotated
    __nv_bfloat16 *qtr, *ktr, *qsr, *ksr;              // rotated copies (workspace)
    __nv_bfloat16 *ot, *os;
    float *lt, *ls;
};

__device__ __forceinline__ int find_seq(const int32_t *off, int batch, int id)
{
    int lo = 0, hi = batch - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (off[mid] <= id) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// ---------------------------------------------------------------------------
// Plan: one block scans the batch.  A sequence is valid when its state has no
// error, 0 <= f0 = n0 - m0 k <= k, the new summaries are exactly the chunks
// the block completes, floor((f0 + T) / k), and they fit the capacity.  An
// invalid sequence gets its state error set and is left untouched.
// ---------------------------------------------------------------------------
constexpr int kPlanThreads = 1024;

// State checks of sequence b for a block of T tokens and S summaries.
__host__ __device__ __forceinline__ int chunk_state_code(const Args &a, int b, int T, int S, int32_t *n0p, int32_t *m0p)
{
    const int32_t *st = a.state + 4 * (int64_t)b;
    const int32_t n0 = st[0], m0 = st[1];
    *n0p = n0; *m0p = m0;
    if (st[3] != 0) return st[3];
    const int64_t f0 = (int64_t)n0 - (int64_t)m0 * a.k;
    if (n0 < 0 || m0 < 0 || f0 < 0 || f0 > a.k || (int64_t)S != (f0 + T) / a.k) return KSA_ERR_STATE;
    if ((int64_t)m0 + S > a.cap || (int64_t)n0 + T > (int64_t)INT32_MAX) return KSA_ERR_CAPACITY;
    return KSA_OK;
}

// (chunk_state_code and chunk_ranges are host-callable too, for CPU tests.)
// Chunks of the tensor-core path for a valid sequence: query chunks
// [cbeg, ncb) and window chunks [kvb, ncb), kvb covering both the first
// query chunk's window and the chunk of the first new summary.
__host__ __device__ __forceinline__ void chunk_ranges(const Args &a, int32_t n0, int32_t m0, int T, int *cbeg, int *kvb,
                                             int *ncb)
{
    const int64_t n1 = (int64_t)n0 + T;
    *cbeg = n0 / a.k;
    *ncb = (int)((n1 + a.k - 1) / a.k);
    *kvb = max(0, min(*cbeg - a.w, m0));
}

__global__ void __launch_bounds__(kPlanThreads) chunk_plan_kernel(Args a, int reset_err)
{
    constexpr int NA = 5;   // text blocks, summary blocks, work units, query chunks, window chunks
    __shared__ int32_t s_sc[NA][kPlanThreads];
    __shared__ int s_bad;
    const int t = threadIdx.x;
    if (t == 0) {
        if (reset_err) *a.err = 0;
        s_bad = 0;
    }
    __syncthreads();
    const int per = (a.batch + kPlanThreads - 1) / kPlanThreads;
    const int b0 = min(a.batch, t * per), b1 = min(a.batch, b0 + per);
    int32_t acc[NA] = {0, 0, 0, 0, 0};
    int bad = 0;
    for (int b = b0; b < b1; ++b) {
        const int T = a.cu_t[b + 1] - a.cu_t[b], S = a.cu_s[b + 1] - a.cu_s[b];
        if (T < 0 || S < 0) { bad = 1; continue; }
        acc[0] += (T + RB - 1) / RB;
        acc[1] += (S + RB - 1) / RB;
        int32_t n0, m0;
        if (a.uc > 0 && T > 0 && chunk_state_code(a, b, T, S, &n0, &m0) == KSA_OK) {
            int cb, kb, nc;
            chunk_ranges(a, n0, m0, T, &cb, &kb, &nc);
            acc[2] += (nc - cb + a.uc - 1) / a.uc;
            acc[3] += nc - cb;
            acc[4] += nc - kb;
        }
    }
    for (int i = 0; i < NA; ++i) s_sc[i][t] = acc[i];
    if (bad) s_bad = 1;
    __syncthreads();
    for (int off = 1; off < kPlanThreads; off <<= 1) {
        int32_t x[NA];
        for (int i = 0; i < NA; ++i) x[i] = t >= off ? s_sc[i][t - off] : 0;
        __syncthreads();
        for (int i = 0; i < NA; ++i) s_sc[i][t] += x[i];
        __syncthreads();
    }
    const bool cu_ok = !s_bad && a.cu_t[0] == 0 && a.cu_s[0] == 0 && (int64_t)a.cu_t[a.batch] == a.total_t &&
                       (int64_t)a.cu_s[a.batch] == a.total_s;
    if (!cu_ok) {
        if (t == 0) set_error(a.err, KSA_ERR_INVALID);
        return;
    }
    int32_t o[NA];
    for (int i = 0; i < NA; ++i) o[i] = t ? s_sc[i][t - 1] : 0;
    for (int b = b0; b < b1; ++b) {
        const int T = a.cu_t[b + 1] - a.cu_t[b], S = a.cu_s[b + 1] - a.cu_s[b];
        int32_t n0, m0;
        const int code = chunk_state_code(a, b, T, S, &n0, &m0);
        if (code != KSA_OK && a.state[4 * (int64_t)b + 3] == 0) a.state[4 * (int64_t)b + 3] = code;
        const int ok = code == KSA_OK;
        a.snap[b] = Snap{n0, m0, ok, 0};
        a.tb_off[b] = o[0];
        a.sb_off[b] = o[1];
        o[0] += (T + RB - 1) / RB;
        o[1] += (S + RB - 1) / RB;
        if (a.uc > 0) {
            int cb = 0, kb = 0, nc = 0;
            if (ok && T > 0) chunk_ranges(a, n0, m0, T, &cb, &kb, &nc);
            a.uoff[b] = o[2]; a.qoff[b] = o[3]; a.kvoff[b] = o[4];
            a.cbeg[b] = cb; a.kvbeg[b] = kb; a.ntot[b] = n0 + T;
            a.qbase[b] = o[3] - cb; a.kvbase[b] = o[4] - kb;
            if (ok && T > 0) {
                o[2] += (nc - cb + a.uc - 1) / a.uc;
                o[3] += nc - cb;
                o[4] += nc - kb;
            }
        }
    }
    if (t == kPlanThreads - 1) {
        a.tb_off[a.batch] = s_sc[0][t];
        a.sb_off[a.batch] = s_sc[1][t];
        if (a.uc > 0) {
            a.uoff[a.batch] = s_sc[2][t];
            a.qoff[a.batch] = s_sc[3][t];
            a.kvoff[a.batch] = s_sc[4][t];
        }
    }
}

// ---------------------------------------------------------------------------
// RoPE of the block's q and k: text token t of sequence b at position n0 + t,
// new summary s at position (m0 + s) k + k - 1 (its chunk's last token).  One
// (cos, sin) table per row, shared by the heads; the same routines as the
// RoPE + interleave and the cache append, so a key rotated here is bitwise the
// key those calls produce.
// ---------------------------------------------------------------------------
constexpr int kRopeThreads = 256;
constexpr int kRopeRows = 4;

__global__ void __launch_bounds__(kRopeThreads) chunk_rope_kernel(Args a)
{
    __shared__ float s_cos[kRopeRows][64], s_sin[kRopeRows][64];
    __shared__ int64_t s_src[kRopeRows];   // input row, -1 = nothing to do
    __shared__ int s_sum[kRopeRows];
    __shared__ int64_t s_pos[kRopeRows];
    if (*a.err != 0) return;
    const int t = threadIdx.x, half = a.d / 2;
    const int64_t row0 = (int64_t)blockIdx.x * kRopeRows;
    if (t < kRopeRows) {
        const int64_t R = row0 + t;
        int64_t src = -1, pos = 0;
        int is_sum = 0;
        if (R < a.total_t + a.total_s) {
            is_sum = R >= a.total_t;
            const int64_t i = is_sum ? R - a.total_t : R;
            const int32_t *cu = is_sum ? a.cu_s : a.cu_t;
            const int b = find_seq(cu, a.batch, (int)i);
            const Snap sn = a.snap[b];
            if (sn.ok) {
                src = i;
                const int64_t loc = i - cu[b];
                pos = is_sum ? ((int64_t)sn.m0 + loc) * a.k + a.k - 1 : (int64_t)sn.n0 + loc;
            }
        }
        s_src[t] = src; s_sum[t] = is_sum; s_pos[t] = pos;
    }
    __syncthreads();
    for (int e = t; e < kRopeRows * half; e += kRopeThreads) {
        const int r = e / half, pr = e % half;
        float c = 1.f, s = 0.f;
        if (a.rotate && s_src[r] >= 0) rope_cos_sin((double)s_pos[r], pr, a.d, a.log2_theta, &c, &s);
        s_cos[r][pr] = c;
        s_sin[r][pr] = s;
    }
    __syncthreads();
    const int ch = half / 8;                 // 16-byte chunks per half head row
    const int qv = a.Hq * ch, kv = a.Hkv * ch;
    for (int e = t; e < kRopeRows * (qv + kv); e += kRopeThreads) {
        const int r = e / (qv + kv), it = e % (qv + kv);
        const int64_t src = s_src[r];
        if (src < 0) continue;
        const bool isq = it < qv;
        const int j = isq ? it : it - qv, H = isq ? a.Hq : a.Hkv;
        const int h = j / ch, c = j % ch;
        const __nv_bfloat16 *in = isq ? (s_sum[r] ? a.qs : a.qt) : (s_sum[r] ? a.ks : a.kt);
        __nv_bfloat16 *out = isq ? (s_sum[r] ? a.qsr : a.qtr) : (s_sum[r] ? a.ksr : a.ktr);
        const int64_t base = (src * H + h) * (a.d / 8);
        uint4 lo = reinterpret_cast<const uint4 *>(in)[base + c];
        uint4 hi = reinterpret_cast<const uint4 *>(in)[base + c + ch];
        rope_rot8(lo, hi, s_cos[r] + 8 * c, s_sin[r] + 8 * c);
        reinterpret_cast<uint4 *>(out)[base + c] = lo;
        reinterpret_cast<uint4 *>(out)[base + c + ch] = hi;
    }
}

// ---------------------------------------------------------------------------
// Attention.  Keys are named by kind and index within the sequence: text by
// absolute position p, summaries by chunk j.
// ---------------------------------------------------------------------------

// K and V rows (D elements) of a key of sequence b, kv head g.
template <int D>
__host__ __device__ __forceinline__ void key_rows(const Args &a, const Snap &sn, int b, int g, int kind, int idx,
                                         const __nv_bfloat16 *&pk, const __nv_bfloat16 *&pv)
{
    const int64_t cache_row = ((int64_t)b * a.Hkv + g) * a.S;
    if (kind == SUM_ROWS) {
        if (idx >= sn.m0) {
            const int64_t r = ((int64_t)a.cu_s[b] + idx - sn.m0) * a.Hkv + g;
            pk = a.ksr + r * D; pv = a.vs + r * D;
        } else {
            const int64_t slot = 1 + a.k + (int64_t)a.w * a.k + idx;
            pk = a.ck + (cache_row + slot) * D; pv = a.cv + (cache_row + slot) * D;
        }
        return;
    }
    if (idx >= sn.n0) {
        const int64_t r = ((int64_t)a.cu_t[b] + idx - sn.n0) * a.Hkv + g;
        pk = a.ktr + r * D; pv = a.vt + r * D;
        return;
    }
    // a cached token: the open chunk m0 (slot k - r) or a ring block
    const int c = idx / a.k, r = idx - c * a.k;
    int64_t slot;
    if (c >= sn.m0) slot = a.k - r;
    else slot = a.w > 0 ? a.k + 1 + (int64_t)(c % a.w) * a.k + (a.k - 1 - r) : 0;
    pk = a.ck + (cache_row + slot) * D; pv = a.cv + (cache_row + slot) * D;
}

template <int D>
__global__ void __launch_bounds__(kThreads) chunk_attn_kernel(Args a)
{
    constexpr int KC = D / 16, NT = D / 8, V8 = D / 8;
    using Row = __nv_bfloat16[D + 8];
    extern __shared__ __align__(16) uint8_t ck_smem[];
    Row *sKV = reinterpret_cast<Row *>(ck_smem);   // two buffers of (K, V), RB rows each
    if (*a.err != 0) return;
    const int nt = a.tb_off[a.batch], ns = a.sb_off[a.batch];
    const int x = blockIdx.x;
    int kind, id;
    if (x < nt) { kind = TEXT_ROWS; id = nt - 1 - x; }   // late text blocks first
    else if (x < nt + ns) { kind = SUM_ROWS; id = x - nt; }
    else return;
    const int32_t *off = kind == TEXT_ROWS ? a.tb_off : a.sb_off;
    const int b = find_seq(off, a.batch, id);
    const Snap sn = a.snap[b];
    if (!sn.ok) return;
    const int32_t *cu = kind == TEXT_ROWS ? a.cu_t : a.cu_s;
    const int idx0 = (id - off[b]) * RB;
    const int cnt = min(RB, cu[b + 1] - cu[b] - idx0);
    const int h = blockIdx.y, g = h / a.G;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gr = lane >> 2, tt = lane & 3;
    const int64_t in0 = (int64_t)cu[b] + idx0;   // first input row of the block
    const int k = a.k, w = a.w;

    // query positions (text) or chunks (summaries) and the key ranges they see
    const int q0 = (kind == TEXT_ROWS ? sn.n0 : sn.m0) + idx0, q1 = q0 + cnt - 1;
    int s_lo, s_hi, t_lo, t_hi;
    if (kind == TEXT_ROWS) {
        const int ca = q0 / k, cb = q1 / k;
        s_lo = 0; s_hi = max(0, cb - w);
        t_lo = max(0, ca - w) * k; t_hi = q1 + 1;
    } else {
        s_lo = q0; s_hi = q1 + 1;
        t_lo = q0 * k; t_hi = (q1 + 1) * k;
    }
    const int nsb = (s_hi - s_lo + RB - 1) / RB, ntb = (t_hi - t_lo + RB - 1) / RB, nkb = nsb + ntb;
    // per-row visible ranges: text keys [lt_lo, lt_hi], summary keys [ls_lo, ls_hi)
    int lt_lo[2], lt_hi[2], ls_lo[2], ls_hi[2];
    bool live[2];
#pragma unroll
    for (int xr = 0; xr < 2; ++xr) {
        const int r = 16 * warp + gr + 8 * xr;
        live[xr] = r < cnt;
        const int q = q0 + r;
        if (!live[xr]) { lt_lo[xr] = 1; lt_hi[xr] = 0; ls_lo[xr] = ls_hi[xr] = 0; }
        else if (kind == TEXT_ROWS) {
            const int c = q / k;
            lt_lo[xr] = max(0, c - w) * k; lt_hi[xr] = q; ls_lo[xr] = 0; ls_hi[xr] = max(0, c - w);
        } else {
            lt_lo[xr] = q * k; lt_hi[xr] = q * k + k - 1; ls_lo[xr] = q; ls_hi[xr] = q + 1;
        }
    }
    auto key_block = [&](int kb, int &kk, int &k0, int &kc) {
        if (kb < nsb) { kk = SUM_ROWS; k0 = s_lo + kb * RB; kc = min(RB, s_hi - k0); }
        else { kk = TEXT_ROWS; k0 = t_lo + (kb - nsb) * RB; kc = min(RB, t_hi - k0); }
    };
    auto prefetch = [&](int kb) {   // key block kb -> buffer kb % 2 (one commit group)
        int kk, k0, kc;
        key_block(kb, kk, k0, kc);
        Row *bK = sKV + (kb & 1) * 2 * RB, *bV = bK + RB;
        for (int e = threadIdx.x; e < RB * V8; e += kThreads) {
            const int r = e / V8, c8 = e % V8;
            if (r < kc) {
                const __nv_bfloat16 *pk, *pv;
                key_rows<D>(a, sn, b, g, kk, k0 + r, pk, pv);
                wm::cp_async16(&bK[r][c8 * 8], pk + c8 * 8);
                wm::cp_async16(&bV[r][c8 * 8], pv + c8 * 8);
            } else {
                *reinterpret_cast<uint4 *>(&bK[r][c8 * 8]) = make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4 *>(&bV[r][c8 * 8]) = make_uint4(0, 0, 0, 0);
            }
        }
        wm::cp_commit();
    };

    // Q of this head through buffer 1 (free until key block 1 is fetched)
    {
        Row *sQ = sKV + 2 * RB;
        const __nv_bfloat16 *qsrc = kind == TEXT_ROWS ? a.qtr : a.qsr;
        for (int e = threadIdx.x; e < RB * V8; e += kThreads) {
            const int r = e / V8, c8 = e % V8;
            uint4 v = make_uint4(0, 0, 0, 0);
            if (r < cnt) v = reinterpret_cast<const uint4 *>(qsrc + ((in0 + r) * a.Hq + h) * D)[c8];
            *reinterpret_cast<uint4 *>(&sQ[r][c8 * 8]) = v;
        }
    }
    if (nkb > 0) prefetch(0);
    __syncthreads();
    uint32_t qf[KC][4];
#pragma unroll
    for (int c = 0; c < KC; ++c) wm::frag_a<D>(qf[c], sKV + 2 * RB, 16 * warp, 16 * c);
    __syncthreads();   // buffer 1 may now take key block 1

    float acc[NT][4];
#pragma unroll
    for (int i = 0; i < NT; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
    float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
    // every query row of the block sees every key of a block when ...
    const int ca = q0 / k, cb = q1 / k;
    for (int kb = 0; kb < nkb; ++kb) {
        int kk, k0, kc;
        key_block(kb, kk, k0, kc);
        if (kb + 1 < nkb) {
            prefetch(kb + 1);
            wm::cp_wait<1>();
        } else {
            wm::cp_wait<0>();
        }
        __syncthreads();   // key block kb has landed for every thread
        const Row *sK = sKV + (kb & 1) * 2 * RB, *sV = sK + RB;
        // ... it is whole and lies inside every row's range (text queries only)
        bool full = kc == RB && kind == TEXT_ROWS;
        if (full) full = kk == SUM_ROWS ? k0 + kc - 1 < ca - w : (k0 + kc - 1 <= q0 && k0 >= max(0, cb - w) * k);
        float s[8][4];
#pragma unroll
        for (int i = 0; i < 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = 0.f;
#pragma unroll
        for (int c = 0; c < KC; ++c)
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                uint32_t bk[4];
                wm::frag_b_nk<D>(bk, sK, 16 * np, 16 * c);
                wm::mma16816(s[2 * np], qf[c][0], qf[c][1], qf[c][2], qf[c][3], bk[0], bk[1]);
                wm::mma16816(s[2 * np + 1], qf[c][0], qf[c][1], qf[c][2], qf[c][3], bk[2], bk[3]);
            }
        // scores in log2 units, masked; row maxima over the quad
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int n8 = 0; n8 < 8; ++n8)
#pragma unroll
            for (int z = 0; z < 4; ++z) {
                const int xr = z >> 1;
                float v = s[n8][z] * a.scale_log2;
                if (!full) {
                    const int col = 8 * n8 + 2 * tt + (z & 1), key = k0 + col;
                    const bool vis = col < kc && (kk == TEXT_ROWS ? (key >= lt_lo[xr] && key <= lt_hi[xr])
                                                                  : (key >= ls_lo[xr] && key < ls_hi[xr]));
                    if (!vis) v = -INFINITY;
                }
                s[n8][z] = v;
                mx[xr] = fmaxf(mx[xr], v);
            }
        float base[2], alpha[2];
#pragma unroll
        for (int xr = 0; xr < 2; ++xr) {
            mx[xr] = fmaxf(mx[xr], __shfl_xor_sync(0xffffffffu, mx[xr], 1));
            mx[xr] = fmaxf(mx[xr], __shfl_xor_sync(0xffffffffu, mx[xr], 2));
            const float mn = fmaxf(mrow[xr], mx[xr]);
            base[xr] = mn == -INFINITY ? 0.f : mn;   // a row with nothing visible yet keeps p = 0
            alpha[xr] = wm::ex2(mrow[xr] - base[xr]);
            mrow[xr] = mn;
            lrow[xr] *= alpha[xr];
        }
        if (__any_sync(0xffffffffu, alpha[0] != 1.f || alpha[1] != 1.f)) {
#pragma unroll
            for (int i = 0; i < NT; ++i) {
                acc[i][0] *= alpha[0]; acc[i][1] *= alpha[0];
                acc[i][2] *= alpha[1]; acc[i][3] *= alpha[1];
            }
        }
        // P (bf16 A fragments of 16 keys each) and the row sums
        uint32_t pf[4][4];
#pragma unroll
        for (int n8 = 0; n8 < 8; ++n8) {
            float e[4];
#pragma unroll
            for (int z = 0; z < 4; ++z) {
                e[z] = wm::ex2(s[n8][z] - base[z >> 1]);
                lrow[z >> 1] += e[z];
            }
            const int j = n8 >> 1;
            if ((n8 & 1) == 0) { pf[j][0] = wm::pack2(e[0], e[1]); pf[j][1] = wm::pack2(e[2], e[3]); }
            else { pf[j][2] = wm::pack2(e[0], e[1]); pf[j][3] = wm::pack2(e[2], e[3]); }
        }
        // O += P V (k = keys, n = dims)
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int np = 0; np < NT / 2; ++np) {
                uint32_t bv[4];
                wm::frag_b_kn<D>(bv, sV, 16 * j, 16 * np);
                wm::mma16816(acc[2 * np], pf[j][0], pf[j][1], pf[j][2], pf[j][3], bv[0], bv[1]);
                wm::mma16816(acc[2 * np + 1], pf[j][0], pf[j][1], pf[j][2], pf[j][3], bv[2], bv[3]);
            }
        __syncthreads();   // buffer kb % 2 is read: the next prefetch may overwrite it
    }
    // o = acc / l; lse = ln(l) + max (natural log)
    __nv_bfloat16 *obase = kind == TEXT_ROWS ? a.ot : a.os;
    float *lbase = kind == TEXT_ROWS ? a.lt : a.ls;
#pragma unroll
    for (int xr = 0; xr < 2; ++xr) {
        float l = lrow[xr];
        l += __shfl_xor_sync(0xffffffffu, l, 1);
        l += __shfl_xor_sync(0xffffffffu, l, 2);
        if (!live[xr]) continue;
        const int64_t row = in0 + 16 * warp + gr + 8 * xr;
        const float inv = 1.f / l;
        __nv_bfloat16 *dst = obase + (row * a.Hq + h) * D;
#pragma unroll
        for (int i = 0; i < NT; ++i)
            *reinterpret_cast<uint32_t *>(dst + 8 * i + 2 * tt) = wm::pack2(acc[i][2 * xr] * inv, acc[i][2 * xr + 1] * inv);
        if (lbase && tt == 0) lbase[row * a.Hq + h] = (mrow[xr] + log2f(l)) * 0.69314718055994531f;
    }
}

// ---------------------------------------------------------------------------
// Summary rows of the block: summary s_j sees the k text tokens of chunk j
// and itself (section 2.2.1), k + 1 keys.  One warp per (new summary, kv
// head): the keys are the rows of a 16-row MMA tile (S^T = K Q^T with the G
// query heads of the kv head as MMA columns, O^T = V^T P^T), 16 keys per
// step with an online softmax across steps.  Lane (g, t) loads dims
// [32v + 8t, +8) of key rows g and g + 8 with 16-byte loads and hands the
// words to the MMA unchanged; q is loaded in the same permuted order, so the
// dot products are unchanged.  A key row is read where it lives: a token of
// the open chunk from its cache slot, a new token from the block, the
// summary from the block.
// ---------------------------------------------------------------------------
constexpr int kSumWarps = 4;

template <int D, int G>
__global__ void __launch_bounds__(kSumWarps * 32) chunk_sum_kernel(Args a)
{
    static_assert(G <= 8, "query heads per kv head must fit the 8 MMA columns");
    constexpr int NV = D / 32, NC = D / 16, NM = D / 16;
    __shared__ float s_o[kSumWarps][G][D];
    __shared__ float s_ml[kSumWarps][2][G];
    if (*a.err != 0) return;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t task = (int64_t)blockIdx.x * kSumWarps + warp;
    if (task >= a.total_s * a.Hkv) return;   // warp-uniform; only warp-level syncs below
    const int64_t row = task / a.Hkv;         // the summary's input row
    const int h = (int)(task % a.Hkv);
    const int b = find_seq(a.cu_s, a.batch, (int)row);
    const Snap sn = a.snap[b];
    if (!sn.ok) return;
    const int64_t j = sn.m0 + (row - a.cu_s[b]);   // its chunk
    const int g = lane >> 2, tt = lane & 3;
    uint32_t qb[NC][2];
#pragma unroll
    for (int c = 0; c < NC; ++c) {
        const int d0 = 32 * (c / 2) + 8 * tt + 4 * (c % 2);
        if (g < G) {
            const uint32_t *qp = reinterpret_cast<const uint32_t *>(a.qsr + (row * a.Hq + (int64_t)h * G + g) * D + d0);
            qb[c][0] = qp[0];
            qb[c][1] = qp[1];
        } else {
            qb[c][0] = qb[c][1] = 0u;
        }
    }
    // uint4 base of key row r (r < k: text position j k + r; r = k: the summary)
    auto key_row = [&](int r, const uint4 *&kp, const uint4 *&vp) {
        int64_t off;
        if (r == a.k) {
            off = (row * a.Hkv + h) * (D / 8);
            kp = reinterpret_cast<const uint4 *>(a.ksr) + off;
            vp = reinterpret_cast<const uint4 *>(a.vs) + off;
            return;
        }
        const int64_t p = j * a.k + r;
        if (p < sn.n0) {   // a token of the open chunk m0, cached at slot k - r
            off = (((int64_t)b * a.Hkv + h) * a.S + (a.k - (p - (int64_t)sn.m0 * a.k))) * (D / 8);
            kp = reinterpret_cast<const uint4 *>(a.ck) + off;
            vp = reinterpret_cast<const uint4 *>(a.cv) + off;
        } else {
            off = (((int64_t)a.cu_t[b] + p - sn.n0) * a.Hkv + h) * (D / 8);
            kp = reinterpret_cast<const uint4 *>(a.ktr) + off;
            vp = reinterpret_cast<const uint4 *>(a.vt) + off;
        }
    };
    float o[NM][4];
#pragma unroll
    for (int i = 0; i < NM; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};   // heads 2tt, 2tt + 1 (log2 units)
    for (int kb = 0; kb <= a.k; kb += 16) {
        const int r0 = kb + g, r1 = kb + g + 8;
        const bool in0 = r0 <= a.k, in1 = r1 <= a.k;
        const uint4 *k0p = nullptr, *v0p = nullptr, *k1p = nullptr, *v1p = nullptr;
        if (in0) key_row(r0, k0p, v0p);
        if (in1) key_row(r1, k1p, v1p);
        uint4 kA[NV], kB[NV], vA[NV], vB[NV];
#pragma unroll
        for (int v = 0; v < NV; ++v) {
            const uint4 z = make_uint4(0, 0, 0, 0);
            kA[v] = in0 ? k0p[4 * v + tt] : z;
            kB[v] = in1 ? k1p[4 * v + tt] : z;
            vA[v] = in0 ? v0p[4 * v + tt] : z;
            vB[v] = in1 ? v1p[4 * v + tt] : z;
        }
        float sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            const int v = c / 2, hh = c % 2;
            wm::mma16816(sc, wm::word(kA[v], 2 * hh), wm::word(kB[v], 2 * hh), wm::word(kA[v], 2 * hh + 1),
                         wm::word(kB[v], 2 * hh + 1), qb[c][0], qb[c][1]);
        }
        float x[4];
        x[0] = in0 ? sc[0] * a.scale_log2 : -INFINITY;
        x[1] = in0 ? sc[1] * a.scale_log2 : -INFINITY;
        x[2] = in1 ? sc[2] * a.scale_log2 : -INFINITY;
        x[3] = in1 ? sc[3] * a.scale_log2 : -INFINITY;
        float corr[2], pv[4];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            float mx = fmaxf(x[e], x[e + 2]);
#pragma unroll
            for (int off = 4; off < 32; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
            const float m_new = fmaxf(m_run[e], mx);   // finite: key 0 is always present
            corr[e] = wm::ex2(m_run[e] - m_new);
            pv[e] = wm::ex2(x[e] - m_new);
            pv[e + 2] = wm::ex2(x[e + 2] - m_new);
            l_run[e] = l_run[e] * corr[e] + pv[e] + pv[e + 2];
            m_run[e] = m_new;
        }
#pragma unroll
        for (int i = 0; i < NM; ++i) {
            o[i][0] *= corr[0]; o[i][1] *= corr[1];
            o[i][2] *= corr[0]; o[i][3] *= corr[1];
        }
        const uint32_t pb0 = wm::movtrans(wm::pack2(pv[0], pv[1]));
        const uint32_t pb1 = wm::movtrans(wm::pack2(pv[2], pv[3]));
#pragma unroll
        for (int i = 0; i < NM; ++i) {
            const int v = i / 2, pp = i % 2;
            wm::mma16816(o[i], wm::movtrans(wm::word(vA[v], 2 * pp)), wm::movtrans(wm::word(vA[v], 2 * pp + 1)),
                         wm::movtrans(wm::word(vB[v], 2 * pp)), wm::movtrans(wm::word(vB[v], 2 * pp + 1)), pb0, pb1);
        }
    }
#pragma unroll
    for (int e = 0; e < 2; ++e)
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) l_run[e] += __shfl_xor_sync(0xffffffffu, l_run[e], off);
    // O^T rows: m-tile i = (v, pp), row g -> dim 32v + 8(g/2) + 4pp + (g%2), row g+8 -> that + 2
#pragma unroll
    for (int i = 0; i < NM; ++i) {
        const int v = i / 2, pp = i % 2;
        const int dA = 32 * v + 8 * (g / 2) + 4 * pp + (g % 2);
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int head = 2 * tt + e;
            if (head < G) {
                s_o[warp][head][dA] = o[i][e];
                s_o[warp][head][dA + 2] = o[i][2 + e];
            }
        }
    }
    if (g == 0) {
#pragma unroll
        for (int e = 0; e < 2; ++e)
            if (2 * tt + e < G) {
                s_ml[warp][0][2 * tt + e] = m_run[e];
                s_ml[warp][1][2 * tt + e] = l_run[e];
            }
    }
    __syncwarp();
    for (int idx = lane; idx < G * (D / 2); idx += 32) {
        const int gg = idx / (D / 2), w2 = idx % (D / 2);
        const float inv = 1.f / s_ml[warp][1][gg];
        const uint32_t pr = wm::pack2(s_o[warp][gg][2 * w2] * inv, s_o[warp][gg][2 * w2 + 1] * inv);
        reinterpret_cast<uint32_t *>(a.os + (row * a.Hq + (int64_t)h * G + gg) * D)[w2] = pr;
    }
    if (a.ls && lane < G)
        a.ls[row * a.Hq + (int64_t)h * G + lane] =
            (s_ml[warp][0][lane] + log2f(s_ml[warp][1][lane])) * 0.69314718055994530942f;
}

// ---------------------------------------------------------------------------
// Tensor-core path helpers.
// ---------------------------------------------------------------------------
constexpr int kCopyThreads = 256;

// The block's summaries (rotated K, V) into slots 1 + k + w k + m0 + s.  No
// query of this call reads those slots through the warp-level kernel (it
// takes new summaries from the workspace), and no earlier state reads them.
__global__ void __launch_bounds__(kCopyThreads) chunk_sumwrite_kernel(Args a)
{
    if (*a.err != 0) return;
    const int V8 = a.d / 8;
    const int64_t items = a.total_s * a.Hkv * V8;
    const uint4 *ks = reinterpret_cast<const uint4 *>(a.ksr), *vs = reinterpret_cast<const uint4 *>(a.vs);
    for (int64_t e = (int64_t)blockIdx.x * kCopyThreads + threadIdx.x; e < items;
         e += (int64_t)gridDim.x * kCopyThreads) {
        const int64_t row = e / ((int64_t)a.Hkv * V8), rem = e % ((int64_t)a.Hkv * V8);
        const int g = (int)(rem / V8), c = (int)(rem % V8);
        const int b = find_seq(a.cu_s, a.batch, (int)row);
        const Snap sn = a.snap[b];
        if (!sn.ok) continue;
        const int64_t slot = 1 + a.k + (int64_t)a.w * a.k + sn.m0 + (row - a.cu_s[b]);
        const int64_t dst = (((int64_t)b * a.Hkv + g) * a.S + slot) * V8 + c;
        reinterpret_cast<uint4 *>(a.ck)[dst] = ks[e];
        reinterpret_cast<uint4 *>(a.cv)[dst] = vs[e];
    }
}

// One CTA per chunk of the gathered buffers (grid = the window buffer's
// extent, which is at least the query buffer's).  Window chunk x of sequence
// b is absolute chunk kvbeg + (x - kvoff): text slot r holds position
// c k + r from the cache (older than the block), the block, or zero past
// the block; the summary slot is zero (summary keys come from the cache).
// Query chunk x likewise: the rotated q of new positions, zero elsewhere.
// Chunks past the last sequence are zero, so no tile ever loads stale bytes.
__global__ void __launch_bounds__(kCopyThreads) chunk_gather_kernel(Args a)
{
    if (*a.err != 0) return;
    const int x = blockIdx.x, V8 = a.d / 8;
    const uint4 zero = make_uint4(0, 0, 0, 0);
    // window rows (K and V)
    {
        const int nkv = a.kvoff[a.batch];
        int b = -1;
        int64_t c = 0;
        if (x < nkv) {
            b = find_seq(a.kvoff, a.batch, x);
            c = (int64_t)a.kvbeg[b] + (x - a.kvoff[b]);
        }
        uint4 *dk = reinterpret_cast<uint4 *>(a.ka) + (int64_t)x * (a.k + 1) * a.Hkv * V8;
        uint4 *dv = reinterpret_cast<uint4 *>(a.va) + (int64_t)x * (a.k + 1) * a.Hkv * V8;
        const int items = (a.k + 1) * a.Hkv * V8;
        for (int e = threadIdx.x; e < items; e += kCopyThreads) {
            const int r = e / (a.Hkv * V8), rem = e % (a.Hkv * V8), g = rem / V8, cc = rem % V8;
            uint4 kv = zero, vv = zero;
            if (b >= 0 && r < a.k) {
                const Snap sn = a.snap[b];
                const int64_t p = c * a.k + r;
                if (p < sn.n0) {
                    const int64_t cp = p / a.k, rr = p - cp * a.k;
                    int64_t slot;
                    if (cp >= sn.m0) slot = a.k - rr;
                    else slot = a.w > 0 ? a.k + 1 + (cp % a.w) * a.k + (a.k - 1 - rr) : 0;
                    const int64_t row = ((int64_t)b * a.Hkv + g) * a.S + slot;
                    kv = reinterpret_cast<const uint4 *>(a.ck)[row * V8 + cc];
                    vv = reinterpret_cast<const uint4 *>(a.cv)[row * V8 + cc];
                } else if (p < a.ntot[b]) {
                    const int64_t row = ((int64_t)a.cu_t[b] + p - sn.n0) * a.Hkv + g;
                    kv = reinterpret_cast<const uint4 *>(a.ktr)[row * V8 + cc];
                    vv = reinterpret_cast<const uint4 *>(a.vt)[row * V8 + cc];
                }
            }
            dk[e] = kv;
            dv[e] = vv;
        }
    }
    // query rows
    if (x < a.q_chunks) {
        const int nq = a.qoff[a.batch];
        int b = -1;
        int64_t c = 0;
        if (x < nq) {
            b = find_seq(a.qoff, a.batch, x);
            c = (int64_t)a.cbeg[b] + (x - a.qoff[b]);
        }
        uint4 *dq = reinterpret_cast<uint4 *>(a.qa) + (int64_t)x * (a.k + 1) * a.Hq * V8;
        const int items = (a.k + 1) * a.Hq * V8;
        for (int e = threadIdx.x; e < items; e += kCopyThreads) {
            const int r = e / (a.Hq * V8), rem = e % (a.Hq * V8), h = rem / V8, cc = rem % V8;
            uint4 qv = zero;
            if (b >= 0 && r < a.k) {
                const int64_t p = c * a.k + r, n0 = a.snap[b].n0;
                if (p >= n0 && p < a.ntot[b]) {
                    const int64_t row = ((int64_t)a.cu_t[b] + p - n0) * a.Hq + h;
                    qv = reinterpret_cast<const uint4 *>(a.qtr)[row * V8 + cc];
                }
            }
            dq[e] = qv;
        }
    }
}

// The new text rows' outputs (and LSE) from the gathered layout to
// [total_text, Hq, d]: one CTA per row.
__global__ void __launch_bounds__(kCopyThreads) chunk_scatter_kernel(Args a)
{
    if (*a.err != 0) return;
    const int64_t i = blockIdx.x;
    const int b = find_seq(a.cu_t, a.batch, (int)i);
    const Snap sn = a.snap[b];
    if (!sn.ok) return;
    const int64_t p = sn.n0 + (i - a.cu_t[b]);
    const int64_t row = ((int64_t)a.qbase[b] + p / a.k) * (a.k + 1) + p % a.k;
    const int V8 = a.d / 8;
    const uint4 *src = reinterpret_cast<const uint4 *>(a.oa) + row * a.Hq * V8;
    uint4 *dst = reinterpret_cast<uint4 *>(a.ot) + i * a.Hq * V8;
    for (int e = threadIdx.x; e < a.Hq * V8; e += kCopyThreads) dst[e] = src[e];
    if (a.lt)
        for (int h = threadIdx.x; h < a.Hq; h += kCopyThreads) a.lt[i * a.Hq + h] = a.la[row * a.Hq + h];
}

// ---------------------------------------------------------------------------
// Extend the cache of (sequence, kv head) by the block (Figure 4):
//  (4d) when the block completes the open chunk m0, that chunk's f0 cached
//       tokens move from slots k - r to its ring block (if it is among the
//       last w complete chunks after the call);
//  (4b/4d) each new text token goes to the open chunk's slot k - r when its
//       chunk is still open at the end, else to its chunk's ring block when
//       that chunk is among the last w complete ones, else nowhere (its
//       summary stands for it);
//  (4e) new summary s_j to slot 1 + k + w k + j.
// Then the state becomes {n0 + T, m0 + S}.  Slot 0 and stale slots are left
// as they are: no later decode step reads them before they are rewritten.
// ---------------------------------------------------------------------------
constexpr int kAppendThreads = 256;

__global__ void __launch_bounds__(kAppendThreads) chunk_append_kernel(Args a)
{
    if (*a.err != 0) return;
    const int b = blockIdx.x, g = blockIdx.y, t = threadIdx.x;
    const Snap sn = a.snap[b];
    if (!sn.ok) return;
    const int k = a.k, w = a.w, V8 = a.d / 8;
    const int T = a.cu_t[b + 1] - a.cu_t[b], S = a.cu_s[b + 1] - a.cu_s[b];
    const int64_t n0 = sn.n0, m0 = sn.m0, f0 = n0 - m0 * k, m1 = m0 + S;
    uint4 *K = reinterpret_cast<uint4 *>(a.ck) + ((int64_t)b * a.Hkv + g) * a.S * V8;
    uint4 *V = reinterpret_cast<uint4 *>(a.cv) + ((int64_t)b * a.Hkv + g) * a.S * V8;
    if (S > 0 && w > 0 && m0 >= m1 - w) {
        const int64_t ring = k + 1 + (m0 % w) * k;
        for (int64_t e = t; e < f0 * V8; e += kAppendThreads) {
            const int64_t r = e / V8, c = e % V8;
            K[(ring + k - 1 - r) * V8 + c] = K[(k - r) * V8 + c];
            V[(ring + k - 1 - r) * V8 + c] = V[(k - r) * V8 + c];
        }
    }
    __syncthreads();   // the open chunk's slots are read before new tokens overwrite them
    const uint4 *kt = reinterpret_cast<const uint4 *>(a.ktr), *vt = reinterpret_cast<const uint4 *>(a.vt);
    // only the open chunk and the last w complete chunks are kept: start at
    // the first kept position
    const int64_t keep = max(n0, (w > 0 ? max((int64_t)0, m1 - w) : m1) * k);
    for (int64_t e = (keep - n0) * V8 + t; e < (int64_t)T * V8; e += kAppendThreads) {
        const int64_t tq = e / V8, c = e % V8;
        const int64_t p = n0 + tq, cp = p / k, r = p - cp * k;
        int64_t slot;
        if (cp >= m1) slot = k - r;
        else if (w > 0 && cp >= m1 - w) slot = k + 1 + (cp % w) * k + (k - 1 - r);
        else continue;
        const int64_t src = ((int64_t)a.cu_t[b] + tq) * a.Hkv + g;
        K[slot * V8 + c] = kt[src * V8 + c];
        V[slot * V8 + c] = vt[src * V8 + c];
    }
    const uint4 *ks = reinterpret_cast<const uint4 *>(a.ksr), *vs = reinterpret_cast<const uint4 *>(a.vs);
    // (the tensor-core path wrote the summaries before its attention)
    for (int64_t e = t; e < (a.uc > 0 ? 0 : (int64_t)S * V8); e += kAppendThreads) {
        const int64_t s = e / V8, c = e % V8;
        const int64_t slot = 1 + k + (int64_t)w * k + m0 + s;
        const int64_t src = ((int64_t)a.cu_s[b] + s) * a.Hkv + g;
        K[slot * V8 + c] = ks[src * V8 + c];
        V[slot * V8 + c] = vs[src * V8 + c];
    }
    if (g == 0 && t == 0) {
        int32_t *st = a.state + 4 * (int64_t)b;
        st[0] = (int32_t)(n0 + T);
        st[1] = (int32_t)m1;
    }
}

// ---------------------------------------------------------------------------
// Query chunks of the tensor-core path (0 when the shape is not one the
// prefill kernel takes).
static int tc_unit_chunks(const ksa_params *p)
{
    const int G = p->num_q_heads / p->num_kv_heads;
    if (G != 1 && G != 2 && G != 4 && G != 8) return 0;
    if (p->head_dim != 64 && p->head_dim != 128) return 0;
    return prefill_unit_chunks(p);
}

struct Layout {
    size_t err, snap, tb, sb, qtr, ktr, qsr, ksr;
    size_t arr[8], qa, ka, va, oa, la, total;
    int64_t q_chunks, kv_chunks, max_units;
};

static Layout layout(const ksa_params *p, int batch, int64_t total_t, int64_t total_s)
{
    Layout L;
    const size_t d = (size_t)p->head_dim, Hq = (size_t)p->num_q_heads, Hkv = (size_t)p->num_kv_heads;
    size_t o = 0;
    L.err = o; o += align_up(16);
    L.snap = o; o += align_up(sizeof(Snap) * (size_t)batch);
    L.tb = o; o += align_up(sizeof(int32_t) * (size_t)(batch + 1));
    L.sb = o; o += align_up(sizeof(int32_t) * (size_t)(batch + 1));
    L.qtr = o; o += align_up((size_t)total_t * Hq * d * 2);
    L.ktr = o; o += align_up((size_t)total_t * Hkv * d * 2);
    L.qsr = o; o += align_up((size_t)total_s * Hq * d * 2);
    L.ksr = o; o += align_up((size_t)total_s * Hkv * d * 2);
    const int uc = tc_unit_chunks(p);
    L.q_chunks = L.kv_chunks = L.max_units = 0;
    if (uc > 0 && total_t > 0) {
        // a sequence's query chunks number at most T/k + 2 and its window
        // chunks at most w + 1 more
        L.q_chunks = total_t / p->k + 2LL * batch;
        L.kv_chunks = L.q_chunks + (int64_t)batch * (p->w + 1);
        L.max_units = L.q_chunks / uc + batch;
        for (int i = 0; i < 8; ++i) { L.arr[i] = o; o += align_up(sizeof(int32_t) * (size_t)(batch + 1)); }
        const size_t rows_q = (size_t)L.q_chunks * (p->k + 1), rows_kv = (size_t)L.kv_chunks * (p->k + 1);
        L.qa = o; o += align_up(rows_q * Hq * d * 2);
        L.oa = o; o += align_up(rows_q * Hq * d * 2);
        L.la = o; o += align_up(rows_q * Hq * 4);
        L.ka = o; o += align_up(rows_kv * Hkv * d * 2);
        L.va = o; o += align_up(rows_kv * Hkv * d * 2);
    }
    L.total = o;
    return L;
}

template <int D>
static int launch_attn(const Args &a, int64_t blocks, cudaStream_t st)
{
    const int smem = 4 * RB * (D + 8) * (int)sizeof(__nv_bfloat16);
    if (cudaFuncSetAttribute(chunk_attn_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return KSA_ERR_CUDA;
    dim3 grid((unsigned)blocks, (unsigned)a.Hq);
    chunk_attn_kernel<D><<<grid, kThreads, smem, st>>>(a);
    return cudaGetLastError() == cudaSuccess ? KSA_OK : KSA_ERR_CUDA;
}

template <int D>
static int launch_sum_d(int G, const Args &a, unsigned blocks, cudaStream_t st)
{
    switch (G) {
    case 1: chunk_sum_kernel<D, 1><<<blocks, kSumWarps * 32, 0, st>>>(a); break;
    case 2: chunk_sum_kernel<D, 2><<<blocks, kSumWarps * 32, 0, st>>>(a); break;
    case 4: chunk_sum_kernel<D, 4><<<blocks, kSumWarps * 32, 0, st>>>(a); break;
    case 8: chunk_sum_kernel<D, 8><<<blocks, kSumWarps * 32, 0, st>>>(a); break;
    default: return KSA_ERR_UNSUPPORTED;
    }
    return cudaGetLastError() == cudaSuccess ? KSA_OK : KSA_ERR_CUDA;
}

static int launch_sum(int d, int G, const Args &a, unsigned blocks, cudaStream_t st)
{
    return d == 128 ? launch_sum_d<128>(G, a, blocks, st) : launch_sum_d<64>(G, a, blocks, st);
}

}  // namespace ck

size_t prefill_chunk_workspace_bytes(const ksa_params *p, int batch, int64_t total_text, int64_t total_sum)
{
    return ck::layout(p, batch, total_text, total_sum).total;
}

int launch_prefill_chunk(const ksa_params *p, const ksa_cache *c, const int32_t *cu_t, int64_t total_t,
                         const int32_t *cu_s, int64_t total_s, const void *qt, const void *kt, const void *vt,
                         const void *qs, const void *ks, const void *vs, void *ot, void *os, float *lt, float *ls,
                         void *ws, int32_t *dev_err, cudaStream_t st)
{
    using namespace ck;
    const int B = c->batch;
    const Layout L = layout(p, B, total_t, total_s);
    char *w = static_cast<char *>(ws);
    Args a;
    a.k = p->k; a.w = p->w; a.Hq = p->num_q_heads; a.Hkv = p->num_kv_heads; a.G = a.Hq / a.Hkv;
    a.batch = B; a.d = p->head_dim;
    a.S = 1 + (int64_t)p->k + (int64_t)p->w * p->k + c->cap_summaries;
    a.cap = c->cap_summaries;
    const float scale = p->scale > 0.f ? p->scale : 1.f / sqrtf((float)p->head_dim);
    a.scale_log2 = scale * 1.4426950408889634f;
    a.rotate = p->rope_theta > 0.0;
    a.log2_theta = a.rotate ? log2(p->rope_theta) : 0.0;
    a.cu_t = cu_t; a.cu_s = cu_s; a.total_t = total_t; a.total_s = total_s;
    a.snap = reinterpret_cast<Snap *>(w + L.snap);
    a.tb_off = reinterpret_cast<int32_t *>(w + L.tb);
    a.sb_off = reinterpret_cast<int32_t *>(w + L.sb);
    a.state = c->state;
    int32_t *own_err = reinterpret_cast<int32_t *>(w + L.err);
    a.err = dev_err ? dev_err : own_err;
    a.ck = static_cast<__nv_bfloat16 *>(c->k); a.cv = static_cast<__nv_bfloat16 *>(c->v);
    a.qt = (const __nv_bfloat16 *)qt; a.kt = (const __nv_bfloat16 *)kt; a.vt = (const __nv_bfloat16 *)vt;
    a.qs = (const __nv_bfloat16 *)qs; a.ks = (const __nv_bfloat16 *)ks; a.vs = (const __nv_bfloat16 *)vs;
    a.qtr = reinterpret_cast<__nv_bfloat16 *>(w + L.qtr); a.ktr = reinterpret_cast<__nv_bfloat16 *>(w + L.ktr);
    a.qsr = reinterpret_cast<__nv_bfloat16 *>(w + L.qsr); a.ksr = reinterpret_cast<__nv_bfloat16 *>(w + L.ksr);
    a.ot = (__nv_bfloat16 *)ot; a.os = (__nv_bfloat16 *)os; a.lt = lt; a.ls = ls;
    // tensor-core path for the text rows when the shape allows and the cache
    // coordinates fit the tensor maps
    const bool tc = L.q_chunks > 0 && a.S <= INT32_MAX && L.kv_chunks * (p->k + 1) <= INT32_MAX;
    a.uc = tc ? tc_unit_chunks(p) : 0;
    a.q_chunks = L.q_chunks; a.kv_chunks = L.kv_chunks;
    if (tc) {
        int32_t *arr[8];
        for (int i = 0; i < 8; ++i) arr[i] = reinterpret_cast<int32_t *>(w + L.arr[i]);
        a.cbeg = arr[0]; a.kvbeg = arr[1]; a.ntot = arr[2]; a.qbase = arr[3]; a.kvbase = arr[4];
        a.qoff = arr[5]; a.kvoff = arr[6]; a.uoff = arr[7];
        a.qa = reinterpret_cast<__nv_bfloat16 *>(w + L.qa); a.oa = reinterpret_cast<__nv_bfloat16 *>(w + L.oa);
        a.ka = reinterpret_cast<__nv_bfloat16 *>(w + L.ka); a.va = reinterpret_cast<__nv_bfloat16 *>(w + L.va);
        a.la = reinterpret_cast<float *>(w + L.la);
    } else {
        a.cbeg = a.kvbeg = a.ntot = a.qbase = a.kvbase = a.qoff = a.kvoff = a.uoff = nullptr;
        a.qa = a.oa = a.ka = a.va = nullptr;
        a.la = nullptr;
    }

    chunk_plan_kernel<<<1, kPlanThreads, 0, st>>>(a, a.err == own_err);
    if (cudaGetLastError() != cudaSuccess) return KSA_ERR_CUDA;
    const int64_t rows = total_t + total_s;
    if (rows > 0) {
        const int64_t rb = (rows + kRopeRows - 1) / kRopeRows;
        if (rb > INT32_MAX) return KSA_ERR_UNSUPPORTED;
        chunk_rope_kernel<<<(unsigned)rb, kRopeThreads, 0, st>>>(a);
        if (cudaGetLastError() != cudaSuccess) return KSA_ERR_CUDA;
        if (tc) {
            const int64_t sitems = total_s * a.Hkv * (p->head_dim / 8);
            const int64_t sblocks = sitems > 0 ? min((int64_t)4 * sm_count(), (sitems + kCopyThreads - 1) / kCopyThreads) : 0;
            if (sblocks > 0) chunk_sumwrite_kernel<<<(unsigned)sblocks, kCopyThreads, 0, st>>>(a);
            if (cudaGetLastError() != cudaSuccess) return KSA_ERR_CUDA;
            if (L.kv_chunks > INT32_MAX) return KSA_ERR_UNSUPPORTED;
            chunk_gather_kernel<<<(unsigned)L.kv_chunks, kCopyThreads, 0, st>>>(a);
            if (cudaGetLastError() != cudaSuccess) return KSA_ERR_CUDA;
            ChunkTiles t;
            t.tile_off = a.uoff; t.cbeg = a.cbeg; t.ntot = a.ntot; t.qbase = a.qbase; t.kvbase = a.kvbase;
            t.q_chunks = L.q_chunks; t.kv_chunks = L.kv_chunks; t.max_units = L.max_units;
            t.qa = a.qa; t.ka = a.ka; t.va = a.va; t.oa = a.oa; t.lse = a.la;
            int rc = launch_prefill_cache(p, c, t, a.err, st);
            if (rc != KSA_OK) return rc;
            chunk_scatter_kernel<<<(unsigned)total_t, kCopyThreads, 0, st>>>(a);
            if (cudaGetLastError() != cudaSuccess) return KSA_ERR_CUDA;
        }
        if (tc) {
            // summary rows: one warp per (summary, kv head)
            const int64_t tasks = total_s * a.Hkv;
            if (tasks > 0) {
                const int64_t sb = (tasks + kSumWarps - 1) / kSumWarps;
                if (sb > INT32_MAX) return KSA_ERR_UNSUPPORTED;
                const int rc = launch_sum(p->head_dim, a.G, a, (unsigned)sb, st);
                if (rc != KSA_OK) return rc;
            }
        } else {
            const int64_t blocks = (total_t / RB + B) + (total_s / RB + B);
            if (blocks > INT32_MAX) return KSA_ERR_UNSUPPORTED;
            const int rc = p->head_dim == 128 ? launch_attn<128>(a, blocks, st) : launch_attn<64>(a, blocks, st);
            if (rc != KSA_OK) return rc;
        }
    }
    dim3 grid((unsigned)B, (unsigned)a.Hkv);
    chunk_append_kernel<<<grid, kAppendThreads, 0, st>>>(a);
    return cudaGetLastError() == cudaSuccess ? KSA_OK : KSA_ERR_CUDA;
}

}  // namespace ksa

// prefill_bwd_sm100.cu -- dk, dv of the KSA prefill from the text query rows
// on tcgen05 (TMA -> SMEM -> tcgen05.mma -> TMEM).
//
// Kwai Summary Attention Technical Report: the forward is Eq. (10),
// softmax(Q K^T / sqrt(d) + M_KSA) V, under the mask of section 2.2.2,
// Eqs. (2)-(3): text t_i (chunk c = floor(i/k)) sees the text of chunks
// c-w .. c causally and the summaries s_0 .. s_{c-w-1}.  Read from the key
// side, text key p (chunk c_p) is seen by the text queries p ..
// (c_p + w + 1) k - 1 and summary key j by the text queries from
// (j + w + 1) k on.  The gradients are the textbook ones: P = exp(S - lse),
// dP = dO V^T, dS = P (dP - D) with D = rowsum(dO * O), dv = P^T dO,
// dk = scale dS^T Q.
//
// Design.  A CTA owns one tile of 128 keys of one kind (128 consecutive text
// tokens or 128 consecutive summaries of one sequence) of one kv head: its K
// and V sit in shared memory for the whole CTA and its rows are the 128
// TMEM lanes.  It walks a share of its steps; a step is one q head of the kv
// head's group x NQ consecutive text query positions (TMA boxes over the
// augmented layout's text slots; NQ = 64 when k divides 64, else 128), and
// takes four MMAs:
//     S^T  = K Q^T      (SS, M 128 keys, N NQ queries, K d)
//     dP^T = V dO^T     (SS)
//     dV  += P^T dO     (TS: P^T written as bf16 over S^T, B = dO MN-major)
//     dK  += dS^T Q     (TS: dS^T written as bf16 over dP^T)
// TMEM holds S^T and dP^T (two buffers each at NQ = 64, so the next step's
// products run while this step's accumulations read P^T and dS^T), dV and
// dK.  Eight elementwise warps (two per TMEM lane quarter, NQ / 2 query
// columns each) turn S^T into P^T and dP^T into dS^T; the mask of a key row
// inside a step is one interval of columns, from coordinates.  The summary
// query rows (a summary sees its own chunk and itself) are left to a
// CUDA-core kernel of prefill_bwd.cu.  Shares of the same key tile (long
// summary ranges) add their dK, dV into fp32 accumulators.  All mbarrier
// waits are bounded.
#include <cuda.h>
#include <math.h>

#include "ksa_internal.cuh"
#include "tc_sm100.cuh"

namespace ksa {
namespace bt {

using namespace tc;

constexpr int BK = 128;       // keys per tile (TMEM lanes)
constexpr int BQ = 128;       // query positions per dq tile (MMA M) and per key tile's query tiles of dq
constexpr int HQ = BQ / 2;    // key columns per elementwise warp of dq
constexpr int kWarpTMA = 8;   // K, V once, then Q and dO per step
constexpr int kWarpMMA = 9;   // MMA issuer, TMEM owner
constexpr int kWarpLD = 10;   // per-step LSE and D, zero rows past the sequence
constexpr int kWarpMMA2 = 11; // second MMA issuer (an issuing thread sustains ~70 cycles per MMA)
constexpr int kThreads = 384;
constexpr uint32_t kTmemCols = 512;

// dk/dv geometry: NQ query positions per step (64 when k divides 64, else
// 128) and NBUF S^T / dP^T buffers (two at NQ = 64: the next step's products
// go to the other buffer while dV and dK read this one's P^T and dS^T).
template <int D, int NQ>
struct DkvCfg {
    static constexpr int HQ2 = NQ / 2;              // query columns per elementwise warp
    static constexpr int NBUF = NQ == 64 ? 2 : 1;
    static constexpr int QS = NQ == 64 ? 4 : 2;     // Q / dO stages
    static constexpr int kSplit = NQ == 64 ? 256 : 128;   // steps per CTA (16384 query positions)
    static constexpr int kTile = BK * D * 2;        // a 128 x D bf16 K or V tile
    static constexpr int kQTile = NQ * D * 2;       // an NQ x D bf16 Q or dO tile
    static constexpr int kQHalf = NQ * 128;         // one 64-column half of it
    static constexpr int kK = 0;
    static constexpr int kV = kK + kTile;
    static constexpr int kQ = kV + kTile;           // [QS] query tiles
    static constexpr int kDO = kQ + QS * kQTile;    // [QS] dO tiles
    static constexpr int kLD = kDO + QS * kQTile;   // [QS][lse2, D][NQ] floats
    static constexpr int kBar = kLD + QS * 2 * NQ * 4;
    // kv, qt[QS], qf[QS], qe[QS], s[NBUF], dp[NBUF], p[NBUF], ds[NBUF], dv, dk, drain
    static constexpr int kNumBars = 1 + 3 * QS + 4 * NBUF + 3;
    static constexpr int kMisc = kBar + kNumBars * 8;
    static constexpr int kBytes = kMisc + 16;
    static_assert(kBytes <= 227 * 1024, "shared memory budget");
    static_assert(2 * NBUF * NQ + 2 * D <= (int)kTmemCols, "TMEM budget");
    static_assert(HQ2 % 32 == 0, "elementwise column groups");
};

struct TArgs {
    CUtensorMap tm_kt, tm_ks, tm_vt, tm_vs, tm_q, tm_do;   // 128-row boxes (dq: query tiles; K/V tiles)
    CUtensorMap tm_qs, tm_dos;                             // nqs-row boxes: the dk/dv steps' Q and dO
    int k, w, G, Hq, Hkv, batch;
    float scale, scale_log2;
    const int32_t *cu;
    Plan pl;
    const int32_t *ks_off, *kt_off;   // [B+1] first summary / text key tile of each sequence
    const int32_t *item_off;          // [tiles+1] first CTA of each key tile (summary tiles first)
    int max_tiles;
    int nqs, split;                   // dk/dv: query positions per step, steps per CTA
    int bpw;                          // dk/dv: query blocks of nqs per share window, max(1, split / G)
    int32_t *err;
    const float *lse, *dsum;
    float *dk32, *dv32;
};

// A key tile, the text query range that sees it, and its CTA shares.
// key_tile is host-callable too, for CPU tests of the ranges against the
// dense mask.
//
// The range [qlo, qhi) is cut into nq blocks of nqs query positions.  A
// share (one CTA) takes the blocks of one window of bpw blocks, each block
// for all G q heads of the kv head.  A summary tile's windows are aligned
// to the sequence's block grid, common to all its summary tiles (their qlo
// differ by multiples of 128 k, a multiple of nqs), so that the shares of
// neighbouring summary tiles over one window read the same Q and dO blocks
// and, walking the window from its last block down, read them at about the
// same time: the data is fetched from DRAM once and reused from L2.  lead
// is the tile's first block's place in its window (0 for text tiles, whose
// shares start at qlo), nsh the number of shares.
struct KTile {
    int b, sum, j0, kcnt, n, m, c0, qlo, qhi, nq, lead, nsh;
};

__host__ __device__ __forceinline__ int find_off(const int32_t *off, int batch, int id)
{
    int lo = 0, hi = batch - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (off[mid] <= id) lo = mid; else hi = mid - 1;
    }
    return lo;
}

__host__ __device__ __forceinline__ void key_tile(const TArgs &a, int tile, KTile &T)
{
    const int ns = a.ks_off[a.batch];
    T.sum = tile < ns;
    const int32_t *off = T.sum ? a.ks_off : a.kt_off;
    const int id = T.sum ? tile : tile - ns;
    T.b = find_off(off, a.batch, id);
    T.j0 = (id - off[T.b]) * BK;
    T.n = a.cu[T.b + 1] - a.cu[T.b];
    T.m = T.n / a.k;
    T.c0 = a.pl.chunk_off[T.b];
    if (T.sum) {
        T.kcnt = min(BK, T.m - T.j0);
        T.qlo = window_end(T.j0, a.w, a.k, T.n);   // first text query of summary j0
        T.qhi = T.n;
    } else {
        T.kcnt = min(BK, T.n - T.j0);
        const int cb = (T.j0 + T.kcnt - 1) / a.k;
        T.qlo = T.j0;
        T.qhi = window_end(cb, a.w, a.k, T.n);     // past the last text query of chunk cb's keys
    }
    T.nq = T.qhi > T.qlo ? (int)(((int64_t)T.qhi - T.qlo + a.nqs - 1) / a.nqs) : 0;   // dk/dv steps per q head
    T.lead = T.sum ? (T.qlo / a.nqs) % a.bpw : 0;
    T.nsh = T.nq > 0 ? (T.nq + T.lead + a.bpw - 1) / a.bpw : 0;
}

// Blocks [r_lo, r_hi) of share sh of tile T (relative to T.qlo).
__host__ __device__ __forceinline__ void share_blocks(const TArgs &a, const KTile &T, int sh, int &r_lo, int &r_hi)
{
    r_lo = max(0, sh * a.bpw - T.lead);
    r_hi = min(T.nq, (sh + 1) * a.bpw - T.lead);
}

// The text queries [lo, hi) that see key row r of tile T (text position or
// summary index j0 + r).  Host-callable too, for the same CPU tests.
__host__ __device__ __forceinline__ void key_queries(const TArgs &a, const KTile &T, int r, int &lo, int &hi)
{
    const int key = T.j0 + r;
    if (T.sum) {
        lo = window_end(key, a.w, a.k, T.n);
        hi = T.n;
    } else {
        lo = key;
        hi = window_end(key / a.k, a.w, a.k, T.n);
    }
}

// Key tiles (summary tiles of all sequences, then text tiles) and the CTA
// offsets of their nsh shares each.
__global__ void __launch_bounds__(1024) bt_plan_kernel(TArgs a, int32_t *ks_off, int32_t *kt_off, int32_t *item_off)
{
    __shared__ int part[1024];
    __shared__ int s_nt;
    if (threadIdx.x == 0) {
        int s = 0, t = 0;
        for (int b = 0; b < a.batch; ++b) {
            ks_off[b] = s;
            kt_off[b] = t;
            const int n = max(a.cu[b + 1] - a.cu[b], 0);
            s += (n / a.k + BK - 1) / BK;
            t += (n + BK - 1) / BK;
        }
        ks_off[a.batch] = s;
        kt_off[a.batch] = t;
        s_nt = s + t;
        if (s + t > a.max_tiles) {
            set_error(a.err, KSA_ERR_UNSUPPORTED);
            s_nt = 0;
        }
    }
    __syncthreads();
    const int NT = s_nt;
    const int per = (NT + 1023) / 1024;
    const int lo = min(NT, (int)threadIdx.x * per), hi = min(NT, lo + per);
    int sum = 0;
    for (int t = lo; t < hi; ++t) {
        KTile T;
        key_tile(a, t, T);
        sum += T.nsh;
    }
    part[threadIdx.x] = sum;
    __syncthreads();
    if (threadIdx.x == 0) {   // exclusive scan of the 1024 partial counts
        int run = 0;
        for (int i = 0; i < 1024; ++i) {
            const int v = part[i];
            part[i] = run;
            run += v;
        }
        item_off[NT] = run;
    }
    __syncthreads();
    int run = part[threadIdx.x];
    for (int t = lo; t < hi; ++t) {
        item_off[t] = run;
        KTile T;
        key_tile(a, t, T);
        run += T.nsh;
    }
}

template <int D, int NQ>
__global__ void __launch_bounds__(kThreads, 1) bt_dkv_kernel(const __grid_constant__ TArgs a)
{
    using L = DkvCfg<D, NQ>;
    constexpr int QS = L::QS, NBUF = L::NBUF, HQ2 = L::HQ2;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = smem_raw;
    const uint32_t sbase = smem_u32(smem);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMisc);
    volatile int *abort = reinterpret_cast<volatile int *>(smem + L::kMisc + 4);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (*a.err != 0) return;
    if (sbase & 1023u) {
        if (threadIdx.x == 0) set_error(a.err, KSA_ERR_UNSUPPORTED);
        return;
    }
    // this CTA's key tile and share (uniform over the CTA; empty CTAs leave
    // before any barrier or TMEM is touched)
    const int NT = a.ks_off[a.batch] + a.kt_off[a.batch];
    if (NT > a.max_tiles) return;
    const int item = blockIdx.x;
    if (item >= a.item_off[NT]) return;
    const int tile = find_off(a.item_off, NT, item);
    KTile T;
    key_tile(a, tile, T);
    const int g = blockIdx.y;
    int r_lo, r_hi;
    share_blocks(a, T, item - a.item_off[tile], r_lo, r_hi);
    const int n_steps = (r_hi - r_lo) * a.G;
    if (n_steps <= 0) return;

    auto bar = [&](int i) { return sbase + L::kBar + 8u * (uint32_t)i; };
    constexpr int B_KV = 0;
    auto B_QT = [](int s) { return 1 + s; };              // Q, dO landed
    auto B_QF = [](int s) { return 1 + QS + s; };         // + LSE, D, zero rows: ready
    auto B_QE = [](int s) { return 1 + 2 * QS + s; };     // stage free
    auto B_S = [](int b) { return 1 + 3 * QS + b; };      // S^T of buffer b computed
    auto B_DP = [](int b) { return 1 + 3 * QS + NBUF + b; };
    auto B_P = [](int b) { return 1 + 3 * QS + 2 * NBUF + b; };    // P^T written
    auto B_DS = [](int b) { return 1 + 3 * QS + 3 * NBUF + b; };   // dS^T written
    constexpr int B_DV = 1 + 3 * QS + 4 * NBUF, B_DK = B_DV + 1, B_DRAIN = B_DV + 2;

    if (threadIdx.x == 0) {
        mbar_init(bar(B_KV), 1);
        for (int s = 0; s < QS; ++s) {
            mbar_init(bar(B_QT(s)), 1);
            mbar_init(bar(B_QF(s)), 32);
            mbar_init(bar(B_QE(s)), 2);   // one commit per issuer
        }
        for (int b = 0; b < NBUF; ++b) {
            mbar_init(bar(B_S(b)), 1);
            mbar_init(bar(B_DP(b)), 1);
            mbar_init(bar(B_P(b)), 256);
            mbar_init(bar(B_DS(b)), 256);
        }
        mbar_init(bar(B_DV), 1);
        mbar_init(bar(B_DK), 1);
        mbar_init(bar(B_DRAIN), 2);   // one commit per issuer, after its last MMA
        *abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kWarpMMA) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // TMEM: S^T[NBUF], dP^T[NBUF] (NQ columns each), dV, dK (D columns each)
    auto T_S = [&](int b) { return tmem + (uint32_t)(b * NQ); };
    auto T_DP = [&](int b) { return tmem + (uint32_t)((NBUF + b) * NQ); };
    const uint32_t T_DV = tmem + 2 * NBUF * NQ, T_DK = T_DV + D;
    constexpr uint32_t kHalf = BK * 128;   // one 64-column half of a K or V tile
    constexpr uint32_t kTileBytes = (uint32_t)L::kTile, kQBytes = (uint32_t)L::kQTile;
    constexpr uint32_t kQHalf = (uint32_t)L::kQHalf;

    // step s of the share -> (query block, q head): the share's last block
    // first, each block for the G q heads in turn
    auto step_q0 = [&](int s) { return T.qlo + (r_hi - 1 - s / a.G) * NQ; };
    auto step_h = [&](int s) { return g * a.G + s % a.G; };

    if (warp == kWarpTMA) {
        if (lane == 0) {
            bool ok = true;
            int q_issued[QS] = {0};
            mbar_expect_tx(bar(B_KV), 2 * kTileBytes);
            for (int hf = 0; hf < D / 64; ++hf) {
                if (T.sum) {
                    tma_load_4d(sbase + L::kK + hf * kHalf, &a.tm_ks, bar(B_KV), hf * 64, g, a.k, T.c0 + T.j0);
                    tma_load_4d(sbase + L::kV + hf * kHalf, &a.tm_vs, bar(B_KV), hf * 64, g, a.k, T.c0 + T.j0);
                } else {
                    tma_load_4d(sbase + L::kK + hf * kHalf, &a.tm_kt, bar(B_KV), hf * 64, g, 0, T.c0 + T.j0 / a.k);
                    tma_load_4d(sbase + L::kV + hf * kHalf, &a.tm_vt, bar(B_KV), hf * 64, g, 0, T.c0 + T.j0 / a.k);
                }
            }
            for (int s = 0; s < n_steps; ++s) {
                const int st = s % QS;
                if (s >= QS && !(ok = mbar_wait_sleep(bar(B_QE(st)), (uint32_t)((s / QS) - 1) & 1u, abort, a.err)))
                    break;
                const int chunk = T.c0 + step_q0(s) / a.k, h = step_h(s);
                mbar_expect_tx(bar(B_QT(st)), 2 * kQBytes);
                for (int hf = 0; hf < D / 64; ++hf) {
                    tma_load_4d(sbase + L::kQ + st * kQBytes + hf * kQHalf, &a.tm_qs, bar(B_QT(st)), hf * 64, h, 0,
                                chunk);
                    tma_load_4d(sbase + L::kDO + st * kQBytes + hf * kQHalf, &a.tm_dos, bar(B_QT(st)), hf * 64, h,
                                0, chunk);
                }
                q_issued[st]++;
            }
            // every load issued lands before the CTA exits
            for (uint32_t it = 0; it < kSpinLimit && !mbar_try_wait(bar(B_KV), 0); ++it) {}
            if (!ok)
                for (int st = 0; st < QS; ++st)
                    if (q_issued[st]) {
                        const uint32_t ph = (uint32_t)(q_issued[st] - 1) & 1u;
                        for (uint32_t it = 0; it < kSpinLimit && !mbar_try_wait(bar(B_QT(st)), ph); ++it) {}
                    }
        }
    } else if (warp == kWarpLD) {
        // per step: the step's LSE (log2 units) and D, fetched one step ahead
        // into registers (the loads of step s + 1 are in flight while step s
        // waits for its tiles); once the tiles have landed, zero the query
        // rows past the sequence (they meet P = 0 and dS = 0 in the MMAs,
        // which need them finite) and publish LSE and D in shared memory
        constexpr int PER = NQ / 32;
        float l2v[PER], ddv[PER];
        auto fetch = [&](int s) {
            const int q0 = step_q0(s), h = step_h(s), qn = min(NQ, T.n - q0);
#pragma unroll
            for (int u = 0; u < PER; ++u) {
                const int r = lane + 32 * u, pos = q0 + r;
                const int64_t row = (int64_t)(T.c0 + pos / a.k) * (a.k + 1) + pos % a.k;
                l2v[u] = r < qn ? a.lse[row * a.Hq + h] : 0.f;
                ddv[u] = r < qn ? a.dsum[row * a.Hq + h] : 0.f;
            }
        };
        bool ok = true;
        fetch(0);
        for (int s = 0; s < n_steps && ok; ++s) {
            const int st = s % QS;
            ok = __all_sync(0xffffffffu, mbar_wait_sleep(bar(B_QT(st)), (uint32_t)(s / QS) & 1u, abort, a.err));
            if (!ok) break;
            const int qn = min(NQ, T.n - step_q0(s));
            if (qn < NQ) {
                const int per_row = 8 * (D / 64);   // 16-byte words of a row over both halves
                for (int e = lane; e < (NQ - qn) * per_row; e += 32) {
                    const int r = qn + e / per_row, hf = (e % per_row) / 8, c = e % 8;
                    const uint32_t off = (uint32_t)(hf * kQHalf + r * 128 + c * 16);
                    *reinterpret_cast<uint4 *>(smem + L::kQ + st * kQBytes + off) = make_uint4(0, 0, 0, 0);
                    *reinterpret_cast<uint4 *>(smem + L::kDO + st * kQBytes + off) = make_uint4(0, 0, 0, 0);
                }
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            }
            float *ld = reinterpret_cast<float *>(smem + L::kLD) + st * 2 * NQ;
#pragma unroll
            for (int u = 0; u < PER; ++u) {
                ld[lane + 32 * u] = l2v[u] * 1.4426950408889634f;
                ld[NQ + lane + 32 * u] = ddv[u];
            }
            mbar_arrive(bar(B_QF(st)));
            if (s + 1 < n_steps) fetch(s + 1);
        }
    } else if (warp == kWarpMMA || warp == kWarpMMA2) {
        // Two issuers, one per chain: kWarpMMA the P side (S^T = K Q^T, then
        // dV += P^T dO), kWarpMMA2 the dS side (dP^T = V dO^T, then
        // dK += dS^T Q).  With two buffers a side issues step t's product
        // before the accumulation of step t - 1, which reads the other
        // buffer; a buffer is reused once this side's accumulation of the
        // step two back has read it.
        if (lane == 0) {
            const bool pside = warp == kWarpMMA;
            const uint32_t id_ss = idesc_f16(BK, NQ, false);
            const uint32_t id_ts = idesc_f16(BK, D, true);
            const int b_in0 = pside ? B_P(0) : B_DS(0), b_x0 = pside ? B_S(0) : B_DP(0);
            const int b_acc = pside ? B_DV : B_DK;
            const uint32_t T_ACC = pside ? T_DV : T_DK;
            const uint64_t dA = sdesc(sbase + (pside ? L::kK : L::kV), 16, 1024);   // SS A: K or V
            bool ok = mbar_wait_sleep(bar(B_KV), 0, abort, a.err);
            for (int t = 0; t < n_steps + NBUF - 1 && ok; ++t) {
                if (t < n_steps) {
                    const int st = t % QS, b = t % NBUF;
                    if (!(ok = mbar_wait_sleep(bar(B_QF(st)), (uint32_t)(t / QS) & 1u, abort, a.err))) break;
                    if (t >= NBUF && !(ok = mbar_wait_sleep(bar(b_acc), (uint32_t)(t - NBUF) & 1u, abort, a.err)))
                        break;
                    tc_fence_after();
                    const uint64_t dB =
                        sdesc(sbase + (pside ? L::kQ : L::kDO) + st * kQBytes, 16, 1024);   // SS B: Q or dO
                    const uint32_t T_X = pside ? T_S(b) : T_DP(b);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk)
                        mma_ss(T_X, dA + ((uint32_t)((kk / 4) * kHalf + (kk % 4) * 32) >> 4),
                               dB + ((uint32_t)((kk / 4) * kQHalf + (kk % 4) * 32) >> 4), id_ss, kk > 0);
                    tc_commit(bar(b_x0 + b));
                }
                const int s = t - (NBUF - 1);
                if (s >= 0) {
                    const int st = s % QS, b = s % NBUF;
                    if (!(ok = mbar_wait_sleep(bar(b_in0 + b), (uint32_t)(s / NBUF) & 1u, abort, a.err))) break;
                    tc_fence_after();
                    // half h's bf16 pairs sit in columns [HQ2 h, HQ2 h + HQ2/2) of
                    // S^T / dP^T and meet rows [HQ2 h, HQ2 h + HQ2) of dO / Q
                    const uint64_t dC = sdesc(sbase + (pside ? L::kDO : L::kQ) + st * kQBytes, kQHalf, 1024);
                    const uint32_t T_X = pside ? T_S(b) : T_DP(b);
#pragma unroll
                    for (int h = 0; h < 2; ++h)
#pragma unroll
                        for (int kk = 0; kk < HQ2 / 16; ++kk)
                            mma_ts(T_ACC, T_X + h * HQ2 + kk * 8, dC + (uint32_t)(((h * (HQ2 / 16) + kk) * 2048) >> 4),
                                   id_ts, (s > 0 || h > 0 || kk > 0) ? 1u : 0u);
                    tc_commit(bar(b_acc));
                    tc_commit(bar(B_QE(st)));
                }
            }
            tc_commit(bar(B_DRAIN));
            for (uint32_t it = 0; it < kSpinLimit && !mbar_try_wait(bar(B_DRAIN), 0); ++it) {}
        }
    } else if (warp < 8) {
        // ================= elementwise: 8 warps, HQ2 query columns each =================
        const int half = warp >> 2, quarter = warp & 3;
        const int r = quarter * 32 + lane;   // key row = TMEM lane
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const bool live = r < T.kcnt;
        const int key = T.j0 + r;            // text position or summary index
        int klo, khi;                        // the text queries that see it
        key_queries(a, T, r, klo, khi);
        const float sl2 = a.scale_log2;
        bool ok = true;
        for (int s = 0; s < n_steps; ++s) {
            const int st = s % QS, b = s % NBUF;
            const uint32_t ph = (uint32_t)(s / NBUF) & 1u;
            const int q0 = step_q0(s);
            const int qn = min(NQ, T.n - q0);
            // this row's visible columns [lo, hi) of the step, inside this half
            int lo = klo - q0, hi = min(qn, khi - q0);
            if (!live) lo = hi = 0;
            lo = max(lo - half * HQ2, 0);
            hi = min(hi - half * HQ2, HQ2);
            if (hi < lo) hi = lo;
            // every column of this half visible to every row of the warp: no mask
            const bool full = __all_sync(0xffffffffu, lo == 0 && hi == HQ2);
            ok = ok && __all_sync(0xffffffffu, mbar_wait(bar(B_QF(st)), (uint32_t)(s / QS) & 1u, abort, a.err));
            ok = ok && __all_sync(0xffffffffu, mbar_wait(bar(B_S(b)), ph, abort, a.err));
            if (!ok) break;
            const float *l2 = reinterpret_cast<const float *>(smem + L::kLD) + st * 2 * NQ + half * HQ2;
            const float *dd = l2 + NQ;
            float p[HQ2];
            {
                uint32_t sr[HQ2];
                tc_fence_after();
#pragma unroll
                for (int cc = 0; cc < HQ2 / 32; ++cc) tmem_ld32(T_S(b) + lane_off + half * HQ2 + cc * 32, sr + cc * 32);
                tmem_wait_ld();
                if (full) {
#pragma unroll
                    for (int e = 0; e < HQ2; ++e) p[e] = ex2(fmaf(__uint_as_float(sr[e]), sl2, -l2[e]));
                } else {
#pragma unroll
                    for (int e = 0; e < HQ2; ++e) {
                        const float x = fmaf(__uint_as_float(sr[e]), sl2, -l2[e]);
                        p[e] = (e >= lo && e < hi) ? ex2(x) : 0.f;
                    }
                }
#pragma unroll
                for (int grp = 0; grp < HQ2 / 32; ++grp) {
                    uint32_t pk[16];
#pragma unroll
                    for (int e2 = 0; e2 < 16; ++e2) pk[e2] = pack_bf16(p[grp * 32 + 2 * e2], p[grp * 32 + 2 * e2 + 1]);
                    tmem_st16(T_S(b) + lane_off + half * HQ2 + grp * 16, pk);
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar(B_P(b)));
            }
            ok = __all_sync(0xffffffffu, mbar_wait(bar(B_DP(b)), ph, abort, a.err));
            if (!ok) break;
            tc_fence_after();
#pragma unroll
            for (int grp = 0; grp < HQ2 / 32; ++grp) {
                uint32_t dr[32], pk[16];
                tmem_ld32(T_DP(b) + lane_off + half * HQ2 + grp * 32, dr);
                tmem_wait_ld();
                float ds[32];
                if (full) {
#pragma unroll
                    for (int e = 0; e < 32; ++e) ds[e] = p[grp * 32 + e] * (__uint_as_float(dr[e]) - dd[grp * 32 + e]);
                } else {
#pragma unroll
                    for (int e = 0; e < 32; ++e) {
                        const int c = grp * 32 + e;
                        ds[e] = (c >= lo && c < hi) ? p[c] * (__uint_as_float(dr[e]) - dd[c]) : 0.f;
                    }
                }
#pragma unroll
                for (int e2 = 0; e2 < 16; ++e2) pk[e2] = pack_bf16(ds[2 * e2], ds[2 * e2 + 1]);
                // dS^T of this half -> dP^T columns [HQ2 half + 16 grp, +16), which
                // this thread has already loaded
                tmem_st16(T_DP(b) + lane_off + half * HQ2 + grp * 16, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(B_DS(b)));
        }
        // ---- epilogue: dK (scaled) and dV rows into the fp32 accumulators ----
        // (the drain barrier completes once, after every MMA of both issuers)
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(B_DRAIN), 0, abort, a.err));
        if (ok) {
            tc_fence_after();
            const int64_t row = T.sum ? (int64_t)(T.c0 + key) * (a.k + 1) + a.k
                                      : (int64_t)(T.c0 + key / a.k) * (a.k + 1) + key % a.k;
            float4 *pk = reinterpret_cast<float4 *>(a.dk32 + (row * a.Hkv + g) * D + half * (D / 2));
            float4 *pv = reinterpret_cast<float4 *>(a.dv32 + (row * a.Hkv + g) * D + half * (D / 2));
#pragma unroll 1
            for (int cc = 0; cc < D / 64; ++cc) {
                uint32_t vk[32], vv[32];
                tmem_ld32(T_DK + lane_off + half * (D / 2) + cc * 32, vk);
                tmem_ld32(T_DV + lane_off + half * (D / 2) + cc * 32, vv);
                tmem_wait_ld();
                if (live) {
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        atomicAdd(pk + cc * 8 + e,
                                  make_float4(__uint_as_float(vk[4 * e]) * a.scale, __uint_as_float(vk[4 * e + 1]) * a.scale,
                                              __uint_as_float(vk[4 * e + 2]) * a.scale,
                                              __uint_as_float(vk[4 * e + 3]) * a.scale));
                        atomicAdd(pv + cc * 8 + e, make_float4(__uint_as_float(vv[4 * e]), __uint_as_float(vv[4 * e + 1]),
                                                               __uint_as_float(vv[4 * e + 2]),
                                                               __uint_as_float(vv[4 * e + 3])));
                    }
                }
            }
        }
    }

    // ---- teardown --------------------------------------------------------
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kWarpMMA) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                     : "memory");
    }
}

// ---------------------------------------------------------------------------
// dq of the text query rows.  A CTA owns 128 consecutive text query
// positions of one q head (rows = TMEM lanes; Q and dO stay in shared
// memory) and walks the key tiles those rows can see: the summary tiles
// s_0 .. s_{c_last-w-1}, then the text tiles from chunk c_first - w on.  A
// step is three MMAs:
//     S   = Q K^T      (SS, M 128 queries, N 128 keys)
//     dP  = dO V^T     (SS, into one of two dP buffers)
//     dQ += dS K       (TS: dS written as bf16 over its dP buffer, B = K
//                       MN-major)
// S is released as soon as the elementwise warps have loaded it, so the
// next step's S runs while they form dS; the two dP buffers let dP(j+1)
// run before dQ(j) has read dS(j).  TMEM: S, dP x 2, dQ.
constexpr int KST = 3;   // K stages (a K tile is read by S(j) and by dQ(j) one step later)
constexpr int VST = 2;   // V stages

template <int D>
struct SmemQ {
    static constexpr int kTile = BK * D * 2;
    static constexpr int kQ = 0;
    static constexpr int kDO = kQ + kTile;
    static constexpr int kK = kDO + kTile;            // [KST]
    static constexpr int kV = kK + KST * kTile;       // [VST]
    static constexpr int kBar = kV + VST * kTile;
    // q, kf[KST], ke[KST], vf[VST], ve[VST], s, sc, dp, ds, dq, drain
    static constexpr int kNumBars = 1 + 2 * KST + 2 * VST + 6;
    static constexpr int kMisc = kBar + kNumBars * 8;
    static constexpr int kBytes = kMisc + 16;
    static_assert(kBytes <= 227 * 1024, "shared memory budget");
    static_assert(3 * BK + D <= (int)kTmemCols, "TMEM budget");
};

// The query tile of a dq CTA and its key tiles: text tiles in reverse order
// (late tiles see the most summaries); ceil(ns / 128) summary tiles, then
// the text keys [t_lo, q0 + qn) in tiles of 128.  Host-callable too, for
// CPU tests of the tile list against the dense mask.
struct QTile {
    int b, n, m, c0, q0, qn, c_first, ns, n_sum, t_lo, n_win;
};

__host__ __device__ __forceinline__ bool q_tile(const TArgs &a, int cta, QTile &Q)
{
    const int ntt = a.kt_off[a.batch];
    if (cta >= ntt) return false;
    const int qt = ntt - 1 - cta;
    Q.b = find_off(a.kt_off, a.batch, qt);
    Q.n = a.cu[Q.b + 1] - a.cu[Q.b];
    Q.m = Q.n / a.k;
    Q.c0 = a.pl.chunk_off[Q.b];
    Q.q0 = (qt - a.kt_off[Q.b]) * BQ;
    Q.qn = min(BQ, Q.n - Q.q0);
    Q.c_first = Q.q0 / a.k;
    const int c_last = (Q.q0 + Q.qn - 1) / a.k;
    Q.ns = max(0, min(Q.m, c_last - a.w));              // summaries any row may see
    Q.n_sum = (Q.ns + BK - 1) / BK;
    Q.t_lo = max(0, Q.c_first - a.w) * a.k;
    Q.n_win = (Q.q0 + Q.qn - Q.t_lo + BK - 1) / BK;
    return true;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1) bq_dq_kernel(const __grid_constant__ TArgs a, __nv_bfloat16 *dq)
{
    using L = SmemQ<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = smem_raw;
    const uint32_t sbase = smem_u32(smem);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMisc);
    volatile int *abort = reinterpret_cast<volatile int *>(smem + L::kMisc + 4);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (*a.err != 0) return;
    if (sbase & 1023u) {
        if (threadIdx.x == 0) set_error(a.err, KSA_ERR_UNSUPPORTED);
        return;
    }
    QTile Q;
    if (!q_tile(a, (int)blockIdx.x, Q)) return;
    const int m = Q.m, c0 = Q.c0, q0 = Q.q0, qn = Q.qn;
    const int h = blockIdx.y, g = h / a.G;
    const int c_first = Q.c_first;
    const int n_sum = Q.n_sum, t_lo = Q.t_lo;
    const int n_steps = n_sum + Q.n_win;                  // >= 1: every row sees itself

    auto bar = [&](int i) { return sbase + L::kBar + 8u * (uint32_t)i; };
    constexpr int B_Q = 0;
    auto B_KF = [](int s) { return 1 + s; };
    auto B_KE = [](int s) { return 1 + KST + s; };
    auto B_VF = [](int s) { return 1 + 2 * KST + s; };
    auto B_VE = [](int s) { return 1 + 2 * KST + VST + s; };
    constexpr int B_S = 1 + 2 * KST + 2 * VST, B_SC = B_S + 1, B_DP = B_S + 2, B_DS = B_S + 3, B_DQ = B_S + 4,
                  B_DRAIN = B_S + 5;

    if (threadIdx.x == 0) {
        mbar_init(bar(B_Q), 1);
        for (int s = 0; s < KST; ++s) {
            mbar_init(bar(B_KF(s)), 1);
            mbar_init(bar(B_KE(s)), 1);
        }
        for (int s = 0; s < VST; ++s) {
            mbar_init(bar(B_VF(s)), 1);
            mbar_init(bar(B_VE(s)), 1);
        }
        mbar_init(bar(B_S), 1);
        mbar_init(bar(B_SC), 256);
        mbar_init(bar(B_DP), 1);
        mbar_init(bar(B_DS), 256);
        mbar_init(bar(B_DQ), 1);
        mbar_init(bar(B_DRAIN), 2);   // one commit per issuer, after its last MMA
        *abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == kWarpMMA) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t T_S = tmem, T_DQ = tmem + 3 * BK;
    auto T_DP = [&](int j) { return tmem + (uint32_t)(BK + (j & 1) * BK); };
    constexpr uint32_t kHalf = BK * 128;
    constexpr uint32_t kTileBytes = (uint32_t)L::kTile;

    if (warp == kWarpTMA) {
        if (lane == 0) {
            bool ok = true;
            int k_issued[KST] = {0}, v_issued[VST] = {0};
            mbar_expect_tx(bar(B_Q), 2 * kTileBytes);
            for (int hf = 0; hf < D / 64; ++hf) {
                tma_load_4d(sbase + L::kQ + hf * kHalf, &a.tm_q, bar(B_Q), hf * 64, h, 0, c0 + c_first);
                tma_load_4d(sbase + L::kDO + hf * kHalf, &a.tm_do, bar(B_Q), hf * 64, h, 0, c0 + c_first);
            }
            // K of step j, then V of step j: K runs a stage further ahead
            for (int j = 0; j < n_steps && ok; ++j) {
                const bool sum = j < n_sum;
                const int c1 = g, c2 = sum ? a.k : 0;
                const int c3 = sum ? c0 + j * BK : c0 + (t_lo + (j - n_sum) * BK) / a.k;
                const CUtensorMap *mk = sum ? &a.tm_ks : &a.tm_kt, *mv = sum ? &a.tm_vs : &a.tm_vt;
                const int sk = j % KST, sv = j % VST;
                if (j >= KST && !(ok = mbar_wait_sleep(bar(B_KE(sk)), (uint32_t)((j / KST) - 1) & 1u, abort, a.err)))
                    break;
                mbar_expect_tx(bar(B_KF(sk)), kTileBytes);
                for (int hf = 0; hf < D / 64; ++hf)
                    tma_load_4d(sbase + L::kK + sk * kTileBytes + hf * kHalf, mk, bar(B_KF(sk)), hf * 64, c1, c2, c3);
                k_issued[sk]++;
                if (j >= VST && !(ok = mbar_wait_sleep(bar(B_VE(sv)), (uint32_t)((j / VST) - 1) & 1u, abort, a.err)))
                    break;
                mbar_expect_tx(bar(B_VF(sv)), kTileBytes);
                for (int hf = 0; hf < D / 64; ++hf)
                    tma_load_4d(sbase + L::kV + sv * kTileBytes + hf * kHalf, mv, bar(B_VF(sv)), hf * 64, c1, c2, c3);
                v_issued[sv]++;
            }
            for (uint32_t it = 0; it < kSpinLimit && !mbar_try_wait(bar(B_Q), 0); ++it) {}
            if (!ok) {
                for (int s = 0; s < KST; ++s)
                    if (k_issued[s]) {
                        const uint32_t ph = (uint32_t)(k_issued[s] - 1) & 1u;
                        for (uint32_t it = 0; it < kSpinLimit && !mbar_try_wait(bar(B_KF(s)), ph); ++it) {}
                    }
                for (int s = 0; s < VST; ++s)
                    if (v_issued[s]) {
                        const uint32_t ph = (uint32_t)(v_issued[s] - 1) & 1u;
                        for (uint32_t it = 0; it < kSpinLimit && !mbar_try_wait(bar(B_VF(s)), ph); ++it) {}
                    }
            }
        }
    } else if (warp == kWarpMMA || warp == kWarpMMA2) {
        // Two issuers: kWarpMMA issues S(j) = Q K(j)^T as soon as K(j) has
        // landed and the elementwise warps have loaded S(j-1); kWarpMMA2
        // issues dP(j) = dO V(j)^T and dQ += dS(j-1) K(j-1).
        if (lane == 0) {
            const uint32_t id_ss = idesc_f16(BK, BK, false);
            const uint32_t id_ts = idesc_f16(BK, D, true);
            bool ok = mbar_wait_sleep(bar(B_Q), 0, abort, a.err);
            if (warp == kWarpMMA) {
                const uint64_t dQd = sdesc(sbase + L::kQ, 16, 1024);
                for (int j = 0; j < n_steps && ok; ++j) {
                    const int sk = j % KST;
                    if (!(ok = mbar_wait_sleep(bar(B_KF(sk)), (uint32_t)(j / KST) & 1u, abort, a.err))) break;
                    if (j > 0 && !(ok = mbar_wait_sleep(bar(B_SC), (uint32_t)(j - 1) & 1u, abort, a.err))) break;
                    tc_fence_after();
                    const uint64_t dKd = sdesc(sbase + L::kK + sk * kTileBytes, 16, 1024);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (uint32_t)((kk / 4) * kHalf + (kk % 4) * 32) >> 4;
                        mma_ss(T_S, dQd + off, dKd + off, id_ss, kk > 0);
                    }
                    tc_commit(bar(B_S));
                }
            } else {
                const uint64_t dOd = sdesc(sbase + L::kDO, 16, 1024);
                // dQ(j) = dS(j) K(j): dS(j) (128 keys as bf16 pairs) sits in
                // dP buffer j % 2, columns [64h, 64h + 32) for key half h.  K(j)'s
                // stage is released here; S(j) read it before dS(j) existed.
                // Inside the loop dS(j) was waited for just before dP(j+1); a
                // second parity wait there could miss the phase if dS(j+1)
                // completed in between, so only the last step waits here.
                auto issue_dq = [&](int j, bool wait_ds) -> bool {
                    if (wait_ds && !mbar_wait_sleep(bar(B_DS), (uint32_t)j & 1u, abort, a.err)) return false;
                    tc_fence_after();
                    const uint64_t dKm = sdesc(sbase + L::kK + (j % KST) * kTileBytes, kHalf, 1024);
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh)
#pragma unroll
                        for (int kk = 0; kk < HQ / 16; ++kk)
                            mma_ts(T_DQ, T_DP(j) + hh * HQ + kk * 8, dKm + (uint32_t)(((hh * (HQ / 16) + kk) * 2048) >> 4),
                                   id_ts, (j > 0 || hh > 0 || kk > 0) ? 1u : 0u);
                    tc_commit(bar(B_DQ));
                    tc_commit(bar(B_KE(j % KST)));
                    return true;
                };
                for (int j = 0; j < n_steps && ok; ++j) {
                    const int sv = j % VST;
                    // dP(j) into buffer j % 2, free once dQ(j-2) has read dS(j-2);
                    // it also waits for dS(j-1), so B_DP never completes a phase
                    // the elementwise warps have not waited for yet (a parity wait
                    // only tells the current phase from the one before it)
                    if (!(ok = mbar_wait_sleep(bar(B_VF(sv)), (uint32_t)(j / VST) & 1u, abort, a.err))) break;
                    if (j > 0 && !(ok = mbar_wait_sleep(bar(B_DS), (uint32_t)(j - 1) & 1u, abort, a.err))) break;
                    if (j > 1 && !(ok = mbar_wait_sleep(bar(B_DQ), (uint32_t)(j - 2) & 1u, abort, a.err))) break;
                    tc_fence_after();
                    const uint64_t dVd = sdesc(sbase + L::kV + sv * kTileBytes, 16, 1024);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (uint32_t)((kk / 4) * kHalf + (kk % 4) * 32) >> 4;
                        mma_ss(T_DP(j), dOd + off, dVd + off, id_ss, kk > 0);
                    }
                    tc_commit(bar(B_DP));
                    tc_commit(bar(B_VE(sv)));
                    if (j > 0 && !(ok = issue_dq(j - 1, false))) break;
                }
                if (ok) ok = issue_dq(n_steps - 1, true);
            }
            tc_commit(bar(B_DRAIN));
            for (uint32_t it = 0; it < kSpinLimit && !mbar_try_wait(bar(B_DRAIN), 0); ++it) {}
        }
    } else if (warp < 8) {
        // ================= elementwise: 8 warps, 64 key columns each =================
        const int half = warp >> 2, quarter = warp & 3;
        const int r = quarter * 32 + lane;   // query row = TMEM lane
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const bool live = r < qn;
        const int qp = q0 + r, c = qp / a.k;
        const int64_t row = (int64_t)(c0 + c) * (a.k + 1) + qp % a.k;
        const float lse2 = live ? a.lse[row * a.Hq + h] * 1.4426950408889634f : 0.f;
        const float dd = live ? a.dsum[row * a.Hq + h] : 0.f;
        const int sum_lim = live ? min(c - a.w, m) : 0;   // sees s_j for j < sum_lim
        const int win_lo = max(0, c - a.w) * a.k;
        const float sl2 = a.scale_log2;
        bool ok = true;
        for (int j = 0; j < n_steps; ++j) {
            int lo, hi;
            if (j < n_sum) {
                lo = 0;
                hi = sum_lim - j * BK;
            } else {
                const int kb = t_lo + (j - n_sum) * BK;
                lo = win_lo - kb;
                hi = live ? qp - kb + 1 : 0;
            }
            lo = max(lo - half * HQ, 0);
            hi = min(hi - half * HQ, HQ);
            if (hi < lo) hi = lo;
            const bool full = __all_sync(0xffffffffu, lo == 0 && hi == HQ);
            ok = __all_sync(0xffffffffu, mbar_wait(bar(B_S), (uint32_t)j & 1u, abort, a.err));
            if (!ok) break;
            float p[HQ];
            {
                uint32_t sr[HQ];
                tc_fence_after();
                tmem_ld32(T_S + lane_off + half * HQ, sr);
                tmem_ld32(T_S + lane_off + half * HQ + 32, sr + 32);
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(bar(B_SC));   // S may be overwritten by the next step's QK
                if (full) {
#pragma unroll
                    for (int e = 0; e < HQ; ++e) p[e] = ex2(fmaf(__uint_as_float(sr[e]), sl2, -lse2));
                } else {
#pragma unroll
                    for (int e = 0; e < HQ; ++e) {
                        const float x = fmaf(__uint_as_float(sr[e]), sl2, -lse2);
                        p[e] = (e >= lo && e < hi) ? ex2(x) : 0.f;
                    }
                }
            }
            ok = __all_sync(0xffffffffu, mbar_wait(bar(B_DP), (uint32_t)j & 1u, abort, a.err));
            if (!ok) break;
            tc_fence_after();
            const uint32_t dpb = T_DP(j) + lane_off + half * HQ;
#pragma unroll
            for (int grp = 0; grp < 2; ++grp) {
                uint32_t dr[32], pk[16];
                tmem_ld32(dpb + grp * 32, dr);
                tmem_wait_ld();
                if (full) {
#pragma unroll
                    for (int e2 = 0; e2 < 16; ++e2) {
                        const int e = grp * 32 + 2 * e2;
                        pk[e2] = pack_bf16(p[e] * (__uint_as_float(dr[2 * e2]) - dd),
                                           p[e + 1] * (__uint_as_float(dr[2 * e2 + 1]) - dd));
                    }
                } else {
#pragma unroll
                    for (int e2 = 0; e2 < 16; ++e2) {
                        const int e = grp * 32 + 2 * e2;
                        const float d0 = (e >= lo && e < hi) ? p[e] * (__uint_as_float(dr[2 * e2]) - dd) : 0.f;
                        const float d1 =
                            (e + 1 >= lo && e + 1 < hi) ? p[e + 1] * (__uint_as_float(dr[2 * e2 + 1]) - dd) : 0.f;
                        pk[e2] = pack_bf16(d0, d1);
                    }
                }
                // dS of this half -> columns [64 half + 16 grp, +16) of its dP
                // buffer, which this thread has already loaded
                tmem_st16(dpb + grp * 16, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(B_DS));
        }
        // ---- epilogue: dq = scale dQ -> bf16, this thread's 64 (or 32) columns ----
        // (the drain barrier completes once, after every MMA of the CTA)
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar(B_DRAIN), 0, abort, a.err));
        if (ok) {
            tc_fence_after();
            uint4 *dst = reinterpret_cast<uint4 *>(dq + (row * a.Hq + h) * D + half * (D / 2));
#pragma unroll 1
            for (int cc = 0; cc < D / 64; ++cc) {
                uint32_t v[32];
                tmem_ld32(T_DQ + lane_off + half * (D / 2) + cc * 32, v);
                tmem_wait_ld();
                if (live) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        uint32_t w4[4];
#pragma unroll
                        for (int z = 0; z < 4; ++z)
                            w4[z] = pack_bf16(__uint_as_float(v[8 * e + 2 * z]) * a.scale,
                                              __uint_as_float(v[8 * e + 2 * z + 1]) * a.scale);
                        dst[cc * 4 + e] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kWarpMMA) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                     : "memory");
    }
}

}  // namespace bt

bool prefill_bwd_tc_supported(const ksa_params *p)
{
    return (p->head_dim == 128 || p->head_dim == 64) && p->k >= 1 && p->k <= bt::BQ && bt::BQ % p->k == 0 &&
           p->num_kv_heads > 0 && p->num_q_heads % p->num_kv_heads == 0;
}

// Host-side sizing of the tensor-core backward, shared by the launch, the
// workspace query and the CPU tests of the work list.
//
// Key tiles: at most aug_rows / 128 + 2 batch + 2 (a sequence's text and
// summary rows each end in at most one partial tile).
static int64_t bt_max_tiles(int batch, int64_t aug_rows) { return aug_rows / bt::BK + 2LL * batch + 2; }

// dk/dv steps of 64 query positions (two S^T / dP^T buffers) when k divides
// 64, else of 128; steps per CTA to match.
static void bt_step_shape(int k, int *nqs, int *split)
{
    *nqs = 64 % k == 0 ? 64 : bt::BQ;
    *split = *nqs == 64 ? bt::DkvCfg<128, 64>::kSplit : bt::DkvCfg<128, 128>::kSplit;
}

// Query blocks per dk/dv share window: as many as fit split steps of G heads.
static int bt_bpw(int G, int split) { return split / G > 1 ? split / G : 1; }

// CTAs of the dk/dv launch: an upper bound on the plan's share count (CTAs
// past it exit).  A tile of nq blocks has at most nq / bpw + 2 shares (a
// summary tile's first window may be partial), a text tile at most
// nq / bpw + 1; a summary tile's queries number at most total_text, a text
// tile's 128 + (w+1) k.
static int64_t bt_dkv_grid(int64_t total_text, int batch, int k, int w, int G, int nqs, int split)
{
    const int64_t bpw = bt_bpw(G, split);
    const int64_t ns_tiles = (total_text / k) / bt::BK + batch, nt_tiles = total_text / bt::BK + batch;
    const int64_t q_sum = (total_text + nqs - 1) / nqs + 1;
    const int64_t q_txt = (bt::BK + (int64_t)(w + 1) * k + nqs - 1) / nqs + 1;
    return ns_tiles * (2 + q_sum / bpw) + nt_tiles * (1 + q_txt / bpw);
}

// CTAs of the dq launch: an upper bound on the query tiles of 128 text
// positions, which are the text key tiles (CTAs past the real count exit).
static int64_t bt_dq_grid(int64_t total_text, int batch) { return total_text / bt::BK + batch; }

size_t prefill_bwd_tc_workspace_bytes(int batch, int64_t aug_rows)
{
    const int64_t tiles = bt_max_tiles(batch, aug_rows);
    return 2 * align_up(sizeof(int32_t) * (size_t)(batch + 1)) + align_up(sizeof(int32_t) * (size_t)(tiles + 1));
}

template <int D, int NQ>
static int bt_launch(const bt::TArgs &a, int64_t grid, int64_t grid_q, __nv_bfloat16 *dq, cudaStream_t st)
{
    using C = bt::DkvCfg<D, NQ>;
    static bool attr = false;
    if (!attr) {
        if (cudaFuncSetAttribute(bt::bt_dkv_kernel<D, NQ>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kBytes) !=
                cudaSuccess ||
            cudaFuncSetAttribute(bt::bq_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 bt::SmemQ<D>::kBytes) != cudaSuccess)
            return KSA_ERR_CUDA;
        attr = true;
    }
    bt::bt_dkv_kernel<D, NQ><<<dim3((unsigned)grid, a.Hkv), bt::kThreads, C::kBytes, st>>>(a);
    bt::bq_dq_kernel<D><<<dim3((unsigned)grid_q, a.Hq), bt::kThreads, bt::SmemQ<D>::kBytes, st>>>(a, dq);
    return KSA_OK;
}

int launch_prefill_bwd_tc(const ksa_params *p, int batch, const int32_t *cu, int64_t total_text, int64_t aug_rows,
                          const void *q, const void *k, const void *v, const void *dout, const float *lse,
                          const float *dsum, float *dk32, float *dv32, void *dq, void *ws, const Plan &pl,
                          int32_t *err, cudaStream_t st)
{
    bt::TArgs a;
    const int d = p->head_dim, kk = p->k;
    const int64_t chunks = aug_rows / (kk + 1);
    const int qrows = bt::BQ / kk;   // chunks per query / text key box
    int nqs, split;
    bt_step_shape(kk, &nqs, &split);
    bool ok = make_map(&a.tm_qs, q, d, p->num_q_heads, kk, chunks, 1, kk, nqs / kk) &&
              make_map(&a.tm_dos, dout, d, p->num_q_heads, kk, chunks, 1, kk, nqs / kk) &&
              make_map(&a.tm_kt, k, d, p->num_kv_heads, kk, chunks, 1, kk, qrows) &&
              make_map(&a.tm_vt, v, d, p->num_kv_heads, kk, chunks, 1, kk, qrows) &&
              make_map(&a.tm_ks, k, d, p->num_kv_heads, kk, chunks, 1, 1, bt::BK) &&
              make_map(&a.tm_vs, v, d, p->num_kv_heads, kk, chunks, 1, 1, bt::BK) &&
              make_map(&a.tm_q, q, d, p->num_q_heads, kk, chunks, 1, kk, qrows) &&
              make_map(&a.tm_do, dout, d, p->num_q_heads, kk, chunks, 1, kk, qrows);
    if (!ok) return KSA_ERR_CUDA;
    a.k = kk; a.w = p->w; a.Hq = p->num_q_heads; a.Hkv = p->num_kv_heads; a.G = a.Hq / a.Hkv; a.batch = batch;
    a.scale = p->scale > 0.f ? p->scale : 1.0f / sqrtf((float)d);
    a.scale_log2 = a.scale * 1.4426950408889634f;
    a.cu = cu; a.pl = pl; a.err = err;
    a.lse = lse; a.dsum = dsum; a.dk32 = dk32; a.dv32 = dv32;
    a.nqs = nqs; a.split = split; a.bpw = bt_bpw(a.G, split);
    char *w = static_cast<char *>(ws);
    const size_t ab = align_up(sizeof(int32_t) * (size_t)(batch + 1));
    int32_t *ks_off = reinterpret_cast<int32_t *>(w), *kt_off = reinterpret_cast<int32_t *>(w + ab);
    int32_t *item_off = reinterpret_cast<int32_t *>(w + 2 * ab);
    const int64_t max_tiles = bt_max_tiles(batch, aug_rows);
    if (max_tiles > 0x7fffffffLL) return KSA_ERR_UNSUPPORTED;
    a.ks_off = ks_off; a.kt_off = kt_off; a.item_off = item_off; a.max_tiles = (int)max_tiles;
    bt::bt_plan_kernel<<<1, 1024, 0, st>>>(a, ks_off, kt_off, item_off);
    const int64_t grid = bt_dkv_grid(total_text, batch, kk, p->w, a.G, nqs, split);
    if (grid > 0x7fffffffLL) return KSA_ERR_UNSUPPORTED;
    if (grid == 0) return KSA_OK;
    const int64_t grid_q = bt_dq_grid(total_text, batch);
    __nv_bfloat16 *dqb = static_cast<__nv_bfloat16 *>(dq);
    int r;
    if (nqs == 64)
        r = d == 128 ? bt_launch<128, 64>(a, grid, grid_q, dqb, st) : bt_launch<64, 64>(a, grid, grid_q, dqb, st);
    else
        r = d == 128 ? bt_launch<128, 128>(a, grid, grid_q, dqb, st) : bt_launch<64, 128>(a, grid, grid_q, dqb, st);
    if (r != KSA_OK) return r;
    return cudaGetLastError() == cudaSuccess ? KSA_OK : KSA_ERR_CUDA;
}

}  // namespace ksa

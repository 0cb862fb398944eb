// prefill_sm100.cu -- KSA prefill forward on sm_100a: TMA -> SMEM ->
// tcgen05.mma -> TMEM, warp-specialised, block-sparse by construction.
//
// Kwai Summary Attention Technical Report:
//   - section 2.3 "Kernel Design": Q/K/V are cut into fixed-size blocks and
//     only block pairs the KSA mask does not zero out entirely are loaded and
//     computed; the L x L mask is never materialised;
//   - section 2.2.2, Eq. (3): text t_i attends to the summaries
//     s_0 .. s_{floor(i/k)-w-1} and to the text of chunks
//     floor(i/k)-w .. floor(i/k), causally;
//   - section 2.2.1: summary s_j attends to its own chunk's k text tokens
//     and (Figure 4c) to itself;
//   - Eq. (10): softmax(Q K^T / sqrt(d) + M_KSA) V.
//
// Design (B200-first, not the report's kernel, whose source is not public):
//   * The augmented layout [chunks, k+1, H, d] is read through 4-D TMA
//     tensor maps.  A summary key tile is one box at slot k spanning 128
//     chunks; a text window tile is one box over the k text slots of
//     floor(128/k) chunks.  Summary rows are never loaded as text keys and
//     text rows never as summary keys, so no tile carries dead rows of the
//     other kind.
//   * A query tile is 128 TMEM lanes holding the G = Hq/Hkv heads of one kv
//     head for floor(128/(G k)) chunks of text rows (GQA packing: every K/V
//     tile serves all G heads).  Each CTA runs one query tile at a time
//     against a stream of K/V tiles, its softmax split over the two 64-key
//     halves of every tile (eight warps, each half with its own running max
//     and O accumulator): S = Q K^T and O += P V are tcgen05.mma (kind::f16,
//     bf16 in, fp32 accumulate in TMEM); P is written back into TMEM as bf16
//     over S and fed as the A operand.
//   * The set of K/V tiles of a work unit follows from its chunk
//     coordinates: ceil(min(m, c_last-w)/128) summary tiles plus the window
//     tiles covering chunks c_first-w .. c_last.  Every other tile of the
//     L x L plane is skipped without being looked at.  Inside a tile the
//     mask of a row is one interval of columns, computed from coordinates.
//   * Warp roles: warps 0-7 softmax (two key halves), warp 8 TMA for Q and
//     K, warp 9 the QK issuer and TMEM owner, warp 10 the PV issuer, warp 11
//     TMA for V, warps 12-15 the epilogue (merge the halves, O / l -> bf16,
//     LSE), which runs while the softmax warps start the next work item.
//     All mbarrier waits are bounded; on expiry the CTA records
//     KSA_ERR_TIMEOUT, drains, frees TMEM and exits.
//   * Summary query rows (k+1 keys each) run on the CUDA cores of the
//     epilogue warps, between the items whose chunks they close.
#include <cuda.h>
#include <math.h>

#include <type_traits>

#include "ksa_internal.cuh"
#include "tc_sm100.cuh"
#include "warp_mma.cuh"

namespace ksa {

namespace pf {

constexpr int BM = 128;        // rows per query tile (= TMEM lanes)
constexpr int BN = 128;        // keys per K/V tile (N = 128 runs the MMA at full rate)
constexpr int HC = BN / 2;     // keys per softmax half
constexpr int NSBUF = 2;       // S buffers: QK(j+1) overlaps the softmax of tile j
constexpr int QSTAGES = 2;     // query tiles: the next item's Q loads while this one runs
constexpr int KSTAGES = 2;     // K pipeline depth
constexpr int VSTAGES = 2;     // V pipeline depth
constexpr int kWarpTMA = 8;    // loads Q and the K tiles
constexpr int kWarpQK = 9;     // issues S = Q K^T, owns TMEM
constexpr int kWarpPV = 10;    // issues O_h += P_h V_h
constexpr int kWarpTMAV = 11;  // loads the V tiles (K loads never wait behind V)
constexpr int kWarpEpi = 12;   // warps 12-15: the epilogue of each work item (one row per thread)
constexpr int kThreads = 512;
// 512 threads at 128 registers each fill the register file; every role fits
// (the softmax no longer holds the epilogue's O rows).
constexpr uint32_t kTmemCols = 512;

template <int D>
struct SmemLayout {
    static constexpr int kQTile = BM * D * 2;   // one 128 x D bf16 query tile
    static constexpr int kKVTile = BN * D * 2;  // one 128 x D bf16 key or value tile
    static constexpr int kQ = 0;
    static constexpr int kK = kQ + QSTAGES * kQTile;
    static constexpr int kV = kK + KSTAGES * kKVTile;
    static constexpr int kO = kV + VSTAGES * kKVTile;           // output tile staging for the TMA store
    static constexpr int kBar = kO + kQTile;
    // barriers: kfull[KS], kempty[KS], vfull[VS], vempty[VS], s[NSBUF], p[2 halves][NSBUF],
    // o[NSBUF], drain x2, o free, q full[QS], q free[QS], item done
    static constexpr int kNumBars = 2 * KSTAGES + 2 * VSTAGES + NSBUF + 2 * NSBUF + NSBUF + 2 + 1 + 2 * QSTAGES + 1;
    static constexpr int kXchg = kBar + kNumBars * 8;  // [2 halves][m, l][128 rows] floats
    static constexpr int kMisc = kXchg + 2 * 2 * BM * 4;
    static constexpr int kBytes = kMisc + 16;
    // the dynamic shared memory base is 1024-byte aligned (checked at run time)
    static constexpr int kAlloc = kBytes;
    static_assert(kAlloc <= 227 * 1024, "shared memory budget");
    static_assert(NSBUF * BN + 2 * D <= (int)kTmemCols, "TMEM budget");  // S buffers, O_0, O_1
};

struct Params {
    CUtensorMap tm_q, tm_ksum, tm_kwin, tm_vsum, tm_vwin, tm_o;
    int k, w, G, Hq, Hkv, Tc, Tk, batch;
    int Gp, HP;          // q heads per query tile (min(G, 128/k)) and head parts per kv head (G / Gp)
    int unit_chunks;
    int64_t aug_rows;
    float scale_log2;   // scale * log2(e)
    float scale;
    const int32_t *cu;
    Plan pl;
    int32_t *err;
    const __nv_bfloat16 *q;   // augmented query tensor (read row by row into TMEM)
    const __nv_bfloat16 *kk, *vv;   // augmented K and V (the summary rows' keys, read by the epilogue warps)
    __nv_bfloat16 *o;
    float *lse;
    // Chunk mode (a block of new tokens against a decode cache): per-sequence
    // arrays of the chunk plan, all null in the plain prefill.  Chunks and
    // summaries are then numbered from the sequence's start (absolute), and
    // each map has its own origin: q/o map chunk = qbase + c, window map
    // chunk = kvbase + c.  The summary maps then cover the cache itself,
    // dims (d, slot, kv head, sequence), summary j at slot sum_slot0 + j
    // (the plain prefill: all origins are the sequence's first chunk and
    // summary j is slot k of chunk j).
    const int32_t *ck_tile_off;   // [B+1] first work unit of each sequence
    const int32_t *ck_cbeg;       // [B] first query chunk
    const int32_t *ck_ntot;       // [B] text tokens after the block
    const int32_t *ck_qbase, *ck_kvbase;
    int sum_slot0;
    int sum_rows;   // 1: the epilogue warps also compute the summary rows of each item's chunks
};

// ---------------------------------------------------------------------------
// PTX wrappers: tc_sm100.cuh
// ---------------------------------------------------------------------------
using namespace tc;

// Instruction descriptor with M = BM.
__host__ __device__ constexpr uint32_t idesc_bf16(int n, bool b_mn_major) { return idesc_f16(BM, n, b_mn_major); }

// ---------------------------------------------------------------------------
// The kernel
// ---------------------------------------------------------------------------

// A work item: one query tile of 128 TMEM lanes (GQA-packed rows: Gp of the
// G q heads of one kv head, starting at q head h0, for unit_chunks chunks)
// and its list of 128-key K/V tiles: the window tiles covering chunks
// c0-w .. cend-1, then the summary tiles.  When G k > 128 the G heads are
// split over G / Gp items, each loading the same K/V tiles.  unit_of is
// host-callable too, so that CPU tests can check the tile lists it yields
// against the dense mask.
struct Unit {
    int hkv, h0, b, nb, mb, ncb, qbase, kvbase, sbase, c0, cend, cw_lo, n_win, T;
};

__host__ __device__ __forceinline__ Unit unit_of(const Params &P, int item, int n_units)
{
    Unit U;
    const int per = P.Hkv * P.HP;
    const int rank = item / per;
    U.hkv = (item % per) / P.HP;
    U.h0 = U.hkv * P.G + ((item % per) % P.HP) * P.Gp;
    const int u = n_units - 1 - rank;  // heaviest (latest) units first
    const int32_t *toff = P.ck_tile_off ? P.ck_tile_off : P.pl.tile_off;
    int lo = 0, hi = P.batch - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (toff[mid] <= u) lo = mid; else hi = mid - 1;
    }
    const int b = lo;
    U.b = b;
    if (P.ck_tile_off) {
        U.nb = P.ck_ntot[b];
        U.qbase = P.ck_qbase[b];
        U.kvbase = P.ck_kvbase[b];
        U.sbase = P.sum_slot0;
        U.c0 = P.ck_cbeg[b] + (u - toff[b]) * P.unit_chunks;
    } else {
        U.nb = P.cu[b + 1] - P.cu[b];
        U.qbase = U.kvbase = U.sbase = P.pl.chunk_off[b];
        U.c0 = (u - toff[b]) * P.unit_chunks;
    }
    U.mb = U.nb / P.k;
    U.ncb = (int)(((int64_t)U.nb + P.k - 1) / P.k);
    U.cend = min(U.ncb, U.c0 + P.unit_chunks);
    const int ns = max(min(U.mb, U.cend - 1 - P.w), 0);   // summaries any row may see
    U.cw_lo = max(0, U.c0 - P.w);
    U.n_win = (U.cend - U.cw_lo + P.Tk - 1) / P.Tk;
    U.T = U.n_win + (ns + BN - 1) / BN;
    return U;
}

// The work item a CTA takes in its n-th round.  Items are numbered heaviest
// first; the rounds alternate direction over the CTAs (snake order), so each
// CTA gets a light item for every heavy one and all CTAs finish together.
__device__ __forceinline__ int item_of_round(int n)
{
    const int g = (int)gridDim.x, b = (int)blockIdx.x;
    return n * g + ((n & 1) ? g - 1 - b : b);
}

// Summary rows (section 2.2.1 and Figure 4c): s_j attends to the k text
// tokens of its chunk and to itself, which are exactly the k+1 consecutive
// augmented rows of chunk j.  One warp computes q heads h0 .. h0+ng-1 of kv
// head hkv for global chunk gc, on the CUDA cores in fp32 with an online
// softmax over the keys; lane l holds dims [l D/32, (l+1) D/32).  The
// epilogue warps run it between items: the rows are independent of the
// text rows' pipeline and take ~0.05 % of the FLOPs.
template <int D>
__device__ __forceinline__ void summary_rows_warp(const Params &P, int64_t gc, int hkv, int h0, int ng, int lane)
{
    constexpr int DL = D / 32;          // dims per lane: 4 (one 8-byte load) or 2 (one 4-byte load)
    constexpr int KB = D == 128 ? 2 : 8;   // keys loaded together (their loads are in flight at once)
    static_assert(DL == 2 || DL == 4, "head_dim 64 or 128");
    using Vec = typename std::conditional<DL == 4, uint2, uint32_t>::type;
    const int k = P.k;
    const int64_t row0 = gc * (k + 1);
    const int64_t srow = row0 + k;
    const float sl2 = P.scale_log2;
    auto unpack = [](const Vec &v, float *f) {
        const uint32_t *w = reinterpret_cast<const uint32_t *>(&v);
#pragma unroll
        for (int e = 0; e < DL / 2; ++e) {
            const float2 x = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w[e]));
            f[2 * e] = x.x;
            f[2 * e + 1] = x.y;
        }
    };
    const Vec *Kr = reinterpret_cast<const Vec *>(P.kk + (row0 * P.Hkv + hkv) * D) + lane;
    const Vec *Vr = reinterpret_cast<const Vec *>(P.vv + (row0 * P.Hkv + hkv) * D) + lane;
    const int64_t rstride = (int64_t)P.Hkv * (D / DL);   // Vec per augmented row
    for (int g0 = 0; g0 < ng; g0 += 4) {
        const int gn = min(4, ng - g0);
        float q[4][DL], o[4][DL], m[4], l[4];
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            m[g] = -INFINITY;
            l[g] = 0.f;
#pragma unroll
            for (int e = 0; e < DL; ++e) o[g][e] = 0.f;
            Vec qv;
            if (g < gn)
                qv = reinterpret_cast<const Vec *>(P.q + (srow * P.Hq + h0 + g0 + g) * D)[lane];
            else
                qv = Vec{};
            unpack(qv, q[g]);
        }
        for (int r0 = 0; r0 <= k; r0 += KB) {
            Vec kv[KB], vv[KB];
#pragma unroll
            for (int u = 0; u < KB; ++u) {
                if (r0 + u <= k) {
                    kv[u] = Kr[(r0 + u) * rstride];
                    vv[u] = Vr[(r0 + u) * rstride];
                }
            }
#pragma unroll
            for (int u = 0; u < KB; ++u) {
                if (r0 + u > k) break;
                float kf[DL], vf[DL];
                unpack(kv[u], kf);
                unpack(vv[u], vf);
                float sc[4];
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    sc[g] = 0.f;
#pragma unroll
                    for (int e = 0; e < DL; ++e) sc[g] = fmaf(q[g][e], kf[e], sc[g]);
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1)
#pragma unroll
                    for (int g = 0; g < 4; ++g) sc[g] += __shfl_xor_sync(0xffffffffu, sc[g], off);
#pragma unroll
                for (int g = 0; g < 4; ++g) {
                    const float x = sc[g] * sl2;
                    const float mn = fmaxf(m[g], x);
                    const float corr = ex2(m[g] - mn);   // 0 on the first key
                    const float pr = ex2(x - mn);
                    l[g] = l[g] * corr + pr;
#pragma unroll
                    for (int e = 0; e < DL; ++e) o[g][e] = fmaf(pr, vf[e], o[g][e] * corr);
                    m[g] = mn;
                }
            }
        }
#pragma unroll
        for (int g = 0; g < 4; ++g) {
            if (g >= gn) break;
            const int head = h0 + g0 + g;
            const float inv = 1.f / l[g];
            Vec ov;
            uint32_t *w = reinterpret_cast<uint32_t *>(&ov);
#pragma unroll
            for (int e = 0; e < DL / 2; ++e) w[e] = pack_bf16(o[g][2 * e] * inv, o[g][2 * e + 1] * inv);
            reinterpret_cast<Vec *>(P.o + (srow * P.Hq + head) * D)[lane] = ov;
            if (P.lse && lane == 0) P.lse[srow * P.Hq + head] = (m[g] + log2f(l[g])) * 0.69314718055994530942f;
        }
    }
}

// Persistent kernel: one CTA per SM walks one work item per round (heavy
// first, in snake order over the CTAs), so the loads and
// first MMAs of the next item overlap the last tiles and the epilogue of
// the current one.  Every role walks the same item list; barrier phases
// follow a tile counter that runs on across items.
//
// The eight softmax warps split every key tile into two halves of 64 keys;
// each half keeps its own running max, row sum and O accumulator in TMEM and
// writes its P into its own half of the S buffer, so the two warps sharing an
// SM sub-partition never wait for each other.  The halves merge in the
// epilogue.
template <int D>
__global__ void __launch_bounds__(kThreads, 1) prefill_kernel(const __grid_constant__ Params P)
{
    using L = SmemLayout<D>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t *smem = smem_raw;
    const uint32_t sbase = smem_u32(smem);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMisc);
    volatile int *abort = reinterpret_cast<volatile int *>(smem + L::kMisc + 4);
    float *xchg = reinterpret_cast<float *>(smem + L::kXchg);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (*P.err != 0) return;
    if (sbase & 1023u) {   // the 128-byte swizzled tiles need a 1024-byte aligned base
        if (threadIdx.x == 0) set_error(P.err, KSA_ERR_UNSUPPORTED);
        return;
    }
    const int n_units = P.ck_tile_off ? P.ck_tile_off[P.batch] : P.pl.tile_off[P.batch];
    const int W = n_units * P.Hkv * P.HP;   // work items
    if ((int)blockIdx.x >= W) return;

    auto bar = [&](int i) { return sbase + L::kBar + 8u * (uint32_t)i; };
    auto B_KF = [&](int s) { return s; };
    auto B_KE = [&](int s) { return KSTAGES + s; };
    auto B_VF = [&](int s) { return 2 * KSTAGES + s; };
    auto B_VE = [&](int s) { return 2 * KSTAGES + VSTAGES + s; };
    constexpr int kB0 = 2 * KSTAGES + 2 * VSTAGES;
    auto B_S = [&](int bf) { return kB0 + bf; };
    auto B_P = [&](int h, int bf) { return kB0 + NSBUF + h * NSBUF + bf; };
    auto B_O = [&](int bf) { return kB0 + 3 * NSBUF + bf; };
    const int B_DRAIN_QK = kB0 + 4 * NSBUF;
    const int B_DRAIN_PV = B_DRAIN_QK + 1;
    const int B_OFREE = B_DRAIN_QK + 2;   // epilogue read O: the next item's PV may overwrite it
    auto B_QF = [&](int q) { return B_DRAIN_QK + 3 + q; };            // query tile landed
    auto B_QE = [&](int q) { return B_DRAIN_QK + 3 + QSTAGES + q; };  // its QKs are done
    const int B_UDONE = B_DRAIN_QK + 3 + 2 * QSTAGES;                  // softmax finished the item

    // ---- setup -----------------------------------------------------------
    if (threadIdx.x == 0) {
        for (int q = 0; q < QSTAGES; ++q) {
            mbar_init(bar(B_QF(q)), 1);
            mbar_init(bar(B_QE(q)), 1);
        }
        for (int s = 0; s < KSTAGES; ++s) {
            mbar_init(bar(B_KF(s)), 1);
            mbar_init(bar(B_KE(s)), 1);
        }
        for (int s = 0; s < VSTAGES; ++s) {
            mbar_init(bar(B_VF(s)), 1);
            mbar_init(bar(B_VE(s)), 1);
        }
        for (int bf = 0; bf < NSBUF; ++bf) {
            mbar_init(bar(B_S(bf)), 1);
            mbar_init(bar(B_P(0, bf)), 128);
            mbar_init(bar(B_P(1, bf)), 128);
            mbar_init(bar(B_O(bf)), 1);
        }
        mbar_init(bar(B_DRAIN_QK), 1);
        mbar_init(bar(B_DRAIN_PV), 1);
        mbar_init(bar(B_OFREE), 128);   // the epilogue warps
        mbar_init(bar(B_UDONE), 256);   // the softmax warps
        *abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // V rows a short window box leaves untouched must hold finite values
    // (P is 0 there, and 0 * NaN would poison O).
    if (P.Tk * P.k < BN) {
        uint4 *vz = reinterpret_cast<uint4 *>(smem + L::kV);
        for (int i = threadIdx.x; i < VSTAGES * L::kKVTile / 16; i += kThreads) vz[i] = make_uint4(0, 0, 0, 0);
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    if (warp == kWarpQK) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    auto S_COL = [&](int bf) { return tmem + (uint32_t)(bf * BN); };
    auto O_COL = [&](int h) { return tmem + (uint32_t)(NSBUF * BN + h * D); };

    const uint32_t q_bytes = (uint32_t)(P.Gp * P.k * P.Tc) * 128u * (D / 64);
    const uint32_t win_bytes = (uint32_t)(P.k * P.Tk) * 128u * (D / 64);
    const uint32_t sum_bytes = (uint32_t)BN * 128u * (D / 64);
    constexpr uint32_t kQHalf = BM * 128;   // bytes of one 64-column half of the query tile
    constexpr uint32_t kKVHalf = BN * 128;  // bytes of one 64-column half of a K/V tile

    if (warp == kWarpTMA || warp == kWarpTMAV) {
        // ================= TMA producers: Q and K (warp 8), V (warp 11) =================
        if (lane == 0) {
            const bool isk = warp == kWarpTMA;
            const int nst = isk ? KSTAGES : VSTAGES;
            int issued[KSTAGES > VSTAGES ? KSTAGES : VSTAGES] = {0};
            int q_issued[QSTAGES] = {0};
            bool ok = true;
            int gt = 0;
            for (int n = 0, item; (item = item_of_round(n)) < W && ok; ++n) {
                const Unit U = unit_of(P, item, n_units);
                if (isk) {
                    // query buffer n % 2 is free once the QKs of item n - 2 are done
                    const int qb = n % QSTAGES;
                    if (n >= QSTAGES &&
                        !(ok = mbar_wait(bar(B_QE(qb)), (uint32_t)((n / QSTAGES) - 1) & 1u, abort, P.err)))
                        break;
                    mbar_expect_tx(bar(B_QF(qb)), q_bytes);
                    for (int hf = 0; hf < D / 64; ++hf)
                        tma_load_4d(sbase + L::kQ + qb * L::kQTile + hf * kQHalf, &P.tm_q, bar(B_QF(qb)), hf * 64,
                                    U.h0, 0, U.qbase + U.c0);
                    q_issued[qb]++;
                }
                for (int j = 0; j < U.T && ok; ++j, ++gt) {
                    const int st = gt % nst;
                    const bool win = j < U.n_win;
                    const uint32_t bytes = win ? win_bytes : sum_bytes;
                    const CUtensorMap *mp = isk ? (win ? &P.tm_kwin : &P.tm_ksum) : (win ? &P.tm_vwin : &P.tm_vsum);
                    // window: (d, head, slot 0, chunk); summaries: (d, head, slot k,
                    // chunk) over the augmented rows, or (d, slot, head, sequence)
                    // over the cache in chunk mode
                    int c1 = U.hkv, c2 = win ? 0 : P.k;
                    int c3 = win ? U.kvbase + U.cw_lo + j * P.Tk : U.sbase + (j - U.n_win) * BN;
                    if (!win && P.ck_tile_off) { c1 = c3; c2 = U.hkv; c3 = U.b; }
                    const int bempty = isk ? B_KE(st) : B_VE(st), bfull = isk ? B_KF(st) : B_VF(st);
                    const uint32_t dst = sbase + (isk ? L::kK : L::kV) + st * L::kKVTile;
                    if (gt >= nst &&
                        !(ok = mbar_wait(bar(bempty), (uint32_t)((gt / nst) - 1) & 1u, abort, P.err)))
                        break;
                    mbar_expect_tx(bar(bfull), bytes);
                    for (int hf = 0; hf < D / 64; ++hf)
                        tma_load_4d(dst + hf * kKVHalf, mp, bar(bfull), hf * 64, c1, c2, c3);
                    issued[st]++;
                }
            }
            if (!ok) {
                // drain: every load issued must land before the CTA exits
                for (int st = 0; st < nst; ++st)
                    if (issued[st]) {
                        const uint32_t ph = (uint32_t)(issued[st] - 1) & 1u;
                        const int bfull = isk ? B_KF(st) : B_VF(st);
                        for (uint32_t it = 0; it < kSpinLimit && !mbar_try_wait(bar(bfull), ph); ++it) {}
                    }
                if (isk)
                    for (int qb = 0; qb < QSTAGES; ++qb)
                        if (q_issued[qb]) {
                            const uint32_t ph = (uint32_t)(q_issued[qb] - 1) & 1u;
                            for (uint32_t it = 0; it < kSpinLimit && !mbar_try_wait(bar(B_QF(qb)), ph); ++it) {}
                        }
            }
        }
    } else if (warp == kWarpQK) {
        // ================= S = Q K^T issuer =================
        // S of tile gt goes to buffer gt % 2, free once both halves' PV of
        // tile gt - 2 (which read P from it) has completed.
        if (lane == 0) {
            const uint32_t id_qk = idesc_bf16(BN, false);
            bool ok = true;
            int gt = 0;
            for (int n = 0, item; (item = item_of_round(n)) < W && ok; ++n) {
                const Unit U = unit_of(P, item, n_units);
                const int qb = n % QSTAGES;
                const uint32_t qa = sbase + L::kQ + qb * L::kQTile;
                if (!(ok = mbar_wait(bar(B_QF(qb)), (uint32_t)(n / QSTAGES) & 1u, abort, P.err))) break;
                for (int j = 0; j < U.T && ok; ++j, ++gt) {
                    const int s = gt % KSTAGES, bf = gt % NSBUF;
                    if (!(ok = mbar_wait(bar(B_KF(s)), (uint32_t)(gt / KSTAGES) & 1u, abort, P.err))) break;
                    if (gt >= NSBUF &&
                        !(ok = mbar_wait(bar(B_O(bf)), (uint32_t)((gt - NSBUF) / NSBUF) & 1u, abort, P.err)))
                        break;
                    tc_fence_after();
                    const uint32_t ka = sbase + L::kK + s * L::kKVTile;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk)
                        mma_ss(S_COL(bf), sdesc(qa + (kk / 4) * kQHalf + (kk % 4) * 32, 16, 1024),
                               sdesc(ka + (kk / 4) * kKVHalf + (kk % 4) * 32, 16, 1024), id_qk, kk > 0);
                    tc_commit(bar(B_S(bf)));
                    tc_commit(bar(B_KE(s)));
                }
                if (ok) tc_commit(bar(B_QE(qb)));
            }
            tc_commit(bar(B_DRAIN_QK));
            for (uint32_t it = 0; it < kSpinLimit && !mbar_try_wait(bar(B_DRAIN_QK), 0); ++it) {}
        }
    } else if (warp == kWarpPV) {
        // ================= O_h += P_h V_h issuer =================
        // Half h's P (its 64 keys as bf16 pairs) sits in S columns
        // [64h, 64h + 32); it multiplies V rows [64h, 64h + 64).
        if (lane == 0) {
            const uint32_t id_pv = idesc_bf16(D, true);
            bool ok = true;
            int gt = 0;
            for (int n = 0, item; (item = item_of_round(n)) < W && ok; ++n) {
                const Unit U = unit_of(P, item, n_units);
                for (int j = 0; j < U.T && ok; ++j, ++gt) {
                    const int s = gt % VSTAGES, bf = gt % NSBUF;
                    if (!(ok = mbar_wait(bar(B_VF(s)), (uint32_t)(gt / VSTAGES) & 1u, abort, P.err))) break;
                    // the previous item's epilogue must have read O before it restarts
                    if (j == 0 && n > 0 &&
                        !(ok = mbar_wait(bar(B_OFREE), (uint32_t)(n - 1) & 1u, abort, P.err)))
                        break;
                    const uint32_t va = sbase + L::kV + s * L::kKVTile;
                    for (int h = 0; h < 2 && ok; ++h) {
                        if (!(ok = mbar_wait(bar(B_P(h, bf)), (uint32_t)(gt / NSBUF) & 1u, abort, P.err))) break;
                        tc_fence_after();
#pragma unroll
                        for (int kk = 0; kk < HC / 16; ++kk)
                            mma_ts(O_COL(h), S_COL(bf) + h * HC + kk * 8,
                                   sdesc(va + (h * (HC / 16) + kk) * 2048, kKVHalf, 1024), id_pv,
                                   (j > 0 || kk > 0) ? 1u : 0u);
                    }
                    if (!ok) break;
                    tc_commit(bar(B_O(bf)));
                    tc_commit(bar(B_VE(s)));
                }
            }
            tc_commit(bar(B_DRAIN_PV));
            for (uint32_t it = 0; it < kSpinLimit && !mbar_try_wait(bar(B_DRAIN_PV), 0); ++it) {}
        }
    } else if (warp < 8) {
        // ================= softmax: 8 warps, two independent key halves =================
        const int half = warp >> 2;                    // keys [64 half, 64 half + 64) of each tile
        const int quarter = warp & 3;
        const int R = quarter * 32 + lane;             // row = TMEM lane
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const int rows_per_chunk = P.k * P.Gp;
        const int cl = R / rows_per_chunk;             // row -> (chunk, slot, head)
        const int r_slot = (R / P.Gp) % P.k;
        const float sl2 = P.scale_log2;
        // An expired wait clears ok; every warp still walks all items.
        bool ok = true;
        int gt = 0;
        for (int n = 0, item; (item = item_of_round(n)) < W; ++n) {
            const Unit U = unit_of(P, item, n_units);
            const int c = U.c0 + cl;
            const int i = c * P.k + r_slot;            // local text index
            const bool valid = cl < P.Tc && c < U.ncb && i < U.nb;
            const int sum_lim = valid ? min(c - P.w, U.mb) : 0;   // sees s_j for j < sum_lim
            const int win_lo = valid ? max(0, c - P.w) * P.k : 0;
            float m_run = -INFINITY;   // this half's running max of raw scores (the P reference)
            float l_run = 0.f;         // this half's row sum
            for (int j = 0; j < U.T; ++j, ++gt) {
                if (!ok) continue;
                const int bf = gt % NSBUF;
                // mask interval [clo, chi) of this row in tile j, relative to this half
                int clo, chi;
                if (j < U.n_win) {
                    const int base = (U.cw_lo + j * P.Tk) * P.k;
                    clo = win_lo - base;
                    chi = valid ? i - base + 1 : 0;
                    chi = min(chi, P.Tk * P.k);
                } else {
                    const int js = (j - U.n_win) * BN;
                    clo = 0;
                    chi = sum_lim - js;
                }
                clo = max(clo - half * HC, 0);
                chi = min(chi - half * HC, HC);
                if (chi < clo) chi = clo;
                ok = __all_sync(0xffffffffu, mbar_wait(bar(B_S(bf)), (uint32_t)(gt / NSBUF) & 1u, abort, P.err));
                if (!ok) continue;
                uint32_t sr[HC];
                float *s = reinterpret_cast<float *>(sr);
                const bool full = __all_sync(0xffffffffu, clo == 0 && chi == HC);
                auto load_s = [&]() {
                    tc_fence_after();
#pragma unroll
                    for (int cc = 0; cc < HC / 32; ++cc)
                        tmem_ld32(S_COL(bf) + lane_off + half * HC + cc * 32, sr + cc * 32);
                    tmem_wait_ld();
                    if (!full) {
#pragma unroll
                        for (int e = 0; e < HC; ++e) s[e] = (e >= clo && e < chi) ? s[e] : -INFINITY;
                    }
                };
                load_s();
                // the row max of this half's 64 keys
                static_assert(HC == 64, "the max tree below covers 64 scores");
                float pm[8];   // three-input max: columns a, a+8, ..., a+56 into pm[a]
#pragma unroll
                for (int a = 0; a < 8; ++a) {
                    pm[a] = max3(s[a], s[a + 8], s[a + 16]);
                    pm[a] = max3(pm[a], s[a + 24], s[a + 32]);
                    pm[a] = max3(pm[a], s[a + 40], s[a + 48]);
                    pm[a] = fmaxf(pm[a], s[a + 56]);
                }
                const float mx = max3(max3(pm[0], pm[1], pm[2]), max3(pm[3], pm[4], pm[5]), fmaxf(pm[6], pm[7]));
                // lazy rescale: keep the reference unless the max exceeds it by
                // more than 8 in log2 units (P stays <= 256; exact either way)
                const float m_new = fmaxf(m_run, mx);
                const bool need = (m_new - m_run) * sl2 > 8.f || m_run == -INFINITY;
                if (__any_sync(0xffffffffu, need && m_new != -INFINITY)) {
                    const float corr = (m_run == -INFINITY) ? 0.f : ex2((m_run - m_new) * sl2);
                    if (j > 0) {
                        const int pb = (gt - 1) % NSBUF;
                        ok = __all_sync(0xffffffffu, mbar_wait(bar(B_O(pb)), (uint32_t)((gt - 1) / NSBUF) & 1u,
                                                               abort, P.err));
                        if (!ok) continue;
                        tc_fence_after();
#pragma unroll 1
                        for (int cc = 0; cc < D / 32; ++cc) {
                            uint32_t orr[32];
                            const uint32_t oa = O_COL(half) + lane_off + cc * 32;
                            tmem_ld32(oa, orr);
                            tmem_wait_ld();
#pragma unroll
                            for (int e = 0; e < 32; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * corr);
                            tmem_st32(oa, orr);
                        }
                    }
                    l_run *= corr;
                    m_run = m_new;
                }
                // P in two groups of 32 keys; each group's bf16 pairs go to TMEM
                // as soon as they are packed, so the first store overlaps the
                // second group's exponentials
                const float mb = (m_run == -INFINITY) ? 0.f : m_run * sl2;
                // x = s sl2 - mb and the row sums on packed fp32 pairs; the
                // sums keep eight partials (element e in partial e % 8)
                const uint64_t sl2x2 = f2_pack(sl2, sl2), nmbx2 = f2_pack(-mb, -mb);
                uint64_t ps2[4];
#pragma unroll
                for (int a = 0; a < 4; ++a) ps2[a] = 0ull;
#pragma unroll
                for (int grp = 0; grp < 2; ++grp) {
                    uint32_t pk[HC / 4];
#pragma unroll
                    for (int e2 = 0; e2 < HC / 4; ++e2) {
                        const int e = grp * (HC / 2) + 2 * e2;
                        float x0, x1;
                        f2_unpack(f2_fma(f2_pack(s[e], s[e + 1]), sl2x2, nmbx2), x0, x1);
                        const float p0 = ex2(x0), p1 = ex2(x1);
                        ps2[(e & 7) >> 1] = f2_add(ps2[(e & 7) >> 1], f2_pack(p0, p1));
                        pk[e2] = pack_bf16(p0, p1);
                    }
                    // P of this half -> S columns [64 half + 16 grp, +16) (its own S region)
                    tmem_st16(S_COL(bf) + lane_off + half * HC + grp * (HC / 4), pk);
                }
                float ps[8];
#pragma unroll
                for (int a = 0; a < 4; ++a) f2_unpack(ps2[a], ps[2 * a], ps[2 * a + 1]);
                l_run += ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar(B_P(half, bf)));
            }
            // ---- end of the item: this half's (m, l) to the epilogue warps,
            // which merge the halves once the item's last PV has completed.
            // The exchange buffer is free once the previous item's epilogue
            // has read it (it reads before releasing O). ----
            if (n > 0)
                ok = ok && __all_sync(0xffffffffu,
                                      mbar_wait(bar(B_OFREE), (uint32_t)(n - 1) & 1u, abort, P.err));
            float *xc = xchg;   // [half][m, l][row]
            xc[(half * 2 + 0) * BM + R] = m_run;
            xc[(half * 2 + 1) * BM + R] = l_run;
            mbar_arrive(bar(B_UDONE));
        }
    } else if (warp >= kWarpEpi) {
        // ================= epilogue: 4 warps, one row per thread =================
        // Merges the two halves' (m, l, O) of each item and stores O / l as
        // bf16 (and the LSE) while the softmax warps run the next item.  O is
        // free for the next item's first PV once it has been read (B_OFREE);
        // that PV waits for it, which bounds how far the softmax runs ahead.
        const int quarter = warp & 3;
        const int R = quarter * 32 + lane;
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const int rows_per_chunk = P.k * P.Gp;
        const int cl = R / rows_per_chunk;
        const int r_slot = (R / P.Gp) % P.k;
        const int g = R % P.Gp;
        const float sl2 = P.scale_log2;
        const bool leader = warp == kWarpEpi && lane == 0;
        bool ok = true;
        int gt = 0;   // tiles up to and including this item
        for (int n = 0, item; (item = item_of_round(n)) < W; ++n) {
            const Unit U = unit_of(P, item, n_units);
            gt += U.T;
            const int c = U.c0 + cl;
            const int i = c * P.k + r_slot;
            const bool valid = cl < P.Tc && c < U.ncb && i < U.nb;
            ok = ok && __all_sync(0xffffffffu, mbar_wait(bar(B_UDONE), (uint32_t)n & 1u, abort, P.err));
            ok = ok && __all_sync(0xffffffffu, mbar_wait(bar(B_O((gt - 1) % NSBUF)), (uint32_t)((gt - 1) / NSBUF) & 1u,
                                                         abort, P.err));
            tc_fence_after();
            const float *xc = xchg;
            const float m0 = xc[0 * BM + R], l0 = xc[1 * BM + R], m1 = xc[2 * BM + R], l1 = xc[3 * BM + R];
            const float M = fmaxf(m0, m1);
            const float f0 = (M == -INFINITY) ? 0.f : ex2((m0 - M) * sl2);
            const float f1 = (M == -INFINITY) ? 0.f : ex2((m1 - M) * sl2);
            const float Lr = l0 * f0 + l1 * f1;
            // Units whose chunks are all whole leave through a TMA store of the
            // staged tile (the query tile's box over o); the last unit of a
            // sequence stores its real rows one by one, so no padding row is written.
            const bool tma_out = U.c0 + P.Tc <= U.mb;
            if (tma_out) {
                // the staging buffer is free once the previous store has read it
                if (leader) asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
                asm volatile("bar.sync 13, 128;" ::: "memory");
            }
            const float inv = Lr > 0.f ? 1.f / Lr : 0.f;
            const float g0 = f0 * inv, g1 = f1 * inv;
            const int64_t row = (int64_t)(U.qbase + c) * (P.k + 1) + r_slot;
            const int head = U.h0 + g;
            uint4 *dst = reinterpret_cast<uint4 *>(P.o + (row * P.Hq + head) * D);
            const uint32_t stage_row = sbase + L::kO + (uint32_t)R * 128u;
#pragma unroll 1
            for (int cc = 0; cc < D / 32 && ok; ++cc) {
                uint32_t a0[32], a1[32];
                tmem_ld32(O_COL(0) + lane_off + cc * 32, a0);
                tmem_ld32(O_COL(1) + lane_off + cc * 32, a1);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    float v[8];
#pragma unroll
                    for (int z = 0; z < 8; ++z)
                        v[z] = __uint_as_float(a0[8 * e + z]) * g0 + __uint_as_float(a1[8 * e + z]) * g1;
                    const uint4 wv = make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]),
                                                pack_bf16(v[6], v[7]));
                    if (tma_out) {
                        // column col of row R: 64-column half col / 64, 16-byte chunk
                        // j = (col % 64) / 8, stored at chunk j ^ (R % 8) (128-byte swizzle)
                        const int col = cc * 32 + 8 * e;
                        const uint32_t hoff = (uint32_t)(col / 64) * kQHalf;
                        const uint32_t j = (uint32_t)((col % 64) / 8);
                        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(stage_row + hoff + ((j ^ (uint32_t)(R & 7)) << 4)),
                                     "r"(wv.x), "r"(wv.y), "r"(wv.z), "r"(wv.w)
                                     : "memory");
                    } else if (valid) {
                        dst[cc * 4 + e] = wv;
                    }
                }
            }
            if (ok && valid && P.lse) P.lse[row * P.Hq + head] = M * P.scale + logf(Lr);
            // O has been read: the PV issuer may start the next item
            tc_fence_before();
            mbar_arrive(bar(B_OFREE));
            if (tma_out) {
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                asm volatile("bar.sync 13, 128;" ::: "memory");
                if (leader && ok) {
#pragma unroll
                    for (int hf = 0; hf < D / 64; ++hf)
                        tma_store_4d(&P.tm_o, sbase + L::kO + hf * kQHalf, hf * 64, U.h0, 0, U.qbase + U.c0);
                    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
                }
            }
            // the summary rows of this item's complete chunks, one warp per chunk
            if (P.sum_rows && ok)
                for (int c2 = U.c0 + (warp - kWarpEpi); c2 < min(U.cend, U.mb); c2 += 4)
                    summary_rows_warp<D>(P, (int64_t)U.qbase + c2, U.hkv, U.h0, P.Gp, lane);
        }
        // every store has finished reading shared memory before the CTA exits
        if (leader) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
    }

    // ---- teardown --------------------------------------------------------
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kWarpQK) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                     : "memory");
    }
}

// ---------------------------------------------------------------------------
// Summary rows: s_j over the k text rows of its chunk and itself, which are
// exactly the k+1 contiguous rows of chunk j in the augmented layout.
// ---------------------------------------------------------------------------
struct SumArgs {
    int k, G, Hq, Hkv, batch;
    int64_t chunks;
    float scale_log2, scale;
    const int32_t *cu;
    Plan pl;
    int32_t *err;
    const __nv_bfloat16 *q, *kk, *v;
    __nv_bfloat16 *o;
    float *lse;
};

// One warp per (chunk, kv head) on the warp-level tensor-core MMA: the keys
// are the MMA rows (S^T = K Q^T, O^T = V^T P^T, G query heads as the 8 MMA
// columns), 16 keys per step with an online softmax across steps.  Lane
// (g, t) = (lane / 4, lane % 4) loads dims [32v + 8t, 32v + 8t + 8) of key
// rows g and g + 8 with 16-byte loads and feeds them to the MMA as they are
// (the dot product is invariant under a common permutation of d).
constexpr int kSumWarps = 4;

template <int D, int G>
__global__ void __launch_bounds__(kSumWarps * 32) summary_rows_kernel(SumArgs a)
{
    static_assert(G <= 8, "query heads per kv head must fit the 8 MMA columns");
    constexpr int NV = D / 32, NC = D / 16, NM = D / 16;
    __shared__ float s_o[kSumWarps][G][D];
    __shared__ float s_ml[kSumWarps][2][G];
    if (*a.err != 0) return;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t task = (int64_t)blockIdx.x * kSumWarps + warp;
    if (task >= a.chunks * a.Hkv) return;   // warp-uniform; only warp-level syncs below
    const int64_t gc = task / a.Hkv;
    const int h = (int)(task % a.Hkv);
    int lo = 0, hi = a.batch - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (a.pl.chunk_off[mid] <= gc) lo = mid; else hi = mid - 1;
    }
    const int b = lo;
    const int n = a.cu[b + 1] - a.cu[b];
    if (gc - a.pl.chunk_off[b] >= n / a.k) return;  // trailing partial chunk: no summary
    const int64_t row0 = gc * (a.k + 1);
    const int64_t srow = row0 + a.k;
    const int g = lane >> 2, tt = lane & 3;
    // B fragments of Q^T: column (head) g, k-chunk c = 2v + hh covers dims
    // 32v + 8tt + 4hh + {0,1} (b0) and {2,3} (b1): two bf16 words of q
    uint32_t qb[NC][2];
#pragma unroll
    for (int c = 0; c < NC; ++c) {
        const int d0 = 32 * (c / 2) + 8 * tt + 4 * (c % 2);
        if (g < G) {
            const uint32_t *qp = reinterpret_cast<const uint32_t *>(a.q + (srow * a.Hq + (int64_t)h * G + g) * D + d0);
            qb[c][0] = qp[0];
            qb[c][1] = qp[1];
        } else {
            qb[c][0] = qb[c][1] = 0u;
        }
    }
    float o[NM][4];
#pragma unroll
    for (int i = 0; i < NM; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};   // heads 2tt, 2tt + 1 (log2 units)
    const int64_t rstride = (int64_t)a.Hkv * (D / 8);   // uint4 per augmented row
    const uint4 *Kb = reinterpret_cast<const uint4 *>(a.kk) + row0 * rstride + (int64_t)h * (D / 8);
    const uint4 *Vb = reinterpret_cast<const uint4 *>(a.v) + row0 * rstride + (int64_t)h * (D / 8);
    // keys: rows 0 .. k of the chunk (its k text rows, then the summary itself)
    for (int kb = 0; kb <= a.k; kb += 16) {
        const int r0 = kb + g, r1 = kb + g + 8;
        const bool in0 = r0 <= a.k, in1 = r1 <= a.k;
        uint4 kA[NV], kB[NV], vA[NV], vB[NV];
#pragma unroll
        for (int v = 0; v < NV; ++v) {
            const uint4 z = make_uint4(0, 0, 0, 0);
            kA[v] = in0 ? Kb[r0 * rstride + 4 * v + tt] : z;
            kB[v] = in1 ? Kb[r1 * rstride + 4 * v + tt] : z;
            vA[v] = in0 ? Vb[r0 * rstride + 4 * v + tt] : z;
            vB[v] = in1 ? Vb[r1 * rstride + 4 * v + tt] : z;
        }
        float sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            const int v = c / 2, hh = c % 2;
            wm::mma16816(sc, wm::word(kA[v], 2 * hh), wm::word(kB[v], 2 * hh), wm::word(kA[v], 2 * hh + 1),
                         wm::word(kB[v], 2 * hh + 1), qb[c][0], qb[c][1]);
        }
        // sc[0..1]: key r0, heads 2tt, 2tt+1; sc[2..3]: key r1
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
            corr[e] = wm::ex2(m_run[e] - m_new);       // 0 on the first step
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
    // the G output rows of s_j: bf16 pairs, 128 contiguous bytes per instruction
    for (int idx = lane; idx < G * (D / 2); idx += 32) {
        const int gg = idx / (D / 2), w2 = idx % (D / 2);
        const float inv = 1.f / s_ml[warp][1][gg];
        const uint32_t pr = wm::pack2(s_o[warp][gg][2 * w2] * inv, s_o[warp][gg][2 * w2 + 1] * inv);
        reinterpret_cast<uint32_t *>(a.o + (srow * a.Hq + (int64_t)h * G + gg) * D)[w2] = pr;
    }
    if (a.lse && lane < G)
        a.lse[srow * a.Hq + (int64_t)h * G + lane] =
            (s_ml[warp][0][lane] + log2f(s_ml[warp][1][lane])) * 0.69314718055994530942f;
}

}  // namespace pf

// ---------------------------------------------------------------------------
// Host side
// ---------------------------------------------------------------------------

// Longest chunk whose summary rows the epilogue warps take (k + 1 keys per
// row, one warp per chunk).  Same box, 32K tokens, whole call: with the
// epilogue warps at every k, k = 16 / 32 / 64 took 1.05-1.09 / 1.07-1.08 /
// 1.61-1.62 ms; with the separate kernel above k = 8, 0.87-0.91 / 0.68-0.69
// / 0.67 ms; k = 8 unchanged (1.273-1.275 ms).
constexpr int kEpilogueSumMaxK = 8;

// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// 4-D view [chunks][k+1][H][d] of an augmented tensor, box (64, bh, bs, bc).
bool make_map(CUtensorMap *m, const void *base, int d, int H, int k, int64_t chunks, int bh, int bs, int bc)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)(k + 1), (cuuint64_t)chunks};
    cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2, (cuuint64_t)(k + 1) * H * d * 2};
    cuuint32_t box[4] = {64, (cuuint32_t)bh, (cuuint32_t)bs, (cuuint32_t)bc};
    cuuint32_t es[4] = {1, 1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// q heads per query tile: all G of a kv head when G k <= 128 rows, else as
// many as fit (128 / k); 0 when the shape is not supported.
int prefill_heads_per_tile(const ksa_params *p)
{
    const int G = p->num_q_heads / p->num_kv_heads;
    if (p->k < 1 || p->k > pf::BM) return 0;
    const int Gp = G < pf::BM / p->k ? G : pf::BM / p->k;
    return (Gp >= 1 && G % Gp == 0) ? Gp : 0;
}

int prefill_unit_chunks(const ksa_params *p)
{
    const int Gp = prefill_heads_per_tile(p);
    return Gp ? pf::BM / (Gp * p->k) : 0;
}

template <int D>
static int launch_prefill_t(const ksa_params *p, int batch, const int32_t *cu, int64_t total_text,
                            int64_t aug_rows, const void *qa, const void *ka, const void *va, void *oa,
                            float *lse, const Plan &pl, int32_t *err, cudaStream_t st)
{
    using L = pf::SmemLayout<D>;
    pf::Params P;
    const int k = p->k, Hq = p->num_q_heads, Hkv = p->num_kv_heads, G = Hq / Hkv;
    const int64_t chunks = aug_rows / (k + 1);
    P.k = k; P.w = p->w; P.G = G; P.Hq = Hq; P.Hkv = Hkv;
    P.Gp = prefill_heads_per_tile(p);
    if (P.Gp < 1) return KSA_ERR_UNSUPPORTED;
    P.HP = G / P.Gp;
    P.Tc = pf::BM / (P.Gp * k);
    P.Tk = pf::BN / k;
    if (P.Tc < 1 || P.Tk < 1) return KSA_ERR_UNSUPPORTED;
    P.batch = batch;
    P.unit_chunks = P.Tc;
    P.aug_rows = aug_rows;
    float scale = p->scale > 0.f ? p->scale : 1.0f / sqrtf((float)D);
    P.scale = scale;
    P.scale_log2 = scale * 1.4426950408889634f;
    P.cu = cu; P.pl = pl; P.err = err;
    P.q = (const __nv_bfloat16 *)qa;
    P.kk = (const __nv_bfloat16 *)ka;
    P.vv = (const __nv_bfloat16 *)va;
    P.o = (__nv_bfloat16 *)oa;
    P.lse = lse;
    P.ck_tile_off = P.ck_cbeg = P.ck_ntot = P.ck_qbase = P.ck_kvbase = nullptr;
    P.sum_slot0 = 0;
    // The summary rows run on the prefill kernel's epilogue warps (one warp
    // per chunk, between items) for chunks of up to 8 tokens; longer chunks
    // make those rows slow enough to hold up the items' O hand-off, so they
    // take the separate warp-MMA kernel after the prefill.
    P.sum_rows = k <= kEpilogueSumMaxK ? 1 : 0;
    bool ok = make_map(&P.tm_q, qa, D, Hq, k, chunks, P.Gp, k, P.Tc) &&
              make_map(&P.tm_ksum, ka, D, Hkv, k, chunks, 1, 1, pf::BN) &&
              make_map(&P.tm_kwin, ka, D, Hkv, k, chunks, 1, k, P.Tk) &&
              make_map(&P.tm_vsum, va, D, Hkv, k, chunks, 1, 1, pf::BN) &&
              make_map(&P.tm_vwin, va, D, Hkv, k, chunks, 1, k, P.Tk) &&
              make_map(&P.tm_o, oa, D, Hq, k, chunks, P.Gp, k, P.Tc);
    if (!ok) return KSA_ERR_CUDA;
    // persistent: one CTA per SM (shared memory and TMEM admit one); each
    // walks the work items round robin.  CTAs beyond the item count exit.
    int64_t units = total_text / ((int64_t)k * P.unit_chunks) + 2LL * batch + 1;
    int64_t grid = units * Hkv * P.HP;
    if (grid > sm_count()) grid = sm_count();
    static bool attr_set[2] = {false, false};
    if (!attr_set[D == 128]) {
        if (cudaFuncSetAttribute(pf::prefill_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc) !=
            cudaSuccess)
            return KSA_ERR_CUDA;
        attr_set[D == 128] = true;
    }
    pf::prefill_kernel<D><<<(unsigned)grid, pf::kThreads, L::kAlloc, st>>>(P);
    if (cudaGetLastError() != cudaSuccess) return KSA_ERR_CUDA;
    if (!P.sum_rows) {
        pf::SumArgs s;
        s.k = k; s.G = G; s.Hq = Hq; s.Hkv = Hkv; s.batch = batch; s.chunks = chunks;
        s.scale = scale; s.scale_log2 = P.scale_log2;
        s.cu = cu; s.pl = pl; s.err = err;
        s.q = (const __nv_bfloat16 *)qa; s.kk = (const __nv_bfloat16 *)ka; s.v = (const __nv_bfloat16 *)va;
        s.o = (__nv_bfloat16 *)oa; s.lse = lse;
        const int64_t tasks = chunks * Hkv;
        if (tasks > 0) {
            const unsigned blocks = (unsigned)((tasks + pf::kSumWarps - 1) / pf::kSumWarps);
            const unsigned thr = pf::kSumWarps * 32;
            switch (G) {
            case 1: pf::summary_rows_kernel<D, 1><<<blocks, thr, 0, st>>>(s); break;
            case 2: pf::summary_rows_kernel<D, 2><<<blocks, thr, 0, st>>>(s); break;
            case 4: pf::summary_rows_kernel<D, 4><<<blocks, thr, 0, st>>>(s); break;
            case 8: pf::summary_rows_kernel<D, 8><<<blocks, thr, 0, st>>>(s); break;
            default: return KSA_ERR_UNSUPPORTED;
            }
            if (cudaGetLastError() != cudaSuccess) return KSA_ERR_CUDA;
        }
    }
    return KSA_OK;
}

// Summary tiles straight from a decode cache [B, Hkv, S, d]: dims (d, slot,
// kv head, sequence), boxes of 128 slots of one (sequence, kv head).  Slots
// past S are outside the map and load as zeros.
static bool make_cache_map(CUtensorMap *m, const void *base, int d, int Hkv, int64_t S, int B)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)S, (cuuint64_t)Hkv, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)S * d * 2, (cuuint64_t)Hkv * S * d * 2};
    cuuint32_t box[4] = {64, (cuuint32_t)pf::BN, 1, 1};
    cuuint32_t es[4] = {1, 1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box, es,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <int D>
static int launch_prefill_cache_t(const ksa_params *p, const ksa_cache *c, const ChunkTiles &t, int32_t *err,
                                  cudaStream_t st)
{
    using L = pf::SmemLayout<D>;
    pf::Params P;
    const int k = p->k, Hq = p->num_q_heads, Hkv = p->num_kv_heads, G = Hq / Hkv;
    P.k = k; P.w = p->w; P.G = G; P.Hq = Hq; P.Hkv = Hkv;
    P.Gp = prefill_heads_per_tile(p);
    if (P.Gp < 1) return KSA_ERR_UNSUPPORTED;
    P.HP = G / P.Gp;
    P.Tc = pf::BM / (P.Gp * k);
    P.Tk = pf::BN / k;
    if (P.Tc < 1 || P.Tk < 1) return KSA_ERR_UNSUPPORTED;
    P.batch = c->batch;
    P.unit_chunks = P.Tc;
    P.aug_rows = t.q_chunks * (k + 1);
    const float scale = p->scale > 0.f ? p->scale : 1.0f / sqrtf((float)D);
    P.scale = scale;
    P.scale_log2 = scale * 1.4426950408889634f;
    P.cu = nullptr;
    P.pl = Plan{nullptr, nullptr, nullptr, nullptr};
    P.err = err;
    P.q = (const __nv_bfloat16 *)t.qa;
    P.kk = P.vv = nullptr;
    P.o = (__nv_bfloat16 *)t.oa;
    P.lse = t.lse;
    P.sum_rows = 0;
    P.ck_tile_off = t.tile_off; P.ck_cbeg = t.cbeg; P.ck_ntot = t.ntot;
    P.ck_qbase = t.qbase; P.ck_kvbase = t.kvbase;
    P.sum_slot0 = 1 + k + p->w * k;
    const int64_t S = 1 + (int64_t)k + (int64_t)p->w * k + c->cap_summaries;
    bool ok = make_map(&P.tm_q, t.qa, D, Hq, k, t.q_chunks, P.Gp, k, P.Tc) &&
              make_map(&P.tm_o, t.oa, D, Hq, k, t.q_chunks, P.Gp, k, P.Tc) &&
              make_map(&P.tm_kwin, t.ka, D, Hkv, k, t.kv_chunks, 1, k, P.Tk) &&
              make_map(&P.tm_vwin, t.va, D, Hkv, k, t.kv_chunks, 1, k, P.Tk) &&
              make_cache_map(&P.tm_ksum, c->k, D, Hkv, S, c->batch) &&
              make_cache_map(&P.tm_vsum, c->v, D, Hkv, S, c->batch);
    if (!ok) return KSA_ERR_CUDA;
    int64_t grid = t.max_units * Hkv * P.HP;
    if (grid > sm_count()) grid = sm_count();
    if (grid < 1) return KSA_OK;
    static bool attr_set[2] = {false, false};
    if (!attr_set[D == 128]) {
        if (cudaFuncSetAttribute(pf::prefill_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc) !=
            cudaSuccess)
            return KSA_ERR_CUDA;
        attr_set[D == 128] = true;
    }
    pf::prefill_kernel<D><<<(unsigned)grid, pf::kThreads, L::kAlloc, st>>>(P);
    return cudaGetLastError() == cudaSuccess ? KSA_OK : KSA_ERR_CUDA;
}

int launch_prefill_cache(const ksa_params *p, const ksa_cache *c, const ChunkTiles &t, int32_t *err, cudaStream_t st)
{
    if (p->head_dim == 128) return launch_prefill_cache_t<128>(p, c, t, err, st);
    if (p->head_dim == 64) return launch_prefill_cache_t<64>(p, c, t, err, st);
    return KSA_ERR_UNSUPPORTED;
}

int launch_prefill(const ksa_params *p, int batch, const int32_t *cu, int64_t total_text, int64_t aug_rows,
                   const void *qa, const void *ka, const void *va, void *oa, float *lse, const Plan &pl,
                   int32_t *err, cudaStream_t st)
{
    if (aug_rows == 0) return KSA_OK;
    if (p->head_dim == 128)
        return launch_prefill_t<128>(p, batch, cu, total_text, aug_rows, qa, ka, va, oa, lse, pl, err, st);
    if (p->head_dim == 64)
        return launch_prefill_t<64>(p, batch, cu, total_text, aug_rows, qa, ka, va, oa, lse, pl, err, st);
    return KSA_ERR_UNSUPPORTED;
}

}  // namespace ksa

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
//     tile serves all G heads).  Each CTA runs two query tiles (two softmax
//     warpgroups) against one stream of K/V tiles: S = Q K^T and O += P V
//     are tcgen05.mma (kind::f16, bf16 in, fp32 accumulate in TMEM); P is
//     written back into TMEM as bf16 over S and fed as the A operand.
//   * The set of K/V tiles of a work unit follows from its chunk
//     coordinates: ceil(min(m, c_last-w)/128) summary tiles plus the window
//     tiles covering chunks c_first-w .. c_last.  Every other tile of the
//     L x L plane is skipped without being looked at.  Inside a tile the
//     mask of a row is one interval of columns, computed from coordinates.
//   * Warp roles: warps 0-7 softmax (two warpgroups), warp 8 TMA producer,
//     warp 9 MMA issuer and TMEM owner.  All mbarrier waits are bounded; on
//     expiry the CTA records KSA_ERR_TIMEOUT, drains, frees TMEM and exits.
//   * Summary query rows (k+1 keys each) run in a separate CUDA-core kernel.
#include <cuda.h>
#include <math.h>

#include "ksa_internal.cuh"

namespace ksa {

namespace pf {

constexpr int BM = 128;        // rows per query tile (= TMEM lanes)
constexpr int BN = 128;        // keys per K/V tile
constexpr int NQ = 2;          // query tiles per CTA
constexpr int STAGES = 2;      // K/V pipeline depth
constexpr int kWarpTMA = 8;
constexpr int kWarpMMA = 9;
constexpr int kThreads = 320;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSpinLimit = 1u << 22;  // bounded waits (~0.5-4 s)

template <int D>
struct SmemLayout {
    static constexpr int kTile = BM * D * 2;  // bytes of one 128 x D bf16 tile
    static constexpr int kQ = 0;
    static constexpr int kK = kQ + NQ * kTile;
    static constexpr int kV = kK + STAGES * kTile;
    static constexpr int kBar = kV + STAGES * kTile;
    // barriers: q, kfull[S], kempty[S], vfull[S], vempty[S], s[NQ], p[NQ], o[NQ], drain
    static constexpr int kNumBars = 1 + 4 * STAGES + 3 * NQ + 1;
    static constexpr int kMisc = kBar + kNumBars * 8;
    static constexpr int kBytes = kMisc + 16;
    // room to align the base to 1024; the rest of the SM's 227 KB is kept as
    // slack (one CTA per SM either way: TMEM holds 512 columns)
    static constexpr int kAlloc = 227 * 1024;
    static_assert(kBytes + 1024 <= kAlloc, "shared memory budget");
};

struct Params {
    CUtensorMap tm_q, tm_ksum, tm_kwin, tm_vsum, tm_vwin;
    int k, w, G, Hq, Hkv, Tc, Tk, batch;
    int unit_chunks;
    int64_t aug_rows;
    float scale_log2;   // scale * log2(e)
    float scale;
    const int32_t *cu;
    Plan pl;
    int32_t *err;
    __nv_bfloat16 *o;
    float *lse;
};

// ---------------------------------------------------------------------------
// PTX wrappers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait: false (after flagging the CTA and the error word) if the
// phase did not complete within kSpinLimit polls or another role aborted.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int *abort,
                                          int32_t *err)
{
    for (uint32_t it = 0; it < kSpinLimit; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort) return false;
    }
    *abort = 1;
    set_error(err, KSA_ERR_TIMEOUT);
    return false;
}

__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap *map, uint32_t bar,
                                            int c0, int c1, int c2, int c3)
{
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T
__device__ __forceinline__ void mma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc]
__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a, uint64_t b, uint32_t idesc, uint32_t acc)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d),
        "r"(a), "l"(b), "r"(idesc), "r"(acc)
        : "memory");
}

// 32 consecutive TMEM columns of this thread's lane -> 32 registers
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t *r)
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t *r)
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
        "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
        "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// Shared-memory matrix descriptor (tcgen05), 128-byte swizzle.
//   bits 0-13 start>>4, 16-29 leading byte offset>>4, 32-45 stride byte
//   offset>>4, 46-47 version 1, 61-63 layout (2 = 128B swizzle).
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);
    d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

// Instruction descriptor, kind::f16: D fp32, A and B bf16, M = 128.
__host__ __device__ constexpr uint32_t idesc_bf16(int n, bool b_mn_major)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) |
           ((uint32_t)(n >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}

// ---------------------------------------------------------------------------
// The kernel
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(kThreads, 1) prefill_kernel(const __grid_constant__ Params P)
{
    using L = SmemLayout<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = smem_u32(smem);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + L::kBar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + L::kMisc);
    volatile int *abort = reinterpret_cast<volatile int *>(smem + L::kMisc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // ---- work unit -------------------------------------------------------
    if (*P.err != 0) return;
    const int n_units = P.pl.tile_off[P.batch];
    const int rank = blockIdx.x / P.Hkv;
    const int hkv = blockIdx.x % P.Hkv;
    if (rank >= n_units) return;
    const int u = n_units - 1 - rank;  // longest (latest) units first
    int b;
    {
        int lo = 0, hi = P.batch - 1;
        while (lo < hi) {
            int mid = (lo + hi + 1) >> 1;
            if (P.pl.tile_off[mid] <= u) lo = mid; else hi = mid - 1;
        }
        b = lo;
    }
    const int nb = P.cu[b + 1] - P.cu[b];
    const int mb = nb / P.k;                       // complete chunks = summaries
    const int ncb = (nb + P.k - 1) / P.k;          // chunks incl. a partial one
    const int goff = P.pl.chunk_off[b];            // first chunk in the layout
    const int c0 = (u - P.pl.tile_off[b]) * P.unit_chunks;
    const int cend = min(ncb, c0 + P.unit_chunks);
    int ns = min(mb, cend - 1 - P.w);              // summaries any row may see
    ns = max(ns, 0);
    const int n_sum_tiles = (ns + BN - 1) / BN;
    const int cw_lo = max(0, c0 - P.w);
    const int n_win_tiles = (cend - cw_lo + P.Tk - 1) / P.Tk;
    const int T = n_win_tiles + n_sum_tiles;

    auto bar = [&](int i) { return sbase + L::kBar + 8u * (uint32_t)i; };
    const int B_Q = 0;
    auto B_KF = [&](int s) { return 1 + s; };
    auto B_KE = [&](int s) { return 1 + STAGES + s; };
    auto B_VF = [&](int s) { return 1 + 2 * STAGES + s; };
    auto B_VE = [&](int s) { return 1 + 3 * STAGES + s; };
    auto B_S = [&](int q) { return 1 + 4 * STAGES + q; };
    auto B_P = [&](int q) { return 1 + 4 * STAGES + NQ + q; };
    auto B_O = [&](int q) { return 1 + 4 * STAGES + 2 * NQ + q; };
    const int B_DRAIN = 1 + 4 * STAGES + 3 * NQ;

    // ---- setup -----------------------------------------------------------
    if (threadIdx.x == 0) {
        mbar_init(bar(B_Q), 1);
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(bar(B_KF(s)), 1);
            mbar_init(bar(B_KE(s)), 1);
            mbar_init(bar(B_VF(s)), 1);
            mbar_init(bar(B_VE(s)), 1);
        }
        for (int q = 0; q < NQ; ++q) {
            mbar_init(bar(B_S(q)), 1);
            mbar_init(bar(B_P(q)), 128);
            mbar_init(bar(B_O(q)), 1);
        }
        mbar_init(bar(B_DRAIN), 1);
        *abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // V rows a short window box leaves untouched must hold finite values
    // (P is 0 there, and 0 * NaN would poison O).
    if (P.Tk * P.k < BN) {
        uint4 *vz = reinterpret_cast<uint4 *>(smem + L::kV);
        for (int i = threadIdx.x; i < STAGES * L::kTile / 16; i += kThreads) vz[i] = make_uint4(0, 0, 0, 0);
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
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
    auto S_COL = [&](int q) { return tmem + (uint32_t)(q * BN); };
    auto O_COL = [&](int q) { return tmem + (uint32_t)(NQ * BN + q * D); };

    const uint32_t q_bytes = (uint32_t)(P.G * P.k * P.Tc) * 128u * (D / 64);
    const uint32_t win_bytes = (uint32_t)(P.k * P.Tk) * 128u * (D / 64);
    const uint32_t sum_bytes = (uint32_t)BN * 128u * (D / 64);
    constexpr uint32_t kHalf = BM * 128;  // bytes of one 64-column half tile

    if (warp == kWarpTMA) {
        // ================= TMA producer =================
        if (lane == 0) {
            int issued_k[STAGES] = {0}, issued_v[STAGES] = {0};
            bool ok = true;
            mbar_expect_tx(bar(B_Q), q_bytes * NQ);
            for (int q = 0; q < NQ; ++q)
                for (int hf = 0; hf < D / 64; ++hf)
                    tma_load_4d(sbase + L::kQ + q * L::kTile + hf * kHalf, &P.tm_q, bar(B_Q), hf * 64,
                                hkv * P.G, 0, goff + c0 + q * P.Tc);
            for (int j = 0; j < T && ok; ++j) {
                const int s = j % STAGES;
                const uint32_t ph = (uint32_t)((j / STAGES) - 1) & 1u;
                const bool win = j < n_win_tiles;
                const uint32_t bytes = win ? win_bytes : sum_bytes;
                const CUtensorMap *mk = win ? &P.tm_kwin : &P.tm_ksum;
                const CUtensorMap *mv = win ? &P.tm_vwin : &P.tm_vsum;
                const int slot = win ? 0 : P.k;
                const int chunk = goff + (win ? cw_lo + j * P.Tk : (j - n_win_tiles) * BN);
                if (j >= STAGES && !(ok = mbar_wait(bar(B_KE(s)), ph, abort, P.err))) break;
                mbar_expect_tx(bar(B_KF(s)), bytes);
                for (int hf = 0; hf < D / 64; ++hf)
                    tma_load_4d(sbase + L::kK + s * L::kTile + hf * kHalf, mk, bar(B_KF(s)), hf * 64, hkv,
                                slot, chunk);
                issued_k[s]++;
                if (j >= STAGES && !(ok = mbar_wait(bar(B_VE(s)), ph, abort, P.err))) break;
                mbar_expect_tx(bar(B_VF(s)), bytes);
                for (int hf = 0; hf < D / 64; ++hf)
                    tma_load_4d(sbase + L::kV + s * L::kTile + hf * kHalf, mv, bar(B_VF(s)), hf * 64, hkv,
                                slot, chunk);
                issued_v[s]++;
            }
            if (!ok) {
                // drain: every load issued must land before the CTA exits
                for (int s = 0; s < STAGES; ++s) {
                    if (issued_k[s]) {
                        uint32_t ph = (uint32_t)(issued_k[s] - 1) & 1u;
                        for (uint32_t it = 0; it < kSpinLimit && !mbar_try_wait(bar(B_KF(s)), ph); ++it) {}
                    }
                    if (issued_v[s]) {
                        uint32_t ph = (uint32_t)(issued_v[s] - 1) & 1u;
                        for (uint32_t it = 0; it < kSpinLimit && !mbar_try_wait(bar(B_VF(s)), ph); ++it) {}
                    }
                }
                for (uint32_t it = 0; it < kSpinLimit && !mbar_try_wait(bar(B_Q), 0); ++it) {}
            }
        }
    } else if (warp == kWarpMMA) {
        // ================= MMA issuer =================
        if (lane == 0) {
            const uint32_t id_qk = idesc_bf16(BN, false);
            const uint32_t id_pv = idesc_bf16(D, true);
            bool ok = mbar_wait(bar(B_Q), 0, abort, P.err);
            tc_fence_after();
            for (int j = 0; j < T && ok; ++j) {
                const int s = j % STAGES;
                const uint32_t ph = (uint32_t)(j / STAGES) & 1u;
                if (!(ok = mbar_wait(bar(B_KF(s)), ph, abort, P.err))) break;
                tc_fence_after();
                for (int q = 0; q < NQ && ok; ++q) {
                    // S_q still holds P_q(j-1) until PV_q(j-1) has consumed it
                    if (j > 0 && !(ok = mbar_wait(bar(B_O(q)), (uint32_t)(j - 1) & 1u, abort, P.err))) break;
                    tc_fence_after();
                    const uint32_t qa = sbase + L::kQ + q * L::kTile;
                    const uint32_t ka = sbase + L::kK + s * L::kTile;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = (kk / 4) * kHalf + (kk % 4) * 32;
                        mma_ss(S_COL(q), sdesc(qa + off, 16, 1024), sdesc(ka + off, 16, 1024), id_qk, kk > 0);
                    }
                    tc_commit(bar(B_S(q)));
                }
                if (!ok) break;
                tc_commit(bar(B_KE(s)));
                if (!(ok = mbar_wait(bar(B_VF(s)), ph, abort, P.err))) break;
                tc_fence_after();
                for (int q = 0; q < NQ && ok; ++q) {
                    if (!(ok = mbar_wait(bar(B_P(q)), (uint32_t)j & 1u, abort, P.err))) break;
                    tc_fence_after();
                    const uint32_t va = sbase + L::kV + s * L::kTile;
#pragma unroll
                    for (int kk = 0; kk < BN / 16; ++kk)
                        mma_ts(O_COL(q), S_COL(q) + kk * 8, sdesc(va + kk * 2048, kHalf, 1024), id_pv,
                               (j > 0 || kk > 0) ? 1u : 0u);
                    tc_commit(bar(B_O(q)));
                }
                if (!ok) break;
                tc_commit(bar(B_VE(s)));
            }
            // all MMAs issued by this thread complete before TMEM is freed
            tc_commit(bar(B_DRAIN));
            for (uint32_t it = 0; it < kSpinLimit && !mbar_try_wait(bar(B_DRAIN), 0); ++it) {}
        }
    } else {
        // ================= softmax warpgroups =================
        const int q = warp >> 2;                       // query tile of this warpgroup
        const int R = (warp & 3) * 32 + lane;          // row = TMEM lane
        const uint32_t lane_off = (uint32_t)((warp & 3) * 32) << 16;
        // row -> (chunk, slot, head)
        const int rows_per_chunk = P.k * P.G;
        const int cl = R / rows_per_chunk;
        const int r_slot = (R / P.G) % P.k;
        const int g = R % P.G;
        const int c = c0 + q * P.Tc + cl;
        const int i = c * P.k + r_slot;                // local text index
        const bool valid = cl < P.Tc && c < ncb && i < nb;
        const int sum_lim = valid ? min(c - P.w, mb) : 0;   // sees s_j for j < sum_lim
        const int win_lo = valid ? max(0, c - P.w) * P.k : 0;
        const float sl2 = P.scale_log2;

        float m_run = -INFINITY;   // running max of raw scores used for P
        float l_run = 0.f;
        bool ok = true;
        for (int j = 0; j < T && ok; ++j) {
            // mask interval [clo, chi) of this row in tile j
            int clo, chi;
            if (j < n_win_tiles) {
                const int base = (cw_lo + j * P.Tk) * P.k;
                clo = win_lo - base;
                chi = valid ? i - base + 1 : 0;
                chi = min(chi, P.Tk * P.k);
            } else {
                const int js = (j - n_win_tiles) * BN;
                clo = 0;
                chi = sum_lim - js;
            }
            clo = max(clo, 0);
            chi = min(chi, BN);
            if (chi < clo) chi = clo;
            if (!(ok = mbar_wait(bar(B_S(q)), (uint32_t)j & 1u, abort, P.err))) break;
            tc_fence_after();
            uint32_t sr[BN];
#pragma unroll
            for (int cc = 0; cc < BN / 32; ++cc) tmem_ld32(S_COL(q) + lane_off + cc * 32, sr + cc * 32);
            tmem_wait_ld();
            float *s = reinterpret_cast<float *>(sr);
            const bool full = __all_sync(0xffffffffu, clo == 0 && chi == BN);
            float mx = -INFINITY;
            if (full) {
#pragma unroll
                for (int e = 0; e < BN; ++e) mx = fmaxf(mx, s[e]);
            } else {
#pragma unroll
                for (int e = 0; e < BN; ++e) {
                    s[e] = (e >= clo && e < chi) ? s[e] : -INFINITY;
                    mx = fmaxf(mx, s[e]);
                }
            }
            // lazy rescale: keep the old max unless the new one exceeds it by
            // more than 8 in log2 units (P stays <= 256, exact either way)
            const float m_new = fmaxf(m_run, mx);
            const bool need = (m_new - m_run) * sl2 > 8.f || m_run == -INFINITY;
            if (__any_sync(0xffffffffu, need && m_new != -INFINITY)) {
                const float corr = (m_run == -INFINITY) ? 0.f : ex2((m_run - m_new) * sl2);
                if (j > 0) {
                    if (!(ok = mbar_wait(bar(B_O(q)), (uint32_t)(j - 1) & 1u, abort, P.err))) break;
                    tc_fence_after();
#pragma unroll 1
                    for (int cc = 0; cc < D / 32; ++cc) {
                        uint32_t orr[32];
                        tmem_ld32(O_COL(q) + lane_off + cc * 32, orr);
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < 32; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * corr);
                        tmem_st32(O_COL(q) + lane_off + cc * 32, orr);
                    }
                }
                l_run *= corr;
                m_run = m_new;
            }
            const float mb2 = (m_run == -INFINITY) ? 0.f : m_run * sl2;
            float sum = 0.f;
            uint32_t pk[BN / 2];
#pragma unroll
            for (int e = 0; e < BN / 2; ++e) {
                float p0 = ex2(fmaf(s[2 * e], sl2, -mb2));
                float p1 = ex2(fmaf(s[2 * e + 1], sl2, -mb2));
                sum += p0 + p1;
                pk[e] = pack_bf16(p0, p1);
            }
            l_run += sum;
#pragma unroll
            for (int cc = 0; cc < BN / 64; ++cc) tmem_st32(S_COL(q) + lane_off + cc * 32, pk + cc * 32);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(bar(B_P(q)));
        }
        // ---- epilogue: O / l -> bf16 rows of the augmented layout ----
        if (ok && T > 0) ok = mbar_wait(bar(B_O(q)), (uint32_t)(T - 1) & 1u, abort, P.err);
        tc_fence_after();
        if (ok) {
            const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
            const int64_t row = (int64_t)(goff + c) * (P.k + 1) + r_slot;
            const int head = hkv * P.G + g;
            uint4 *dst = reinterpret_cast<uint4 *>(P.o + (row * P.Hq + head) * D);
#pragma unroll 1
            for (int cc = 0; cc < D / 32; ++cc) {
                uint32_t orr[32];
                tmem_ld32(O_COL(q) + lane_off + cc * 32, orr);
                tmem_wait_ld();
                if (valid) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        uint4 v;
                        v.x = pack_bf16(__uint_as_float(orr[8 * e + 0]) * inv, __uint_as_float(orr[8 * e + 1]) * inv);
                        v.y = pack_bf16(__uint_as_float(orr[8 * e + 2]) * inv, __uint_as_float(orr[8 * e + 3]) * inv);
                        v.z = pack_bf16(__uint_as_float(orr[8 * e + 4]) * inv, __uint_as_float(orr[8 * e + 5]) * inv);
                        v.w = pack_bf16(__uint_as_float(orr[8 * e + 6]) * inv, __uint_as_float(orr[8 * e + 7]) * inv);
                        dst[cc * 4 + e] = v;
                    }
                }
            }
            if (valid && P.lse) P.lse[row * P.Hq + head] = m_run * P.scale + logf(l_run);
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
// Summary rows: s_j over the k text rows of its chunk and itself, which are
// exactly the k+1 contiguous rows of chunk j in the augmented layout.  One
// warp per (chunk, kv head); CUDA cores (k+1 keys per row).
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

template <int D>
__global__ void __launch_bounds__(256) summary_rows_kernel(SumArgs a)
{
    constexpr int EPL = D / 32;  // elements per lane
    if (*a.err != 0) return;
    const int64_t task = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (task >= a.chunks * a.Hkv) return;
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
    for (int g = 0; g < a.G; ++g) {
        const int head = h * a.G + g;
        float qv[EPL];
        const __nv_bfloat16 *qp = a.q + (srow * a.Hq + head) * D + lane * EPL;
#pragma unroll
        for (int e = 0; e < EPL; ++e) qv[e] = __bfloat162float(qp[e]);
        float mx = -INFINITY;
        float sc[65];
        for (int t = 0; t <= a.k && t < 65; ++t) {
            const __nv_bfloat16 *kp = a.kk + ((row0 + t) * a.Hkv + h) * D + lane * EPL;
            float s = 0.f;
#pragma unroll
            for (int e = 0; e < EPL; ++e) s = fmaf(qv[e], __bfloat162float(kp[e]), s);
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
            sc[t] = s;
            mx = fmaxf(mx, s);
        }
        float l = 0.f, acc[EPL];
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[e] = 0.f;
        for (int t = 0; t <= a.k && t < 65; ++t) {
            float p = ex2((sc[t] - mx) * a.scale_log2);
            l += p;
            const __nv_bfloat16 *vp = a.v + ((row0 + t) * a.Hkv + h) * D + lane * EPL;
#pragma unroll
            for (int e = 0; e < EPL; ++e) acc[e] = fmaf(p, __bfloat162float(vp[e]), acc[e]);
        }
        __nv_bfloat16 *op = a.o + (srow * a.Hq + head) * D + lane * EPL;
#pragma unroll
        for (int e = 0; e < EPL; ++e) op[e] = __float2bfloat16_rn(acc[e] / l);
        if (a.lse && lane == 0) a.lse[srow * a.Hq + head] = mx * a.scale + logf(l);
    }
}

}  // namespace pf

// ---------------------------------------------------------------------------
// Host side
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
static bool make_map(CUtensorMap *m, const void *base, int d, int H, int k, int64_t chunks, int bh, int bs, int bc)
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

int prefill_unit_chunks(const ksa_params *p)
{
    int G = p->num_q_heads / p->num_kv_heads;
    int Tc = pf::BM / (G * p->k);
    return Tc * pf::NQ;
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
    P.Tc = pf::BM / (G * k);
    P.Tk = pf::BN / k;
    if (P.Tc < 1 || P.Tk < 1) return KSA_ERR_UNSUPPORTED;
    P.batch = batch;
    P.unit_chunks = P.Tc * pf::NQ;
    P.aug_rows = aug_rows;
    float scale = p->scale > 0.f ? p->scale : 1.0f / sqrtf((float)D);
    P.scale = scale;
    P.scale_log2 = scale * 1.4426950408889634f;
    P.cu = cu; P.pl = pl; P.err = err;
    P.o = (__nv_bfloat16 *)oa;
    P.lse = lse;
    bool ok = make_map(&P.tm_q, qa, D, Hq, k, chunks, G, k, P.Tc) &&
              make_map(&P.tm_ksum, ka, D, Hkv, k, chunks, 1, 1, pf::BN) &&
              make_map(&P.tm_kwin, ka, D, Hkv, k, chunks, 1, k, P.Tk) &&
              make_map(&P.tm_vsum, va, D, Hkv, k, chunks, 1, 1, pf::BN) &&
              make_map(&P.tm_vwin, va, D, Hkv, k, chunks, 1, k, P.Tk);
    if (!ok) return KSA_ERR_CUDA;
    // units: an upper bound from host totals; surplus CTAs exit at once
    int64_t units = total_text / ((int64_t)k * P.unit_chunks) + 2LL * batch + 1;
    int64_t grid = units * Hkv;
    if (grid > INT32_MAX) return KSA_ERR_UNSUPPORTED;
    static bool attr_set[2] = {false, false};
    if (!attr_set[D == 128]) {
        if (cudaFuncSetAttribute(pf::prefill_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc) !=
            cudaSuccess)
            return KSA_ERR_CUDA;
        attr_set[D == 128] = true;
    }
    pf::prefill_kernel<D><<<(unsigned)grid, pf::kThreads, L::kAlloc, st>>>(P);
    if (cudaGetLastError() != cudaSuccess) return KSA_ERR_CUDA;

    pf::SumArgs s;
    s.k = k; s.G = G; s.Hq = Hq; s.Hkv = Hkv; s.batch = batch; s.chunks = chunks;
    s.scale = scale; s.scale_log2 = P.scale_log2;
    s.cu = cu; s.pl = pl; s.err = err;
    s.q = (const __nv_bfloat16 *)qa; s.kk = (const __nv_bfloat16 *)ka; s.v = (const __nv_bfloat16 *)va;
    s.o = (__nv_bfloat16 *)oa; s.lse = lse;
    int64_t tasks = chunks * Hkv;
    if (tasks > 0) {
        pf::summary_rows_kernel<D><<<(unsigned)((tasks + 7) / 8), 256, 0, st>>>(s);
        if (cudaGetLastError() != cudaSuccess) return KSA_ERR_CUDA;
    }
    return KSA_OK;
}

int launch_prefill(const ksa_params *p, int batch, const int32_t *cu, int64_t total_text, int64_t aug_rows,
                   const void *qa, const void *ka, const void *va, void *oa, float *lse, const Plan &pl,
                   int32_t *err, cudaStream_t st)
{
    if (aug_rows == 0) return KSA_OK;
    if (p->k > 64) return KSA_ERR_UNSUPPORTED;  // summary-row kernel keeps <= 65 scores
    if (p->head_dim == 128)
        return launch_prefill_t<128>(p, batch, cu, total_text, aug_rows, qa, ka, va, oa, lse, pl, err, st);
    if (p->head_dim == 64)
        return launch_prefill_t<64>(p, batch, cu, total_text, aug_rows, qa, ka, va, oa, lse, pl, err, st);
    return KSA_ERR_UNSUPPORTED;
}

}  // namespace ksa

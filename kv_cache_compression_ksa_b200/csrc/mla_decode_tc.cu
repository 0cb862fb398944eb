// mla_decode_tc.cu -- the KSA decode over an MLA latent cache on tcgen05,
// for groups of 128 query heads.
//
// Kwai Summary Attention Technical Report, section 3.2, Eq. (6) and Table 1:
// a KSA layer over MLA caches, per kept slot, the d_c = 512 latent and the
// d_r = 64 RoPE key.  In the absorbed form every head scores the same rows,
// s_hj = scale (q_h . row_j) over the 576 dims, and its output is
// sum_j p_hj c_j over the 512 latent dims.  128 heads make one M = 128 tile:
// per block of 64 slots, S = Q K^T (K = 576) and O += P V (V = the block's
// latent dims).
//
// O alone (128 x 512 fp32) would fill the 512 TMEM columns of an SM, so a
// share of a sequence's slice runs on a cluster of two CTAs that split each
// row's dims: rank 0 takes latent dims 0..255 and the RoPE dims, rank 1
// latent dims 256..511.  TMEM per CTA: its half of O (256 columns), two S
// buffers (64 each) and its latent half of Q (bf16, 128 columns), which
// leaves shared memory room for three K/V stages.  Per block, each CTA
// computes its partial scores S_r = Q_r K_r^T of all 128 heads.  The
// softmax of half the heads belongs to each CTA (the owner: rank 0 owns TMEM
// lanes 32 q + 0..15 of every lane quarter q, rank 1 lanes 32 q + 16..31):
//   * each CTA sends its partial scores of the other's rows (64 x 64 fp32)
//     to the owner through distributed shared memory;
//   * the owner adds them to its own, runs the online softmax of its rows
//     (16-lane TMEM accesses: a thread holds two rows of 16 slots, a row's
//     four threads reduce by shuffles), writes P (bf16) over S in its TMEM
//     and sends P and the rows' rescale factors back by bulk copy;
//   * each CTA writes the received P into its TMEM, rescales its O rows of
//     the other's heads when asked, and accumulates its half of O = P V, a
//     128 x 256 x 64 product with P read from TMEM.
// Per block and direction that is 16 KB of scores and 8 KB of P instead of
// the 32 KB of a full exchange; distributed shared memory moves about 20
// bytes per clock per direction on this part.
//
// Roles (512 threads): warp 0 issues the TMA loads, warp 1 the MMAs; warps
// 4..7 own (lane quarter w % 4), 8..11 send the other rows' partial scores,
// 12..15 store the other rows' P.  Owned rows in every quarter spread the
// softmax over the four SM sub-partitions.  The online softmax works in log2
// units with a lazy rescale: O rows and row sums are rescaled only when a
// block's maximum passes the one in use by more than 8 (so p <= 2^8), once
// the previous PV product has completed.  The exchanges need no
// acknowledgement: an exchange buffer is refilled two blocks later, and the
// sender's next use of it depends, through the S buffer's reuse, on the PV
// product that follows the receiver's read.
//
// Every wait is bounded; a timeout records KSA_ERR_TIMEOUT in the sequence's
// state word.  Both CTAs always meet at a final cluster barrier: a CTA must
// not exit while its peer may still write its shared memory.
#include <cuda.h>
#include <math.h>

#include "ksa_internal.cuh"
#include "mla_common.cuh"
#include "tc_sm100.cuh"

namespace ksa {
namespace mla {
namespace tcm {

using namespace ksa::tc;

constexpr int HT = 128;                 // heads per tile (MMA M)
constexpr int HO = HT / 2;              // heads whose softmax a CTA owns
constexpr int NB = kTcBlock;            // slots per block (QK N, PV K)
constexpr int ST = 3;                   // K/V stages
constexpr int kChunk = NB * 128;        // one 64-dim chunk of a block: 8 KB
constexpr int kQChunk = HT * 128;       // the RoPE chunk of Q (rank 0): 16 KB
constexpr int kStage = 5 * kChunk;      // rank 0: latent 0..255 + RoPE; rank 1: latent 256..511
// shared memory
constexpr int kQR = 0;                               // Q's RoPE dims, 128-byte swizzled (rank 0)
constexpr int kKV = kQR + kQChunk;                   // [ST] stages
// Exchange buffers, in the register order of the 16-lane TMEM accesses
// (thread t of the warp of lane quarter q holds rows t/4 and t/4 + 8 of the
// quarter's 16 rows of one CTA, columns 8r + 2(t % 4) + {0, 1}), so that the
// receiving warp of the same quarter reads what the sending warp held.
constexpr int kRecvS = kKV + ST * kStage;            // [2][4 q][8][32 t] float4: the other CTA's partial scores
constexpr int kRecvSBuf = 4 * 8 * 32 * 16;
constexpr int kRecvP = kRecvS + 2 * kRecvSBuf;       // [2][4 q][4][32 t] uint4: P of the other's heads
constexpr int kRecvPBuf = 4 * 4 * 32 * 16;
constexpr int kAlpha = kRecvP + 2 * kRecvPBuf;       // [2][4 q][16] float: their rescale factors
constexpr int kPStage = kAlpha + 2 * HO * 4;         // [2][4 q][4][32 t] uint4: this CTA's P, sent by bulk copy
constexpr int kAStage = kPStage + 2 * kRecvPBuf;     // [2][4 q][16] float: its rescale factors
constexpr int kPBytes = 4 * 32 * 16, kABytes = 16 * 4;   // one quarter's P and factors
constexpr int kBar = kAStage + 2 * HO * 4;
// kv_full[ST], kv_empty[ST], s_full[2], p_full[2], o_done[2], recv_s[2], recv_p[2], drain
constexpr int B_KV_FULL = 0, B_KV_EMPTY = B_KV_FULL + ST, B_S_FULL = B_KV_EMPTY + ST, B_P_FULL = B_S_FULL + 2,
              B_O_DONE = B_P_FULL + 2, B_RECV_S = B_O_DONE + 2, B_RECV_P = B_RECV_S + 2, B_DRAIN = B_RECV_P + 2,
              kNumBars = B_DRAIN + 1;
constexpr int kMisc = kBar + kNumBars * 8;   // tmem slot, abort flag, go flag, pad, cos[32], sin[32]
constexpr int kBytes = kMisc + 16 + 2 * (DR / 2) * 4;
constexpr int kThreads = 512;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kOCol = 0, kSCol = 256, kQCol = 384;   // O half; S buffer b at 256 + 64 b; Q latent half
constexpr float kRescale = 8.f;
static_assert(kBytes <= 227 * 1024, "shared memory budget");
static_assert(kSCol + 2 * NB <= kQCol && kQCol + 128 <= kTmemCols, "TMEM budget");
static_assert(kKV % 1024 == 0 && kStage % 1024 == 0, "128-byte swizzle atoms");

struct TcArgs {
    CUtensorMap tm_lat;   // latent rows [B][S][576], box 64 dims x NB slots
    Args a;
};

__device__ __forceinline__ uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// this CTA's shared address -> the same offset in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t peer_addr(uint32_t local, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
    return r;
}

__device__ __forceinline__ void st_cluster_v4(uint32_t addr, uint32_t x, uint32_t y, uint32_t z, uint32_t w)
{
    asm volatile("st.shared::cluster.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(x), "r"(y), "r"(z), "r"(w)
                 : "memory");
}

__device__ __forceinline__ void st_cluster_u32(uint32_t addr, uint32_t x)
{
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(x) : "memory");
}

// arrive on an mbarrier of the peer, ordering this thread's earlier
// accesses before it at cluster scope
__device__ __forceinline__ void arrive_cluster(uint32_t addr)
{
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(addr) : "memory");
}

// bounded wait on a local mbarrier whose arrivals come from the peer
__device__ __forceinline__ bool wait_cluster(uint32_t bar, uint32_t parity, volatile int *abort, int32_t *err)
{
    for (uint32_t it = 0; it < kSpinLimit; ++it) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(bar), "r"(parity)
            : "memory");
        if (ok) return true;
        if (*abort) return false;
    }
    *abort = 1;
    set_error(err, KSA_ERR_TIMEOUT);
    return false;
}

// bulk copy of `bytes` from this CTA's shared memory to the peer's, completing
// on the peer's mbarrier
__device__ __forceinline__ void bulk_copy_to_peer(uint32_t dst, uint32_t src, uint32_t bytes, uint32_t bar)
{
    asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "r"(src), "r"(bytes), "r"(bar)
                 : "memory");
}
// Bulk async-groups batch only the copies that complete through a bulk group
// (shared -> global); a copy into the peer's shared memory completes on the
// peer's mbarrier instead, so these group waits do not order its reads of the
// source.  What frees a staging buffer here is the exchange's causal chain
// (see the owner's P staging).
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }

// the same, sleeping in try_wait between checks (for warps whose wake-up is
// not on the critical path, so that they leave issue slots to the others)
__device__ __forceinline__ bool wait_cluster_sleep(uint32_t bar, uint32_t parity, volatile int *abort, int32_t *err)
{
    for (uint32_t it = 0; it < kWaitLimit; ++it) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(bar), "r"(parity), "r"(kSuspendNs)
            : "memory");
        if (ok) return true;
        if (*abort) return false;
    }
    *abort = 1;
    set_error(err, KSA_ERR_TIMEOUT);
    return false;
}

__device__ __forceinline__ void cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// 16-lane TMEM accesses (thread t: lanes base + t/4 and base + t/4 + 8):
// 16x256b.x8: register 4r + 2h + w <-> lane t/4 + 8h, column 8r + 2(t % 4) + w
__device__ __forceinline__ void tmem_ld16x256_x8(uint32_t taddr, uint32_t *r)
{
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x8.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_st16x256_x8(uint32_t taddr, const uint32_t *r)
{
    asm volatile(
        "tcgen05.st.sync.aligned.16x256b.x8.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
        "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
        "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

// 16x128b.x8: register 2r + h <-> lane t/4 + 8h, column 4r + t % 4
__device__ __forceinline__ void tmem_st16x128_x8(uint32_t taddr, const uint32_t *r)
{
    asm volatile(
        "tcgen05.st.sync.aligned.16x128b.x8.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    mla_decode_tc_kernel(const __grid_constant__ TcArgs ta)
{
    const Args &a = ta.a;
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t sbase = smem_u32(smem);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + kMisc);
    volatile int *abort = reinterpret_cast<volatile int *>(smem + kMisc + 4);
    volatile int *go = reinterpret_cast<volatile int *>(smem + kMisc + 8);
    float *s_cos = reinterpret_cast<float *>(smem + kMisc + 16), *s_sin = s_cos + DR / 2;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank(), peer = rank ^ 1u;
    const int split = (int)(blockIdx.x >> 1), hg = (int)blockIdx.y, b = (int)blockIdx.z;
    const int h0 = hg * HT;
    int32_t *err = a.state + 4 * (int64_t)b + 3;
    const int kind = a.kind[b];
    const int64_t n = a.state[4 * (int64_t)b], m = a.state[4 * (int64_t)b + 1];
    int64_t lo = 0, hi = 0;
    const bool slice_ok = decode_slice(kind, n, m, a.k, a.w, &lo, &hi) && hi <= a.S;
    auto bar = [&](int i) { return sbase + kBar + 8u * (uint32_t)i; };

    if (threadIdx.x == 0) {
        for (int s = 0; s < ST; ++s) {
            mbar_init(bar(B_KV_FULL + s), 1);
            mbar_init(bar(B_KV_EMPTY + s), 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(bar(B_S_FULL + s), 1);
            mbar_init(bar(B_P_FULL + s), 256);   // this CTA's owner and receiver warps
            mbar_init(bar(B_O_DONE + s), 1);
            mbar_init(bar(B_RECV_S + s), 128);   // the other CTA's sender warps
            // the other CTA's P: one local arrival with the expected bytes, armed
            // a phase ahead, and the bulk copies' completions
            mbar_init(bar(B_RECV_P + s), 1);
            mbar_expect_tx(bar(B_RECV_P + s), 4 * (kPBytes + kABytes));
        }
        mbar_init(bar(B_DRAIN), 1);
        *abort = 0;
        // the pair's decision, taken once by rank 0: the error word may change
        // while the launch runs, and both CTAs must take the same path
        int g = 0;
        if (rank == 0 && kind != KSA_SKIP && *err == 0) {
            if (!slice_ok) {
                if (split == 0 && hg == 0) set_error(err, KSA_ERR_STATE);
            } else if (sbase & 1023u) {
                set_error(err, KSA_ERR_UNSUPPORTED);
            } else {
                g = 1;
            }
        }
        *go = g;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    cluster_sync();   // both CTAs running, barriers initialised
    if (rank == 0 && threadIdx.x == 0) st_cluster_u32(peer_addr(smem_u32(smem + kMisc + 8), 1), (uint32_t)*go);
    cluster_sync();
    if (!*go) return;   // the same decision in both CTAs, before either touches the other

    const int64_t s0 = lo + (int64_t)split * a.per, s1 = min(hi, s0 + a.per);
    const int nblk = s1 > s0 ? (int)((s1 - s0 + NB - 1) / NB) : 0;
    const int nch = rank == 0 ? 5 : 4;
    constexpr int kWarpTMA = 0, kWarpMMA = 1;
    if (warp == kWarpMMA) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    constexpr int V8 = DL / 8;   // 16-byte units per row
    const uint4 *qg = reinterpret_cast<const uint4 *>(a.q + ((int64_t)b * a.H + h0) * DL);
    // ---- Q's RoPE dims (rank 0), rotated at the query's position n - 1, into
    // the 128-byte swizzled layout of the MMA descriptors ----
    if (rank == 0) {
        for (int r = threadIdx.x; r < DR / 2; r += kThreads) {
            float c = 1.f, s = 0.f;
            if (a.rotate) rope_cos_sin((double)(n - 1), r, DR, a.log2_theta, &c, &s);
            s_cos[r] = c;
            s_sin[r] = s;
        }
        __syncthreads();
        for (int e = threadIdx.x; e < HT * 4; e += kThreads) {
            const int h = e >> 2, c = e & 3;
            uint4 lo4 = qg[(int64_t)h * V8 + DC / 8 + c], hi4 = qg[(int64_t)h * V8 + DC / 8 + c + DR / 16];
            rope_rot8(lo4, hi4, s_cos + 8 * c, s_sin + 8 * c);
            *reinterpret_cast<uint4 *>(smem + kQR + h * 128 + ((c ^ (h & 7)) << 4)) = lo4;
            *reinterpret_cast<uint4 *>(smem + kQR + h * 128 + (((c + DR / 16) ^ (h & 7)) << 4)) = hi4;
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // generic writes -> tensor core reads
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // ---- this rank's latent half of Q into TMEM (the A operand of QK): warps
    // 4..7, thread = head row = TMEM lane, bf16 pairs in k order ----
    if (warp >= 4 && warp < 8) {
        const int row = (warp - 4) * 32 + lane;
        const uint32_t lane_off = (uint32_t)((warp - 4) * 32) << 16;
        const uint4 *src = qg + (int64_t)row * V8 + rank * 32;
#pragma unroll 1
        for (int g = 0; g < 4; ++g) {
            uint32_t v[32];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const uint4 x = src[8 * g + u];
                v[4 * u] = x.x; v[4 * u + 1] = x.y; v[4 * u + 2] = x.z; v[4 * u + 3] = x.w;
            }
            tmem_st32(tmem + lane_off + kQCol + 32 * g, v);
        }
        tmem_wait_st();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    if (warp == kWarpTMA) {
        if (lane == 0) {
            bool ok = true;
            int issued[ST] = {};
            for (int j = 0; j < nblk; ++j) {
                const int stg = j % ST;
                if (j >= ST && !(ok = mbar_wait_sleep(bar(B_KV_EMPTY + stg), (uint32_t)((j / ST) - 1) & 1u, abort, err)))
                    break;
                mbar_expect_tx(bar(B_KV_FULL + stg), (uint32_t)(nch * kChunk));
                const int slot = (int)(s0 + (int64_t)j * NB);
                for (int ci = 0; ci < nch; ++ci) {
                    const int col = ci < 4 ? 256 * (int)rank + 64 * ci : DC;   // rank 0's fifth chunk: the RoPE dims
                    tma_load_4d(sbase + kKV + stg * kStage + ci * kChunk, &ta.tm_lat, bar(B_KV_FULL + stg), col, slot,
                                0, b);
                }
                issued[stg]++;
            }
            // every load issued lands before the CTA exits
            if (!ok)
                for (int stg = 0; stg < ST; ++stg)
                    if (issued[stg]) {
                        const uint32_t ph = (uint32_t)(issued[stg] - 1) & 1u;
                        for (uint32_t it = 0; it < kSpinLimit && !mbar_try_wait(bar(B_KV_FULL + stg), ph); ++it) {}
                    }
        }
    } else if (warp == kWarpMMA) {
        if (lane == 0) {
            const uint32_t id_qk = idesc_f16(HT, NB, false);
            const uint32_t id_pv = idesc_f16(HT, 256, true);
            // descriptors built once; an operand's offset adds to the start
            // address field (addresses stay below 256 KB: no carry)
            const uint64_t dk0 = sdesc(sbase + kKV, 16, 1024);       // K chunks, K-major
            const uint64_t dv0 = sdesc(sbase + kKV, kChunk, 1024);   // V: the latent chunks, MN-major
            const uint64_t dq0 = sdesc(sbase + kQR, 16, 1024);       // Q's RoPE chunk
            bool ok = true;
            for (int j = 0; j <= nblk && ok; ++j) {
                if (j < nblk) {
                    // S(j) = Q K(j)^T over this rank's dims, into S buffer j % 2
                    const int stg = j % ST, sb = j & 1;
                    ok = mbar_wait(bar(B_KV_FULL + stg), (uint32_t)(j / ST) & 1u, abort, err);
                    // the buffer's last reader, PV(j - 2), has completed
                    if (ok && j >= 2) ok = mbar_wait(bar(B_O_DONE + sb), (uint32_t)((j - 2) >> 1) & 1u, abort, err);
                    if (!ok) break;
                    tc_fence_after();
                    const uint64_t dk = dk0 + (uint64_t)((stg * kStage) >> 4);
                    const uint32_t t_s = tmem + kSCol + sb * NB;
                    // latent dims: Q from TMEM (16 bf16 = 8 columns per K step)
#pragma unroll
                    for (int ci = 0; ci < 4; ++ci)
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_ts(t_s, tmem + kQCol + ci * 32 + kk * 8, dk + (uint64_t)((ci * kChunk + kk * 32) >> 4),
                                   id_qk, (ci | kk) ? 1u : 0u);
                    // RoPE dims (rank 0): Q from shared memory
                    if (rank == 0)
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            mma_ss(t_s, dq0 + (uint64_t)((kk * 32) >> 4), dk + (uint64_t)((4 * kChunk + kk * 32) >> 4),
                                   id_qk, 1u);
                    tc_commit(bar(B_S_FULL + sb));
                }
                if (j >= 1) {
                    // O += P(i) V(i): P from TMEM, V = the stage's four latent
                    // chunks (N = 256 dims, MN-major)
                    const int i = j - 1, stg = i % ST, sb = i & 1;
                    if (!(ok = mbar_wait(bar(B_P_FULL + sb), (uint32_t)(i >> 1) & 1u, abort, err))) break;
                    tc_fence_after();
                    const uint64_t dv = dv0 + (uint64_t)((stg * kStage) >> 4);
#pragma unroll
                    for (int kk = 0; kk < NB / 16; ++kk)
                        mma_ts(tmem + kOCol, tmem + kSCol + sb * NB + kk * 8, dv + (uint64_t)((kk * 2048) >> 4), id_pv,
                               (i > 0 || kk > 0) ? 1u : 0u);
                    tc_commit(bar(B_O_DONE + sb));
                    tc_commit(bar(B_KV_EMPTY + stg));
                }
            }
            // every MMA issued has completed before the teardown
            tc_commit(bar(B_DRAIN));
            for (uint32_t it = 0; it < kSpinLimit && !mbar_try_wait(bar(B_DRAIN), 0); ++it) {}
        }
    } else if (warp >= 4) {
        // Rows: rank 0 owns the softmax of lanes 32 q + 0..15 of every lane
        // quarter q, rank 1 of lanes 32 q + 16..31, so that the owners' work
        // spreads over the four SM sub-partitions (warp w runs on w % 4 and
        // reaches the TMEM lanes of quarter w % 4).  Warps 4..7 own, 8..11
        // send the other rows' partial scores, 12..15 store their P.
        const int q = warp & 3, role = (warp - 4) >> 2;   // 0 owner, 1 sender, 2 receiver
        const int lb = 32 * q + 16 * (role == 0 ? (int)rank : (int)peer);   // the warp's 16 lanes
        const uint32_t taddr = (uint32_t)lb << 16;
        const int r0 = lb + (lane >> 2);                  // rows r0 and r0 + 8 of the 128
        constexpr uint32_t FULL = 0xffffffffu;
        auto o_store = [&](void) {
            // this CTA's 256 columns of rows r0, r0 + 8 (unnormalised)
            const int64_t prow = ((int64_t)split * a.batch + b) * a.H + h0 + r0;
#pragma unroll 1
            for (int g = 0; g < 4; ++g) {
                uint32_t o[32];
                tmem_ld16x256_x8(tmem + taddr + kOCol + 64 * g, o);
                tmem_wait_ld();
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    float *dst = a.part_o + (prow + 8 * h) * DC + 256 * rank + 64 * g + 2 * (lane & 3);
#pragma unroll
                    for (int r = 0; r < 8; ++r)
                        *reinterpret_cast<float2 *>(dst + 8 * r) =
                            make_float2(__uint_as_float(o[4 * r + 2 * h]), __uint_as_float(o[4 * r + 2 * h + 1]));
                }
            }
        };
        auto o_rescale = [&](const float *al) {
            // O rows r0, r0 + 8 times al[0], al[1], once PV(j - 1) has completed
#pragma unroll 1
            for (int g = 0; g < 4; ++g) {
                uint32_t o[32];
                tmem_ld16x256_x8(tmem + taddr + kOCol + 64 * g, o);
                tmem_wait_ld();
#pragma unroll
                for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * al[(e >> 1) & 1]);
                tmem_st16x256_x8(tmem + taddr + kOCol + 64 * g, o);
            }
        };
        if (role == 0) {
            // ================= owner: the softmax of rows r0, r0 + 8 =================
            const uint32_t peer_recv_p = peer_addr(sbase + kRecvP, peer);
            const uint32_t peer_alpha = peer_addr(sbase + kAlpha, peer);
            const uint32_t peer_bar_p = peer_addr(bar(B_RECV_P), peer);
            int copies = 0;   // bulk-copy groups this lane committed
            float m_used[2] = {-INFINITY, -INFINITY}, lsum[2] = {0.f, 0.f};
            bool ok = true;
            for (int j = 0; j < nblk; ++j) {
                const int sb = j & 1;
                ok = __all_sync(FULL, mbar_wait(bar(B_S_FULL + sb), (uint32_t)(j >> 1) & 1u, abort, err));
                if (!ok) break;
                tc_fence_after();
                uint32_t sp[32];
                tmem_ld16x256_x8(tmem + taddr + kSCol + sb * NB, sp);
                tmem_wait_ld();
                ok = __all_sync(FULL, wait_cluster(bar(B_RECV_S + sb), (uint32_t)(j >> 1) & 1u, abort, err));
                if (!ok) break;
                // S = own + other partial scores, in log2 units; slots past the
                // share's end masked
                const int cnt = (int)min((int64_t)NB, s1 - (s0 + (int64_t)j * NB));
                float x[32];
                float mx[2] = {-INFINITY, -INFINITY};
                {
                    const float4 *src = reinterpret_cast<const float4 *>(smem + kRecvS + sb * kRecvSBuf) + q * 256 + lane;
#pragma unroll
                    for (int r = 0; r < 8; ++r) {
                        const float4 v = src[32 * r];
                        const float pv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const int c = 8 * r + 2 * (lane & 3) + (e & 1);
                            const float t = (__uint_as_float(sp[4 * r + e]) + pv[e]) * a.scale_log2;
                            x[4 * r + e] = c < cnt ? t : -INFINITY;
                            mx[e >> 1] = fmaxf(mx[e >> 1], x[4 * r + e]);
                        }
                    }
                }
                float alpha[2];
                bool resc_any = false;
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    mx[h] = fmaxf(mx[h], __shfl_xor_sync(FULL, mx[h], 1));
                    mx[h] = fmaxf(mx[h], __shfl_xor_sync(FULL, mx[h], 2));
                    const bool resc = mx[h] > m_used[h] + kRescale;
                    alpha[h] = 1.f;
                    if (resc) {
                        alpha[h] = ex2(m_used[h] - mx[h]);   // 0 at the first block
                        lsum[h] *= alpha[h];
                        m_used[h] = mx[h];
                    }
                    resc_any = resc_any || resc;
                }
                if (j > 0 && __any_sync(FULL, resc_any)) {
                    ok = __all_sync(FULL, mbar_wait(bar(B_O_DONE + (sb ^ 1)), (uint32_t)((j - 1) >> 1) & 1u, abort, err));
                    if (!ok) break;
                    tc_fence_after();
                    o_rescale(alpha);
                }
                uint32_t pk[16];
#pragma unroll
                for (int r = 0; r < 8; ++r)
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const float p0 = ex2(x[4 * r + 2 * h] - m_used[h]), p1 = ex2(x[4 * r + 2 * h + 1] - m_used[h]);
                        lsum[h] += p0 + p1;
                        pk[2 * r + h] = pack_bf16(p0, p1);
                    }
                tmem_st16x128_x8(tmem + taddr + kSCol + sb * NB, pk);   // P over S's first 32 columns
                // P and the rows' factors to the other CTA, which holds the other
                // half of O: staged here, then one bulk copy per quarter, so that
                // this warp does not wait on the distributed shared memory
                {
                    // staging buffer sb was last read by the copy of P(j - 2), which
                    // landed in the other CTA before its PV(j - 2), and so before its
                    // QK(j) and the scores of block j that this warp has received
                    if (lane == 0 && copies >= 2) bulk_wait_read_1();
                    __syncwarp();
                    uint4 *ps = reinterpret_cast<uint4 *>(smem + kPStage + sb * kRecvPBuf + q * kPBytes) + lane;
#pragma unroll
                    for (int u = 0; u < 4; ++u) ps[32 * u] = make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
                    float *as = reinterpret_cast<float *>(smem + kAStage + sb * HO * 4 + q * kABytes);
                    if ((lane & 3) == 0) {
                        as[lane >> 2] = alpha[0];
                        as[(lane >> 2) + 8] = alpha[1];
                    }
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // for the bulk copy's reads
                    __syncwarp();
                    if (lane == 0) {
                        const uint32_t pb = peer_bar_p + 8u * (uint32_t)sb;
                        bulk_copy_to_peer(peer_recv_p + (uint32_t)(sb * kRecvPBuf + q * kPBytes),
                                          sbase + (uint32_t)(kPStage + sb * kRecvPBuf + q * kPBytes), kPBytes, pb);
                        bulk_copy_to_peer(peer_alpha + (uint32_t)(sb * HO * 4 + q * kABytes),
                                          sbase + (uint32_t)(kAStage + sb * HO * 4 + q * kABytes), kABytes, pb);
                        bulk_commit();
                        ++copies;
                    }
                }
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar(B_P_FULL + sb));
            }
            // the last copies land before the other CTA leaves its receive loop,
            // and so before the final cluster barrier
            if (lane == 0) bulk_wait_read_0();
            __syncwarp();
            // ---- epilogue: this CTA's half of the rows' O and the rows' (max, sum) ----
            if (ok && nblk > 0)
                ok = __all_sync(FULL, mbar_wait(bar(B_O_DONE + ((nblk - 1) & 1)), (uint32_t)((nblk - 1) >> 1) & 1u,
                                                abort, err));
            if (ok) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    lsum[h] += __shfl_xor_sync(FULL, lsum[h], 1);
                    lsum[h] += __shfl_xor_sync(FULL, lsum[h], 2);
                }
                if (nblk > 0) {
                    tc_fence_after();
                    o_store();
                }
                if ((lane & 3) == 0) {
                    const int64_t prow = ((int64_t)split * a.batch + b) * a.H + h0 + r0;
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        a.part_ml[(prow + 8 * h) * 2] = m_used[h];
                        a.part_ml[(prow + 8 * h) * 2 + 1] = lsum[h];
                    }
                }
            }
        } else if (role == 1) {
            // ================= sender: the other CTA's rows' partial scores =================
            const uint32_t peer_recv_s = peer_addr(sbase + kRecvS, peer);
            const uint32_t peer_bar_s = peer_addr(bar(B_RECV_S), peer);
            for (int j = 0; j < nblk; ++j) {
                const int sb = j & 1;
                if (!__all_sync(FULL, mbar_wait(bar(B_S_FULL + sb), (uint32_t)(j >> 1) & 1u, abort, err))) break;
                tc_fence_after();
                uint32_t sp[32];
                tmem_ld16x256_x8(tmem + taddr + kSCol + sb * NB, sp);
                tmem_wait_ld();
                tc_fence_before();   // these reads precede the P that the owner's reply brings
                const uint32_t dst = peer_recv_s + (uint32_t)(sb * kRecvSBuf + (q * 256 + lane) * 16);
#pragma unroll
                for (int r = 0; r < 8; ++r)
                    st_cluster_v4(dst + (uint32_t)(r * 32 * 16), sp[4 * r], sp[4 * r + 1], sp[4 * r + 2], sp[4 * r + 3]);
                arrive_cluster(peer_bar_s + 8u * (uint32_t)sb);
            }
        } else {
            // ================= receiver: the owner's P for the other CTA's rows =================
            bool ok = true;
            for (int j = 0; j < nblk; ++j) {
                const int sb = j & 1;
                ok = __all_sync(FULL, wait_cluster_sleep(bar(B_RECV_P + sb), (uint32_t)(j >> 1) & 1u, abort, err));
                if (!ok) break;
                // arm buffer sb's next phase (block j + 2), whose copies start only
                // after this block's P has been read (its product precedes them)
                if (q == 0 && lane == 0 && j + 2 < nblk) mbar_expect_tx(bar(B_RECV_P + sb), 4 * (kPBytes + kABytes));
                uint32_t pk[16];
                {
                    const uint4 *src = reinterpret_cast<const uint4 *>(smem + kRecvP + sb * kRecvPBuf) + q * 128 + lane;
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const uint4 v = src[32 * u];
                        pk[4 * u] = v.x; pk[4 * u + 1] = v.y; pk[4 * u + 2] = v.z; pk[4 * u + 3] = v.w;
                    }
                }
                const float *al_in = reinterpret_cast<const float *>(smem + kAlpha) + sb * HO + q * 16 + (lane >> 2);
                const float alpha[2] = {al_in[0], al_in[8]};
                tc_fence_after();
                if (j > 0 && __any_sync(FULL, alpha[0] != 1.f || alpha[1] != 1.f)) {
                    ok = __all_sync(FULL, mbar_wait(bar(B_O_DONE + (sb ^ 1)), (uint32_t)((j - 1) >> 1) & 1u, abort, err));
                    if (!ok) break;
                    tc_fence_after();
                    o_rescale(alpha);
                }
                tmem_st16x128_x8(tmem + taddr + kSCol + sb * NB, pk);
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(bar(B_P_FULL + sb));
            }
            // ---- epilogue: this CTA's half of the other CTA's rows' O ----
            if (ok && nblk > 0)
                ok = __all_sync(FULL, mbar_wait(bar(B_O_DONE + ((nblk - 1) & 1)), (uint32_t)((nblk - 1) >> 1) & 1u,
                                                abort, err));
            if (ok && nblk > 0) {
                tc_fence_after();
                o_store();
            }
        }
    }

    // ---- teardown ----
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == kWarpMMA)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                     : "memory");
    cluster_sync();   // the other CTA is past every access to this CTA's shared memory
}

}  // namespace tcm

int launch_mla_tc(const Args &a, cudaStream_t st)
{
    using namespace tcm;
    if (a.H % HT != 0 || a.S > 0x7fffffffLL || a.per % NB != 0) return KSA_ERR_UNSUPPORTED;
    TcArgs ta;
    ta.a = a;
    // [B][S][1][576] viewed as make_map's [chunks][k+1][H][d] with k = 0
    if (!make_map(&ta.tm_lat, a.lat, DL, (int)a.S, 0, a.batch, NB, 1, 1)) return KSA_ERR_CUDA;
    static bool attr = false;
    if (!attr) {
        if (cudaFuncSetAttribute(mla_decode_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kBytes) !=
            cudaSuccess)
            return KSA_ERR_CUDA;
        attr = true;
    }
    dim3 grid((unsigned)(2 * a.splits), (unsigned)(a.H / HT), (unsigned)a.batch);
    mla_decode_tc_kernel<<<grid, kThreads, kBytes, st>>>(ta);
    return cudaGetLastError() == cudaSuccess ? KSA_OK : KSA_ERR_CUDA;
}

}  // namespace mla
}  // namespace ksa

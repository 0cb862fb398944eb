// mla_decode.cu -- KSA decode over a latent (MLA) cache.
//
// Kwai Summary Attention Technical Report, section 3.2, Eq. (6): KSA and MLA
// compress different axes, so a KSA layer can cache, per kept token, MLA's
// d_c latent (the non-RoPE keys and values, rebuilt per head by the up
// projections) plus its d_r decoupled RoPE key (section 3.1), i.e.
// n/k (d_c + d_r) values per layer for the summaries.  The cache keeps the
// slot map of section 2.3.1 (Figure 4) with one latent row per slot.
//
// Decoding uses MLA's absorbed form: with the key up-projection folded into
// the query, a head's score against slot j is scale (q_c . c_j + q_r . r_j)
// and its output is sum_j p_j c_j, a d_c-dim latent that the caller's value
// up-projection maps to the head's output.  Every head reads the same rows:
// multi-query attention over rows of d_c + d_r.
//
//   mla_append_kernel   one token per sequence: Figure 4 (b)-(e), rotating
//                       the d_r part at the token's position
//   mla_decode_kernel   one (sequence, group of 16 MT heads, slice share):
//                       32-slot blocks staged by cp.async, QK^T and PV on the
//                       warp-level tensor-core MMA, online softmax
//   mla_combine_kernel  merge the shares of a sequence's slice
#include <math.h>

#include "ksa_internal.cuh"
#include "mla_common.cuh"
#include "warp_mma.cuh"

namespace ksa {
namespace mla {

constexpr int KB = 32;                           // slots per block
constexpr int PITCH = DL + 8;                    // smem row pitch (elements)
constexpr int PPITCH = KB + 8;                   // P tile row pitch

// ---------------------------------------------------------------------------
struct AppendArgs {
    int k, w;
    int64_t S, cap;
    int rotate;
    double log2_theta;
    const int8_t *kind;
    int32_t *state;
    const uint4 *x;     // [B, DL] new latent rows, d_r part not rotated
    uint4 *lat;         // [B, S, DL]
};

constexpr int kAppendThreads = 128;

__global__ void __launch_bounds__(kAppendThreads) mla_append_kernel(AppendArgs a)
{
    __shared__ int s_act;
    __shared__ int64_t s_n, s_m;
    __shared__ float s_cos[DR / 2], s_sin[DR / 2];
    const int b = blockIdx.x, t = threadIdx.x;
    int32_t *st = a.state + 4 * (int64_t)b;
    if (t == 0) {
        const int kind = a.kind[b];
        const int64_t n = st[0], m = st[1], f = n - m * a.k;
        const bool reachable = n >= 0 && m >= 0;   // slots below are only in range for these
        int act = 0;
        if (kind == KSA_TEXT) {
            if (reachable && f >= 0 && f < a.k) act = 1; else st[3] = KSA_ERR_STATE;
        } else if (kind == KSA_SUMMARY) {
            if (!reachable || f != a.k) st[3] = KSA_ERR_STATE;
            else if (m >= a.cap) st[3] = KSA_ERR_CAPACITY;
            else act = 2;
        } else if (kind != KSA_SKIP) {
            st[3] = KSA_ERR_INVALID;
        }
        s_act = act; s_n = n; s_m = m;
    }
    __syncthreads();
    const int act = s_act;
    if (!act) return;
    const int64_t n = s_n, m = s_m, f = n - m * a.k;
    const int64_t pos = act == 1 ? n : n - 1;   // a summary takes its chunk's last position
    for (int r = t; r < DR / 2; r += kAppendThreads) {
        float c = 1.f, s = 0.f;
        if (a.rotate) rope_cos_sin((double)pos, r, DR, a.log2_theta, &c, &s);
        s_cos[r] = c; s_sin[r] = s;
    }
    __syncthreads();
    constexpr int V8 = DL / 8;                 // uint4 per row
    const int64_t dst0 = act == 1 ? a.k - f : 0;
    const int64_t dst1 = act == 2 ? 1 + a.k + (int64_t)a.w * a.k + m : -1;
    uint4 *base = a.lat + (int64_t)b * a.S * V8;
    const uint4 *src = a.x + (int64_t)b * V8;
    // latent part: copied
    for (int c = t; c < DC / 8; c += kAppendThreads) {
        base[dst0 * V8 + c] = src[c];
        if (dst1 >= 0) base[dst1 * V8 + c] = src[c];
    }
    // RoPE part: 4 items of 8 pairs (r, r + d_r/2)
    for (int c = t; c < DR / 16; c += kAppendThreads) {
        uint4 lo = src[DC / 8 + c], hi = src[DC / 8 + c + DR / 16];
        rope_rot8(lo, hi, s_cos + 8 * c, s_sin + 8 * c);
        base[dst0 * V8 + DC / 8 + c] = lo;
        base[dst0 * V8 + DC / 8 + c + DR / 16] = hi;
        if (dst1 >= 0) {
            base[dst1 * V8 + DC / 8 + c] = lo;
            base[dst1 * V8 + DC / 8 + c + DR / 16] = hi;
        }
    }
    // (4d): the finished chunk (slots 1..k) over ring block m mod w
    if (act == 2 && a.w > 0) {
        const int64_t ring = 1 + a.k + (m % a.w) * a.k;
        for (int64_t e = t; e < (int64_t)a.k * V8; e += kAppendThreads) base[ring * V8 + e] = base[V8 + e];
    }
    __syncthreads();
    if (t == 0) {
        if (act == 1) st[0] = (int32_t)(n + 1);
        else st[1] = (int32_t)(m + 1);
    }
}

// ---------------------------------------------------------------------------
// Decode.  Warps 0 .. 2 MT - 1.  QK^T: warp w takes m-tile w % MT (16 heads)
// against slots 16 (w / MT) .. +15 of the block.  PV: warp w owns latent
// dims [w DS, (w+1) DS), DS = DC / (2 MT), for all 16 MT heads (128 fp32
// accumulators per thread whatever MT).  P and the per-head rescale factors
// pass through shared memory.
// ---------------------------------------------------------------------------
template <int MT>
struct Smem {
    static constexpr int HEADS = 16 * MT;
    static constexpr size_t q = 0;
    static constexpr size_t kv = q + (size_t)HEADS * PITCH * 2;            // two blocks of KB rows
    static constexpr size_t p = kv + 2ull * KB * PITCH * 2;
    static constexpr size_t red = p + (size_t)HEADS * PPITCH * 2;         // [2][HEADS] row maxima
    static constexpr size_t alpha = red + 2ull * HEADS * 4;
    static constexpr size_t lsum = alpha + (size_t)HEADS * 4;              // [2][HEADS]
    static constexpr size_t bytes = lsum + 2ull * HEADS * 4;
};

template <int MT>
__global__ void __launch_bounds__(64 * MT) mla_decode_kernel(Args a)
{
    constexpr int NW = 2 * MT, NTH = 32 * NW, HEADS = 16 * MT;
    constexpr int DS = DC / NW, NTW = DS / 8;
    using L = Smem<MT>;
    using Row = __nv_bfloat16[PITCH];
    using PRow = __nv_bfloat16[PPITCH];
    extern __shared__ __align__(16) uint8_t mla_smem[];
    Row *sQ = reinterpret_cast<Row *>(mla_smem + L::q);
    Row *sK = reinterpret_cast<Row *>(mla_smem + L::kv);
    PRow *sP = reinterpret_cast<PRow *>(mla_smem + L::p);
    float *sRed = reinterpret_cast<float *>(mla_smem + L::red);
    float *sAlpha = reinterpret_cast<float *>(mla_smem + L::alpha);
    float *sL = reinterpret_cast<float *>(mla_smem + L::lsum);
    __shared__ float s_cos[DR / 2], s_sin[DR / 2];

    const int split = blockIdx.x, hg = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gr = lane >> 2, tt = lane & 3;
    const int h0 = hg * HEADS;
    const int64_t pidx = ((int64_t)split * a.batch + b) * a.H + h0;   // first partial row of this CTA
    const int kind = a.kind[b];
    const int64_t n = a.state[4 * (int64_t)b], m = a.state[4 * (int64_t)b + 1];
    int64_t lo = 0, hi = 0;
    if (kind == KSA_SKIP || a.state[4 * (int64_t)b + 3] != 0) return;
    if (!decode_slice(kind, n, m, a.k, a.w, &lo, &hi) || hi > a.S) {
        if (split == 0 && hg == 0 && threadIdx.x == 0) a.state[4 * (int64_t)b + 3] = KSA_ERR_STATE;
        return;
    }
    const int64_t s0 = lo + (int64_t)split * a.per, s1 = min(hi, s0 + a.per);
    const int nblk = s1 > s0 ? (int)((s1 - s0 + KB - 1) / KB) : 0;

    // Q of this CTA's heads; the d_r part rotated at the query's position
    const int64_t pos = n - 1;
    for (int r = threadIdx.x; r < DR / 2; r += NTH) {
        float c = 1.f, s = 0.f;
        if (a.rotate) rope_cos_sin((double)pos, r, DR, a.log2_theta, &c, &s);
        s_cos[r] = c; s_sin[r] = s;
    }
    __syncthreads();
    {
        constexpr int V8 = DL / 8;
        const uint4 *qg = reinterpret_cast<const uint4 *>(a.q + ((int64_t)b * a.H + h0) * DL);
        for (int e = threadIdx.x; e < HEADS * (DC / 8); e += NTH) {
            const int h = e / (DC / 8), c = e % (DC / 8);
            *reinterpret_cast<uint4 *>(&sQ[h][8 * c]) = h0 + h < a.H ? qg[(int64_t)h * V8 + c] : make_uint4(0, 0, 0, 0);
        }
        for (int e = threadIdx.x; e < HEADS * (DR / 16); e += NTH) {
            const int h = e / (DR / 16), c = e % (DR / 16);
            uint4 lo4 = make_uint4(0, 0, 0, 0), hi4 = lo4;
            if (h0 + h < a.H) {
                lo4 = qg[(int64_t)h * V8 + DC / 8 + c];
                hi4 = qg[(int64_t)h * V8 + DC / 8 + c + DR / 16];
                rope_rot8(lo4, hi4, s_cos + 8 * c, s_sin + 8 * c);
            }
            *reinterpret_cast<uint4 *>(&sQ[h][DC + 8 * c]) = lo4;
            *reinterpret_cast<uint4 *>(&sQ[h][DC + DR / 2 + 8 * c]) = hi4;
        }
    }
    const __nv_bfloat16 *rows = a.lat + (int64_t)b * a.S * DL;
    auto prefetch = [&](int kb) {   // block kb -> buffer kb % 2 (one commit group)
        Row *dst = sK + (kb & 1) * KB;
        const int64_t r0 = s0 + (int64_t)kb * KB;
        const int cnt = (int)min((int64_t)KB, s1 - r0);
        for (int e = threadIdx.x; e < KB * (DL / 8); e += NTH) {
            const int r = e / (DL / 8), c = e % (DL / 8);
            if (r < cnt) wm::cp_async16(&dst[r][8 * c], rows + (r0 + r) * DL + 8 * c);
            else *reinterpret_cast<uint4 *>(&dst[r][8 * c]) = make_uint4(0, 0, 0, 0);
        }
        wm::cp_commit();
    };
    if (nblk > 0) prefetch(0);

    const int mt = warp % MT, kh = warp / MT;          // QK role
    const int rA = 16 * mt + gr, rB = rA + 8;          // the two heads of this lane's S rows
    float mrow[2] = {-INFINITY, -INFINITY}, lpart[2] = {0.f, 0.f};
    float acc[MT][NTW][4];
#pragma unroll
    for (int i = 0; i < MT; ++i)
#pragma unroll
        for (int j = 0; j < NTW; ++j) acc[i][j][0] = acc[i][j][1] = acc[i][j][2] = acc[i][j][3] = 0.f;

    for (int kb = 0; kb < nblk; ++kb) {
        const int cnt = (int)min((int64_t)KB, s1 - (s0 + (int64_t)kb * KB));
        if (kb + 1 < nblk) {
            prefetch(kb + 1);
            wm::cp_wait<1>();
        } else {
            wm::cp_wait<0>();
        }
        __syncthreads();   // block kb (and, the first time, Q) visible to all
        const Row *K = sK + (kb & 1) * KB;
        // S = Q K^T: 16 heads x 16 slots
        float s[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll 4
        for (int c = 0; c < DL / 16; ++c) {
            uint32_t qa[4], kk[4];
            wm::frag_a<PITCH - 8>(qa, sQ, 16 * mt, 16 * c);
            wm::frag_b_nk<PITCH - 8>(kk, K, 16 * kh, 16 * c);
            wm::mma16816(s[0], qa[0], qa[1], qa[2], qa[3], kk[0], kk[1]);
            wm::mma16816(s[1], qa[0], qa[1], qa[2], qa[3], kk[2], kk[3]);
        }
        // scale to log2 units, mask the block's tail, row maxima over both halves
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int z = 0; z < 4; ++z) {
                const int col = 16 * kh + 8 * j + 2 * tt + (z & 1);
                const float v = col < cnt ? s[j][z] * a.scale_log2 : -INFINITY;
                s[j][z] = v;
                mx[z >> 1] = fmaxf(mx[z >> 1], v);
            }
#pragma unroll
        for (int x = 0; x < 2; ++x) {
            mx[x] = fmaxf(mx[x], __shfl_xor_sync(0xffffffffu, mx[x], 1));
            mx[x] = fmaxf(mx[x], __shfl_xor_sync(0xffffffffu, mx[x], 2));
        }
        if (tt == 0) { sRed[kh * HEADS + rA] = mx[0]; sRed[kh * HEADS + rB] = mx[1]; }
        __syncthreads();
        float base[2];
#pragma unroll
        for (int x = 0; x < 2; ++x) {
            const int r = x ? rB : rA;
            const float mn = fmaxf(mrow[x], fmaxf(sRed[r], sRed[HEADS + r]));
            base[x] = mn == -INFINITY ? 0.f : mn;
            const float al = wm::ex2(mrow[x] - base[x]);
            mrow[x] = mn;
            lpart[x] *= al;
            if (kh == 0 && tt == 0) sAlpha[r] = al;
        }
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            float e[4];
#pragma unroll
            for (int z = 0; z < 4; ++z) {
                e[z] = wm::ex2(s[j][z] - base[z >> 1]);
                lpart[z >> 1] += e[z];
            }
            const int col = 16 * kh + 8 * j + 2 * tt;
            *reinterpret_cast<uint32_t *>(&sP[rA][col]) = wm::pack2(e[0], e[1]);
            *reinterpret_cast<uint32_t *>(&sP[rB][col]) = wm::pack2(e[2], e[3]);
        }
        __syncthreads();   // P and the rescale factors of every head are in shared memory
        // O (all heads, this warp's dims) = alpha O + P V
#pragma unroll
        for (int i = 0; i < MT; ++i) {
            const float a0 = sAlpha[16 * i + gr], a1 = sAlpha[16 * i + gr + 8];
#pragma unroll
            for (int j = 0; j < NTW; ++j) {
                acc[i][j][0] *= a0; acc[i][j][1] *= a0;
                acc[i][j][2] *= a1; acc[i][j][3] *= a1;
            }
        }
#pragma unroll
        for (int kc = 0; kc < KB / 16; ++kc) {
            uint32_t pa[MT][4];
#pragma unroll
            for (int i = 0; i < MT; ++i) wm::frag_a<PPITCH - 8>(pa[i], sP, 16 * i, 16 * kc);
#pragma unroll
            for (int np = 0; np < NTW / 2; ++np) {
                uint32_t vb[4];
                wm::frag_b_kn<PITCH - 8>(vb, K, 16 * kc, warp * DS + 16 * np);
#pragma unroll
                for (int i = 0; i < MT; ++i) {
                    wm::mma16816(acc[i][2 * np], pa[i][0], pa[i][1], pa[i][2], pa[i][3], vb[0], vb[1]);
                    wm::mma16816(acc[i][2 * np + 1], pa[i][0], pa[i][1], pa[i][2], pa[i][3], vb[2], vb[3]);
                }
            }
        }
        __syncthreads();   // buffer kb % 2, P and the maxima may be reused
    }
    // partial sums of this share: l over both key halves
#pragma unroll
    for (int x = 0; x < 2; ++x) {
        float l = lpart[x];
        l += __shfl_xor_sync(0xffffffffu, l, 1);
        l += __shfl_xor_sync(0xffffffffu, l, 2);
        if (tt == 0) sL[kh * HEADS + (x ? rB : rA)] = l;
    }
    if (kh == 0 && tt == 0) {   // the running maxima (equal in both halves)
        sRed[rA] = mrow[0];
        sRed[rB] = mrow[1];
    }
    __syncthreads();
    for (int h = threadIdx.x; h < HEADS; h += NTH) {
        if (h0 + h >= a.H) continue;
        a.part_ml[(pidx + h) * 2] = sRed[h];
        a.part_ml[(pidx + h) * 2 + 1] = sL[h] + sL[HEADS + h];
    }
#pragma unroll
    for (int i = 0; i < MT; ++i)
#pragma unroll
        for (int x = 0; x < 2; ++x) {
            const int h = 16 * i + gr + 8 * x;
            if (h0 + h >= a.H) continue;
            float *dst = a.part_o + (pidx + h) * DC + warp * DS;
#pragma unroll
            for (int j = 0; j < NTW; ++j)
                *reinterpret_cast<float2 *>(dst + 8 * j + 2 * tt) = make_float2(acc[i][j][2 * x], acc[i][j][2 * x + 1]);
        }
}

// ---------------------------------------------------------------------------
// Warp-specialised form for 64-head CTAs.  Warps 0-3 (one warpgroup) each
// take 16 heads: they keep those heads' q fragments in registers for the
// whole slice, compute S = Q K^T of a 32-slot block and its softmax (a row
// never leaves its warp), and publish P and the rescale factors.  Warps 4-11
// each own 64 latent dims of O for all 64 heads and load the latent blocks.
// Blocks and P are double-buffered; named barriers hand them over:
//   1 + b  block in buffer b landed        (PV warps arrive, QK warps sync)
//   3 + b  P and factors of buffer b ready (QK warps arrive, PV warps sync)
//   5 + b  P buffer b read                 (PV warps arrive, QK warps sync)
// Each barrier alternates strictly between the two groups, and both groups
// walk the same blocks, so every phase gets its 384 threads.  Registers move
// from the PV warps (168 -> 160) to the QK warps (168 -> 184, room for their
// 144 q-fragment registers): 4 x 32 x 184 + 8 x 32 x 160 = 384 x 168, exactly
// the launch allocation, so the increase always finds its registers.
// ---------------------------------------------------------------------------
constexpr int WS_THREADS = 384;

struct WsSmem {
    static constexpr int HEADS = 64;
    static constexpr size_t q = 0;
    static constexpr size_t kv = q + (size_t)HEADS * PITCH * 2;
    static constexpr size_t p = kv + 2ull * KB * PITCH * 2;            // two P buffers
    static constexpr size_t alpha = p + 2ull * HEADS * PPITCH * 2;     // two factor buffers
    static constexpr size_t bytes = alpha + 2ull * HEADS * 4;
};

__device__ __forceinline__ void nb_sync(int id) { asm volatile("bar.sync %0, 384;" ::"r"(id) : "memory"); }
__device__ __forceinline__ void nb_arrive(int id) { asm volatile("bar.arrive %0, 384;" ::"r"(id) : "memory"); }

__global__ void __launch_bounds__(WS_THREADS, 1) mla_decode_ws_kernel(Args a)
{
    constexpr int HEADS = 64, NC = DL / 16;
    using L = WsSmem;
    using Row = __nv_bfloat16[PITCH];
    using PRow = __nv_bfloat16[PPITCH];
    extern __shared__ __align__(16) uint8_t mla_smem[];
    Row *sQ = reinterpret_cast<Row *>(mla_smem + L::q);
    Row *sK = reinterpret_cast<Row *>(mla_smem + L::kv);
    PRow *sP = reinterpret_cast<PRow *>(mla_smem + L::p);
    float *sA = reinterpret_cast<float *>(mla_smem + L::alpha);
    __shared__ float s_cos[DR / 2], s_sin[DR / 2];

    const int split = blockIdx.x, hg = blockIdx.y, b = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gr = lane >> 2, tt = lane & 3;
    const int h0 = hg * HEADS;
    const int64_t pidx = ((int64_t)split * a.batch + b) * a.H + h0;
    const int kind = a.kind[b];
    const int64_t n = a.state[4 * (int64_t)b], m = a.state[4 * (int64_t)b + 1];
    int64_t lo = 0, hi = 0;
    if (kind == KSA_SKIP || a.state[4 * (int64_t)b + 3] != 0) return;
    if (!decode_slice(kind, n, m, a.k, a.w, &lo, &hi) || hi > a.S) {
        if (split == 0 && hg == 0 && threadIdx.x == 0) a.state[4 * (int64_t)b + 3] = KSA_ERR_STATE;
        return;
    }
    const int64_t s0 = lo + (int64_t)split * a.per, s1 = min(hi, s0 + a.per);
    const int nblk = s1 > s0 ? (int)((s1 - s0 + KB - 1) / KB) : 0;

    // q of this CTA's heads in shared memory, the d_r part rotated at n - 1
    const int64_t pos = n - 1;
    for (int r = threadIdx.x; r < DR / 2; r += WS_THREADS) {
        float c = 1.f, s = 0.f;
        if (a.rotate) rope_cos_sin((double)pos, r, DR, a.log2_theta, &c, &s);
        s_cos[r] = c; s_sin[r] = s;
    }
    __syncthreads();
    {
        constexpr int V8 = DL / 8;
        const uint4 *qg = reinterpret_cast<const uint4 *>(a.q + ((int64_t)b * a.H + h0) * DL);
        for (int e = threadIdx.x; e < HEADS * (DC / 8); e += WS_THREADS) {
            const int h = e / (DC / 8), c = e % (DC / 8);
            *reinterpret_cast<uint4 *>(&sQ[h][8 * c]) = h0 + h < a.H ? qg[(int64_t)h * V8 + c] : make_uint4(0, 0, 0, 0);
        }
        for (int e = threadIdx.x; e < HEADS * (DR / 16); e += WS_THREADS) {
            const int h = e / (DR / 16), c = e % (DR / 16);
            uint4 lo4 = make_uint4(0, 0, 0, 0), hi4 = lo4;
            if (h0 + h < a.H) {
                lo4 = qg[(int64_t)h * V8 + DC / 8 + c];
                hi4 = qg[(int64_t)h * V8 + DC / 8 + c + DR / 16];
                rope_rot8(lo4, hi4, s_cos + 8 * c, s_sin + 8 * c);
            }
            *reinterpret_cast<uint4 *>(&sQ[h][DC + 8 * c]) = lo4;
            *reinterpret_cast<uint4 *>(&sQ[h][DC + DR / 2 + 8 * c]) = hi4;
        }
    }
    __syncthreads();

    if (warp < 4) {
        // ================= QK and softmax: heads 16 warp .. 16 warp + 15 =================
        asm volatile("setmaxnreg.inc.sync.aligned.u32 184;" ::: "memory");
        uint32_t qf[NC][4];
#pragma unroll
        for (int c = 0; c < NC; ++c) wm::frag_a<PITCH - 8>(qf[c], sQ, 16 * warp, 16 * c);
        const int rA = 16 * warp + gr, rB = rA + 8;
        float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
        for (int kb = 0; kb < nblk; ++kb) {
            const int bb = kb & 1;
            const int cnt = (int)min((int64_t)KB, s1 - (s0 + (int64_t)kb * KB));
            nb_sync(1 + bb);   // block kb landed
            const Row *K = sK + bb * KB;
            float sc[4][4];
#pragma unroll
            for (int i = 0; i < 4; ++i) sc[i][0] = sc[i][1] = sc[i][2] = sc[i][3] = 0.f;
#pragma unroll
            for (int c = 0; c < NC; ++c) {
                uint32_t k0[4], k1[4];
                wm::frag_b_nk<PITCH - 8>(k0, K, 0, 16 * c);
                wm::frag_b_nk<PITCH - 8>(k1, K, 16, 16 * c);
                wm::mma16816(sc[0], qf[c][0], qf[c][1], qf[c][2], qf[c][3], k0[0], k0[1]);
                wm::mma16816(sc[1], qf[c][0], qf[c][1], qf[c][2], qf[c][3], k0[2], k0[3]);
                wm::mma16816(sc[2], qf[c][0], qf[c][1], qf[c][2], qf[c][3], k1[0], k1[1]);
                wm::mma16816(sc[3], qf[c][0], qf[c][1], qf[c][2], qf[c][3], k1[2], k1[3]);
            }
            // scale, mask the tail, softmax over the block's 32 slots
            float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int z = 0; z < 4; ++z) {
                    const int col = 8 * nt + 2 * tt + (z & 1);
                    const float v = col < cnt ? sc[nt][z] * a.scale_log2 : -INFINITY;
                    sc[nt][z] = v;
                    mx[z >> 1] = fmaxf(mx[z >> 1], v);
                }
            float base[2], alpha[2];
#pragma unroll
            for (int x = 0; x < 2; ++x) {
                mx[x] = fmaxf(mx[x], __shfl_xor_sync(0xffffffffu, mx[x], 1));
                mx[x] = fmaxf(mx[x], __shfl_xor_sync(0xffffffffu, mx[x], 2));
                const float mn = fmaxf(mrow[x], mx[x]);
                base[x] = mn == -INFINITY ? 0.f : mn;
                alpha[x] = wm::ex2(mrow[x] - base[x]);
                mrow[x] = mn;
                lrow[x] *= alpha[x];
            }
            uint32_t pw[4][2];
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                float e[4];
#pragma unroll
                for (int z = 0; z < 4; ++z) {
                    e[z] = wm::ex2(sc[nt][z] - base[z >> 1]);
                    lrow[z >> 1] += e[z];
                }
                pw[nt][0] = wm::pack2(e[0], e[1]);
                pw[nt][1] = wm::pack2(e[2], e[3]);
            }
            if (kb >= 2) nb_sync(5 + bb);   // the PV warps have read P buffer bb (block kb - 2)
            PRow *Pb = sP + bb * HEADS;
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                *reinterpret_cast<uint32_t *>(&Pb[rA][8 * nt + 2 * tt]) = pw[nt][0];
                *reinterpret_cast<uint32_t *>(&Pb[rB][8 * nt + 2 * tt]) = pw[nt][1];
            }
            if (tt == 0) { sA[bb * HEADS + rA] = alpha[0]; sA[bb * HEADS + rB] = alpha[1]; }
            nb_arrive(3 + bb);   // P and factors of block kb ready
        }
        // share statistics: max (log2 units) and sum of this share
#pragma unroll
        for (int x = 0; x < 2; ++x) {
            float l = lrow[x];
            l += __shfl_xor_sync(0xffffffffu, l, 1);
            l += __shfl_xor_sync(0xffffffffu, l, 2);
            const int h = x ? rB : rA;
            if (tt == 0 && h0 + h < a.H) {
                a.part_ml[(pidx + h) * 2] = mrow[x];
                a.part_ml[(pidx + h) * 2 + 1] = l;
            }
        }
    } else {
        // ================= PV: latent dims 64 pw .. 64 pw + 63 of all 64 heads =================
        asm volatile("setmaxnreg.dec.sync.aligned.u32 160;" ::: "memory");
        constexpr int NTW = 8, NPT = 256;   // n-tiles of this warp's dims; threads of the group
        const int pw = warp - 4, tid = threadIdx.x - 128;
        const __nv_bfloat16 *rows = a.lat + (int64_t)b * a.S * DL;
        auto issue = [&](int kb) {   // block kb -> buffer kb % 2 (one commit group)
            Row *dst = sK + (kb & 1) * KB;
            const int64_t r0 = s0 + (int64_t)kb * KB;
            const int cnt = (int)min((int64_t)KB, s1 - r0);
            for (int e = tid; e < KB * (DL / 8); e += NPT) {
                const int r = e / (DL / 8), c = e % (DL / 8);
                if (r < cnt) wm::cp_async16(&dst[r][8 * c], rows + (r0 + r) * DL + 8 * c);
                else *reinterpret_cast<uint4 *>(&dst[r][8 * c]) = make_uint4(0, 0, 0, 0);
            }
            wm::cp_commit();
        };
        float acc[4][NTW][4];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < NTW; ++j) acc[i][j][0] = acc[i][j][1] = acc[i][j][2] = acc[i][j][3] = 0.f;
        if (nblk > 0) {
            issue(0);
            if (nblk > 1) { issue(1); wm::cp_wait<1>(); } else { wm::cp_wait<0>(); }
            nb_arrive(1 + 0);   // block 0 landed
        }
        for (int kb = 0; kb < nblk; ++kb) {
            const int bb = kb & 1;
            if (kb + 1 < nblk) {   // block kb + 1 (issued one block ago) landed
                wm::cp_wait<0>();
                nb_arrive(1 + (bb ^ 1));
            }
            nb_sync(3 + bb);   // P of block kb ready
            const Row *V = sK + bb * KB;
            const PRow *Pb = sP + bb * HEADS;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float a0 = sA[bb * HEADS + 16 * i + gr], a1 = sA[bb * HEADS + 16 * i + gr + 8];
#pragma unroll
                for (int j = 0; j < NTW; ++j) {
                    acc[i][j][0] *= a0; acc[i][j][1] *= a0;
                    acc[i][j][2] *= a1; acc[i][j][3] *= a1;
                }
            }
#pragma unroll
            for (int kc = 0; kc < KB / 16; ++kc) {
                uint32_t pa[4][4];
#pragma unroll
                for (int i = 0; i < 4; ++i) wm::frag_a<PPITCH - 8>(pa[i], Pb, 16 * i, 16 * kc);
#pragma unroll
                for (int np = 0; np < NTW / 2; ++np) {
                    uint32_t vb[4];
                    wm::frag_b_kn<PITCH - 8>(vb, V, 16 * kc, 64 * pw + 16 * np);
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        wm::mma16816(acc[i][2 * np], pa[i][0], pa[i][1], pa[i][2], pa[i][3], vb[0], vb[1]);
                        wm::mma16816(acc[i][2 * np + 1], pa[i][0], pa[i][1], pa[i][2], pa[i][3], vb[2], vb[3]);
                    }
                }
            }
            if (kb + 2 < nblk) {
                nb_arrive(5 + bb);   // P buffer bb read; block kb's buffer is free
                issue(kb + 2);
            }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int x = 0; x < 2; ++x) {
                const int h = 16 * i + gr + 8 * x;
                if (h0 + h >= a.H) continue;
                float *dst = a.part_o + (pidx + h) * DC + 64 * pw;
#pragma unroll
                for (int j = 0; j < NTW; ++j)
                    *reinterpret_cast<float2 *>(dst + 8 * j + 2 * tt) = make_float2(acc[i][j][2 * x], acc[i][j][2 * x + 1]);
            }
    }
}

// One CTA per (head, sequence): merge the shares.
constexpr int kCombineThreads = 128;

__global__ void __launch_bounds__(kCombineThreads) mla_combine_kernel(Args a)
{
    const int h = blockIdx.x, b = blockIdx.y;
    const int kind = a.kind[b];
    if (kind == KSA_SKIP || a.state[4 * (int64_t)b + 3] != 0) return;
    float M = -INFINITY;
    for (int s = 0; s < a.splits; ++s) M = fmaxf(M, a.part_ml[(((int64_t)s * a.batch + b) * a.H + h) * 2]);
    const float base = M == -INFINITY ? 0.f : M;
    float Lsum = 0.f;
    float o[DC / kCombineThreads];
#pragma unroll
    for (int i = 0; i < DC / kCombineThreads; ++i) o[i] = 0.f;
    for (int s = 0; s < a.splits; ++s) {
        const int64_t r = ((int64_t)s * a.batch + b) * a.H + h;
        const float ms = a.part_ml[r * 2], ls = a.part_ml[r * 2 + 1];
        if (ls <= 0.f) continue;   // an empty share
        const float f = wm::ex2(ms - base);
        Lsum += ls * f;
        const float4 *src = reinterpret_cast<const float4 *>(a.part_o + r * DC) + threadIdx.x;
        const float4 v = *src;
        o[0] += f * v.x; o[1] += f * v.y; o[2] += f * v.z; o[3] += f * v.w;
    }
    const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
    __nv_bfloat16 *dst = a.o + ((int64_t)b * a.H + h) * DC + 4 * threadIdx.x;
    *reinterpret_cast<uint32_t *>(dst) = wm::pack2(o[0] * inv, o[1] * inv);
    *reinterpret_cast<uint32_t *>(dst + 2) = wm::pack2(o[2] * inv, o[3] * inv);
    if (a.lse && threadIdx.x == 0) a.lse[(int64_t)b * a.H + h] = (M + log2f(Lsum)) * 0.69314718055994531f;
}
static_assert(DC == 4 * kCombineThreads, "combine: four latent dims per thread");

// ---------------------------------------------------------------------------
struct Plan {
    int mt, groups, splits;
    int64_t per;
    bool tc;   // the tensor-core kernel (head groups of 128)
};

// Shares for the tensor-core kernel: each share (one CTA pair) reads its
// rows once and writes 2 x 128 x 512 fp32 partials per 128 heads that the
// combine reads back.  Taken: the share count (at least 4 blocks a share)
// that minimises waves x (share bytes + partial bytes), pairs per wave =
// SMs / 2; ties to the fewer shares.
static Plan plan_tc(const ksa_mla_params *p, int batch, int64_t lmax)
{
    Plan P;
    P.mt = 0;
    P.tc = true;
    P.groups = p->num_heads / 128;
    const int64_t ctas = (int64_t)batch * P.groups, pairs = sm_count() / 2 > 0 ? sm_count() / 2 : 1;
    const int64_t most = lmax / (4 * kTcBlock) > 1 ? lmax / (4 * kTcBlock) : 1;
    const double part = 2.0 * 128 * DC * 4;
    int64_t best_sp = 1;
    double best = -1.0;
    for (int64_t sp = 1; sp <= most && sp <= 1024 && ctas > 0; ++sp) {
        int64_t per = (lmax + sp - 1) / sp;
        per = (per + kTcBlock - 1) / kTcBlock * kTcBlock;
        const int64_t real = (lmax + per - 1) / per;
        const int64_t waves = (ctas * real + pairs - 1) / pairs;
        const double cost = (double)waves * ((double)per * DL * 2 + part);
        if (best < 0 || cost < best * (1 - 1e-9)) { best = cost; best_sp = real; }
    }
    int64_t per = (lmax + best_sp - 1) / best_sp;
    per = (per + kTcBlock - 1) / kTcBlock * kTcBlock;
    if (per < kTcBlock) per = kTcBlock;
    P.per = per;
    P.splits = (int)((lmax + per - 1) / per);
    if (P.splits < 1) P.splits = 1;
    return P;
}

static Plan plan(const ksa_mla_params *p, int batch, int64_t max_text)
{
    Plan P;
    {
        const int64_t mmax = max_text / p->k;
        const int64_t lmax = (int64_t)p->k + 1 + (int64_t)p->w * p->k + (mmax > p->w ? mmax - p->w : 0);
        if (p->num_heads % 128 == 0) return plan_tc(p, batch, lmax);
    }
    P.tc = false;
    P.mt = p->num_heads >= 64 ? 4 : p->num_heads >= 32 ? 2 : 1;
    P.groups = (p->num_heads + 16 * P.mt - 1) / (16 * P.mt);
    const int64_t mmax = max_text / p->k;
    const int64_t lmax = (int64_t)p->k + 1 + (int64_t)p->w * p->k + (mmax > p->w ? mmax - p->w : 0);
    // Enough shares for two CTAs per SM, each at least 4 blocks.  Then, while
    // a share keeps at least 1024 slots (so the partial outputs stay small
    // against the slice), a larger count up to twice the four-wave count may
    // be taken if its last wave is fuller (one CTA per SM fits).
    const int64_t ctas = (int64_t)batch * P.groups, sms = sm_count();
    const int64_t want = ctas > 0 ? (2 * sms + ctas - 1) / ctas : 1;
    const int64_t most = (lmax + 4 * KB - 1) / (4 * KB);
    int64_t sp = want < most ? want : most;
    if (sp < 1) sp = 1;
    const int64_t four = ctas > 0 ? (4 * sms + ctas - 1) / ctas : 1;
    int64_t top = (four > sp ? four : sp) * 2;
    if (top > lmax / 1024) top = lmax / 1024;
    double best = -1.0;
    for (int64_t c = sp, c0 = sp; c <= (top > c0 ? top : c0) && ctas > 0; ++c) {
        const double waves = (double)(ctas * c) / (double)sms;
        const double eff = waves / (double)((ctas * c + sms - 1) / sms);
        if (eff > best + 1e-9) { best = eff; sp = c; }
    }
    if (sp > 1024) sp = 1024;
    int64_t per = (lmax + sp - 1) / sp;
    per = (per + KB - 1) / KB * KB;
    P.splits = (int)((lmax + per - 1) / per);
    P.per = per;
    return P;
}

}  // namespace mla

size_t mla_decode_workspace_bytes(const ksa_mla_params *p, int batch, int64_t max_text)
{
    const mla::Plan P = mla::plan(p, batch, max_text);
    const size_t rows = (size_t)P.splits * batch * p->num_heads;
    return align_up(rows * mla::DC * 4) + align_up(rows * 2 * 4);
}

int launch_mla_append(const ksa_mla_params *p, const ksa_mla_cache *c, const int8_t *kind, const void *x,
                      cudaStream_t st)
{
    if (c->batch == 0) return KSA_OK;
    mla::AppendArgs a;
    a.k = p->k; a.w = p->w;
    a.S = 1 + (int64_t)p->k + (int64_t)p->w * p->k + c->cap_summaries;
    a.cap = c->cap_summaries;
    a.rotate = p->rope_theta > 0.0;
    a.log2_theta = a.rotate ? log2(p->rope_theta) : 0.0;
    a.kind = kind; a.state = c->state;
    a.x = (const uint4 *)x; a.lat = (uint4 *)c->latent;
    mla::mla_append_kernel<<<c->batch, mla::kAppendThreads, 0, st>>>(a);
    return cudaGetLastError() == cudaSuccess ? KSA_OK : KSA_ERR_CUDA;
}

template <int MT>
static int launch_mla_t(const mla::Args &a, int groups, cudaStream_t st)
{
    const size_t smem = mla::Smem<MT>::bytes;
    if (cudaFuncSetAttribute(mla::mla_decode_kernel<MT>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return KSA_ERR_CUDA;
    dim3 grid((unsigned)a.splits, (unsigned)groups, (unsigned)a.batch);
    mla::mla_decode_kernel<MT><<<grid, 64 * MT, smem, st>>>(a);
    return cudaGetLastError() == cudaSuccess ? KSA_OK : KSA_ERR_CUDA;
}

static int launch_mla_ws(const mla::Args &a, int groups, cudaStream_t st)
{
    const size_t smem = mla::WsSmem::bytes;
    if (cudaFuncSetAttribute(mla::mla_decode_ws_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
        cudaSuccess)
        return KSA_ERR_CUDA;
    dim3 grid((unsigned)a.splits, (unsigned)groups, (unsigned)a.batch);
    mla::mla_decode_ws_kernel<<<grid, mla::WS_THREADS, smem, st>>>(a);
    return cudaGetLastError() == cudaSuccess ? KSA_OK : KSA_ERR_CUDA;
}

int launch_mla_decode(const ksa_mla_params *p, const ksa_mla_cache *c, const int8_t *kind, const void *q, void *o,
                      float *lse, int64_t max_text, void *ws, size_t ws_bytes, cudaStream_t st)
{
    if (c->batch == 0) return KSA_OK;
    if (ws_bytes < mla_decode_workspace_bytes(p, c->batch, max_text)) return KSA_ERR_WORKSPACE;
    const mla::Plan P = mla::plan(p, c->batch, max_text);
    if (P.groups > 65535) return KSA_ERR_UNSUPPORTED;
    mla::Args a;
    a.k = p->k; a.w = p->w; a.H = p->num_heads; a.batch = c->batch; a.splits = P.splits;
    a.S = 1 + (int64_t)p->k + (int64_t)p->w * p->k + c->cap_summaries;
    a.per = P.per;
    const float scale = p->scale > 0.f ? p->scale : 1.f / sqrtf((float)(mla::DC + mla::DR));
    a.scale_log2 = scale * 1.4426950408889634f;
    a.rotate = p->rope_theta > 0.0;
    a.log2_theta = a.rotate ? log2(p->rope_theta) : 0.0;
    a.kind = kind; a.state = c->state;
    a.lat = (const __nv_bfloat16 *)c->latent;
    a.q = (const __nv_bfloat16 *)q;
    const size_t rows = (size_t)P.splits * c->batch * p->num_heads;
    a.part_o = reinterpret_cast<float *>(ws);
    a.part_ml = reinterpret_cast<float *>(static_cast<char *>(ws) + align_up(rows * mla::DC * 4));
    a.o = (__nv_bfloat16 *)o;
    a.lse = lse;
    int rc = P.tc        ? mla::launch_mla_tc(a, st)
             : P.mt == 4 ? launch_mla_ws(a, P.groups, st)
             : P.mt == 2 ? launch_mla_t<2>(a, P.groups, st)
                         : launch_mla_t<1>(a, P.groups, st);
    if (rc != KSA_OK) return rc;
    dim3 grid((unsigned)p->num_heads, (unsigned)c->batch);
    mla::mla_combine_kernel<<<grid, mla::kCombineThreads, 0, st>>>(a);
    return cudaGetLastError() == cudaSuccess ? KSA_OK : KSA_ERR_CUDA;
}

}  // namespace ksa

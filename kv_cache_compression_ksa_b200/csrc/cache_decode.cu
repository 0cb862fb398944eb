// cache_decode.cu -- the contiguous KSA decode cache: append and attention.
//
// Kwai Summary Attention Technical Report, section 2.3.1 and Figure 4:
//   (4a) the cache is one tensor per (sequence, kv head): a scratch slot, the
//        current chunk (filled right to left, right edge against the ring),
//        the ring of w sliding chunks, and the append-only summary buffer;
//   (4b) a new text token's K/V goes into the next free current-chunk slot;
//   (4c)-(4e) on chunk completion the summary K/V goes to the scratch slot,
//        the finished chunk is copied over the ring's oldest block, and the
//        summary K/V is appended to the buffer;
//   every decode read is ONE contiguous slice of the cache.
// Decode is bound by HBM bandwidth (the report: "memory-bandwidth
// bottleneck rather than compute-bound"), so the kernel streams the slice
// once with 16-byte loads and splits long slices across CTAs (split-K),
// merging the partial softmax states afterwards.
//
// Cache layout: K, V [B, Hkv, S, d] bf16, S = 1 + k + w*k + cap, so a slice
// of one (sequence, kv head) is a contiguous run of d-element rows.
#include <math.h>

#include "ksa_internal.cuh"
#include "warp_mma.cuh"

namespace ksa {

// ---------------------------------------------------------------------------
// Append
// ---------------------------------------------------------------------------
constexpr int kAppendThreads = 256;

struct AppendArgs {
    int k, w, Hkv, d;
    int64_t S, cap;
    int rotate;
    double log2_theta;
    const int8_t *kind;
    int32_t *state;
    const uint4 *k_new, *v_new;  // [B, Hkv, d]
    uint4 *K, *V;                // [B, Hkv, S, d]
};

__global__ void __launch_bounds__(kAppendThreads) cache_append_kernel(AppendArgs a)
{
    __shared__ int s_act;  // 0 skip, 1 text, 2 summary
    __shared__ int64_t s_n, s_m;
    __shared__ float s_cos[64], s_sin[64];
    const int b = blockIdx.x, t = threadIdx.x;
    int32_t *st = a.state + 4 * (int64_t)b;
    if (t == 0) {
        int kind = a.kind[b];
        int64_t n = st[0], m = st[1];
        int64_t f = n - m * a.k;
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
    const int64_t n = s_n, m = s_m;
    const int half = a.d / 2;
    // text token at position n; summary at its chunk's last text position n-1
    const int64_t pos = act == 1 ? n : n - 1;
    for (int r = t; r < half; r += kAppendThreads) {
        float c = 1.f, s = 0.f;
        if (a.rotate) rope_cos_sin((double)pos, r, a.d, a.log2_theta, &c, &s);
        s_cos[r] = c; s_sin[r] = s;
    }
    __syncthreads();
    const int vec = a.d / 8;           // uint4 per head row
    const int hv = half / 8;           // uint4 per half row
    const int64_t f = n - m * a.k;
    // destination slots of the new K/V
    int64_t dst0 = act == 1 ? a.k - f : 0;
    int64_t dst1 = act == 2 ? 1 + a.k + (int64_t)a.w * a.k + m : -1;
    // K rows: rotate 8 pairs per item
    for (int e = t; e < a.Hkv * hv; e += kAppendThreads) {
        int h = e / hv, c = e % hv;
        const uint4 *src = a.k_new + ((int64_t)b * a.Hkv + h) * vec;
        uint4 lo = src[c], hi = src[c + hv];
        __nv_bfloat162 *x = reinterpret_cast<__nv_bfloat162 *>(&lo);
        __nv_bfloat162 *y = reinterpret_cast<__nv_bfloat162 *>(&hi);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            float2 xv = __bfloat1622float2(x[q]), yv = __bfloat1622float2(y[q]);
            int r0 = 8 * c + 2 * q;
            float c0 = s_cos[r0], c1 = s_cos[r0 + 1], s0 = s_sin[r0], s1 = s_sin[r0 + 1];
            x[q] = __float22bfloat162_rn(make_float2(xv.x * c0 - yv.x * s0, xv.y * c1 - yv.y * s1));
            y[q] = __float22bfloat162_rn(make_float2(yv.x * c0 + xv.x * s0, yv.y * c1 + xv.y * s1));
        }
        uint4 *row = a.K + (((int64_t)b * a.Hkv + h) * a.S) * vec;
        row[dst0 * vec + c] = lo;
        row[dst0 * vec + c + hv] = hi;
        if (dst1 >= 0) {
            row[dst1 * vec + c] = lo;
            row[dst1 * vec + c + hv] = hi;
        }
    }
    for (int e = t; e < a.Hkv * vec; e += kAppendThreads) {
        int h = e / vec, c = e % vec;
        uint4 val = a.v_new[((int64_t)b * a.Hkv + h) * vec + c];
        uint4 *row = a.V + (((int64_t)b * a.Hkv + h) * a.S) * vec;
        row[dst0 * vec + c] = val;
        if (dst1 >= 0) row[dst1 * vec + c] = val;
    }
    // (4d): copy the finished chunk (slots 1..k) over ring block m mod w
    if (act == 2 && a.w > 0) {
        int64_t ring = 1 + a.k + (m % a.w) * a.k;
        int64_t items = (int64_t)a.Hkv * a.k * vec;
        for (int64_t e = t; e < items; e += kAppendThreads) {
            int h = (int)(e / (a.k * vec));
            int64_t rem = e % ((int64_t)a.k * vec);
            int64_t base = (((int64_t)b * a.Hkv + h) * a.S) * vec;
            a.K[base + ring * vec + rem] = a.K[base + 1 * vec + rem];
            a.V[base + ring * vec + rem] = a.V[base + 1 * vec + rem];
        }
    }
    __syncthreads();
    if (t == 0) {
        if (act == 1) st[0] = (int32_t)(n + 1);
        else st[1] = (int32_t)(m + 1);
    }
}

int launch_cache_append(const ksa_params *p, const ksa_cache *c, const int8_t *kind,
                        const void *k_new, const void *v_new, cudaStream_t st)
{
    if (c->batch == 0) return KSA_OK;
    AppendArgs a;
    a.k = p->k; a.w = p->w; a.Hkv = p->num_kv_heads; a.d = p->head_dim;
    a.S = ksa_cache_slots(p, c->cap_summaries);
    a.cap = c->cap_summaries;
    a.rotate = p->rope_theta > 0.0;
    a.log2_theta = a.rotate ? log2(p->rope_theta) : 0.0;
    a.kind = kind; a.state = c->state;
    a.k_new = (const uint4 *)k_new; a.v_new = (const uint4 *)v_new;
    a.K = (uint4 *)c->k; a.V = (uint4 *)c->v;
    cache_append_kernel<<<c->batch, kAppendThreads, 0, st>>>(a);
    return cudaGetLastError() == cudaSuccess ? KSA_OK : KSA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Hand-off: the decode cache of a prefilled batch in one pass.  Sequence b
// (blockIdx.y) lists its rows as: m summaries, then the k tokens of each of
// its last R = min(m, w) complete chunks, then its f open tokens; every
// (row, kv head, 16-byte piece) is one item of a grid-stride loop, so one
// warp copies 512 contiguous bytes of a source row (two heads) and writes
// each head's 256 bytes to its own slot.  HBM-bound copy.
// ---------------------------------------------------------------------------
struct BuildArgs {
    int k, w, Hkv, D8;        // D8: 16-byte pieces per head row
    int64_t S, cap;
    const int32_t *cu;
    Plan pl;
    const int32_t *err;
    const uint4 *ka, *va;     // [aug_rows, Hkv, d]
    uint4 *K, *V;             // [B, Hkv, S, d]
    int32_t *state;
};

constexpr int kBuildThreads = 256;

__global__ void __launch_bounds__(kBuildThreads) cache_build_kernel(BuildArgs a)
{
    const int b = blockIdx.y;
    if (*a.err != 0) return;   // the plan found cu_seqlens inconsistent
    const int n = a.cu[b + 1] - a.cu[b];
    const int k = a.k, m = n / k, f = n - m * k;
    const int64_t cs = a.pl.chunk_off[b];
    const bool lead = blockIdx.x == 0 && threadIdx.x == 0;
    if ((int64_t)m > a.cap) {
        if (lead) a.state[4 * (int64_t)b + 3] = KSA_ERR_CAPACITY;
        return;
    }
    if (lead) {
        a.state[4 * (int64_t)b + 0] = n;
        a.state[4 * (int64_t)b + 1] = m;
        a.state[4 * (int64_t)b + 2] = 0;
        a.state[4 * (int64_t)b + 3] = 0;
    }
    const int R = min(m, a.w);
    const int64_t rows = (int64_t)m + (int64_t)R * k + f;
    const int64_t total = rows * a.Hkv * a.D8;
    for (int64_t it = (int64_t)blockIdx.x * kBuildThreads + threadIdx.x; it < total;
         it += (int64_t)gridDim.x * kBuildThreads) {
        const int j = (int)(it % a.D8);
        const int64_t t = it / a.D8;
        const int h = (int)(t % a.Hkv);
        const int64_t idx = t / a.Hkv;
        int64_t src_row, slot;
        if (idx < m) {                       // summary s_idx
            src_row = (cs + idx) * (k + 1) + k;
            slot = 1 + k + (int64_t)a.w * k + idx;
        } else if (idx < m + (int64_t)R * k) {   // ring: chunk c, token r
            const int64_t q = idx - m;
            const int64_t c = m - R + q / k;
            const int r = (int)(q % k);
            src_row = (cs + c) * (k + 1) + r;
            slot = k + 1 + (c % a.w) * k + (k - 1 - r);
        } else {                             // open chunk m, token r
            const int r = (int)(idx - m - (int64_t)R * k);
            src_row = (cs + m) * (k + 1) + r;
            slot = k - r;
        }
        const int64_t src = (src_row * a.Hkv + h) * a.D8 + j;
        const int64_t dst = (((int64_t)b * a.Hkv + h) * a.S + slot) * a.D8 + j;
        a.K[dst] = a.ka[src];
        a.V[dst] = a.va[src];
    }
}

int launch_cache_build(const ksa_params *p, const ksa_cache *c, const int32_t *cu, const void *k_aug,
                       const void *v_aug, const Plan &pl, int32_t *err, cudaStream_t st)
{
    if (c->batch == 0) return KSA_OK;
    BuildArgs a;
    a.k = p->k; a.w = p->w; a.Hkv = p->num_kv_heads; a.D8 = p->head_dim / 8;
    a.S = ksa_cache_slots(p, c->cap_summaries);
    a.cap = c->cap_summaries;
    a.cu = cu; a.pl = pl; a.err = err;
    a.ka = (const uint4 *)k_aug; a.va = (const uint4 *)v_aug;
    a.K = (uint4 *)c->k; a.V = (uint4 *)c->v;
    a.state = c->state;
    // rows per sequence are at most cap + w k + k; the grid-stride loop covers the rest
    const int64_t max_items = (c->cap_summaries + (int64_t)p->w * p->k + p->k) * a.Hkv * a.D8;
    int64_t gx = (max_items + kBuildThreads - 1) / kBuildThreads;
    const int64_t gmax = 4LL * sm_count();
    if (gx > gmax) gx = gmax;
    if (gx < 1) gx = 1;
    cache_build_kernel<<<dim3((unsigned)gx, (unsigned)c->batch), kBuildThreads, 0, st>>>(a);
    return cudaGetLastError() == cudaSuccess ? KSA_OK : KSA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// Decode: split-K over the contiguous slice.
//
// Grid (nsplit, Hkv, B); 4 warps per CTA, each taking 16 key rows per step.
// The per-key dot products and the P V product run on the warp-level tensor
// core instruction (decode_split_kernel below); softmax runs in the log2
// domain with the scale applied to the fp32 scores.
// ---------------------------------------------------------------------------
constexpr int kDecWarps = 4;
constexpr int kDecThreads = kDecWarps * 32;

struct DecodeArgs {
    int k, w, Hkv, Hq, nsplit;
    int64_t S;
    float scale_log2;
    int rotate;
    double log2_theta;
    const int8_t *kind;
    int32_t *state;
    const __nv_bfloat16 *q;   // [B, Hq, d]
    const uint4 *K, *V;       // [B, Hkv, S, d]
    float *part;              // [B, Hkv, nsplit, G*(2 + d)]
};

__device__ __forceinline__ void bf16x8_to_f32(const uint4 &u, float *f)
{
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
    }
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ float ex2f_approx(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

using wm::mma16816;
using wm::movtrans;
using wm::word;

// Split-K decode on the warp-level tensor-core MMA.  The slice is read with
// 16-byte loads: lane (g, t) = (lane / 4, lane % 4) loads dims
// [32v + 8t, 32v + 8t + 8) of key rows g and g + 8 of each 16-row group.
// Keys are the MMA rows: S^T = K Q^T (A = K, B = Q^T with the G query heads
// as the 8 MMA columns) and O^T = V^T P^T.  The dot product is invariant
// under any permutation of d applied to both q and k, so the fragment a lane
// feeds to the MMA is exactly what it loaded; V and P fragments are turned
// around with movmatrix.  Softmax statistics per head are merged with warp
// shuffles.
template <int D, int G>
__global__ void __launch_bounds__(kDecThreads, 3) decode_split_kernel(DecodeArgs a)
{
    static_assert(G <= 8, "query heads per kv head must fit the 8 MMA columns");
    constexpr int NV = D / 32;     // 16-byte loads per key row and lane
    constexpr int NC = D / 16;     // MMA k-chunks of the QK product
    constexpr int NM = D / 16;     // MMA m-tiles of the PV product
    constexpr int HALF = D / 2;
    __shared__ float s_q[G][D];
    __shared__ float s_cos[HALF], s_sin[HALF];
    __shared__ float s_m[kDecWarps][G], s_l[kDecWarps][G];
    __shared__ float s_acc[kDecWarps][G][D];

    const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int kind = a.kind[b];
    if (kind == KSA_SKIP) return;
    const int64_t n = a.state[4 * (int64_t)b], m = a.state[4 * (int64_t)b + 1];
    int64_t lo, hi;
    if (!decode_slice(kind, n, m, a.k, a.w, &lo, &hi) || hi > a.S) {
        if (split == 0 && h == 0 && t == 0) a.state[4 * (int64_t)b + 3] = KSA_ERR_STATE;
        return;
    }
    // this split's range
    const int64_t L = hi - lo;
    const int64_t per = (L + a.nsplit - 1) / a.nsplit;
    const int64_t r0 = lo + (int64_t)split * per;
    const int64_t r1 = min(hi, r0 + per);

    // rotated q of the G heads of this kv head, position n - 1
    for (int r = t; r < HALF; r += kDecThreads) {
        float c = 1.f, s = 0.f;
        if (a.rotate) rope_cos_sin((double)(n - 1), r, D, a.log2_theta, &c, &s);
        s_cos[r] = c; s_sin[r] = s;
    }
    __syncthreads();
    for (int e = t; e < G * HALF; e += kDecThreads) {
        int g = e / HALF, r = e % HALF;
        const __nv_bfloat16 *qh = a.q + ((int64_t)b * a.Hq + (int64_t)h * G + g) * D;
        float x = __bfloat162float(qh[r]), y = __bfloat162float(qh[r + HALF]);
        float c = s_cos[r], s = s_sin[r];
        // the prefill path stores rotated q as bf16; round the same way
        s_q[g][r] = __bfloat162float(__float2bfloat16_rn(x * c - y * s));
        s_q[g][r + HALF] = __bfloat162float(__float2bfloat16_rn(y * c + x * s));
    }
    __syncthreads();

    const int g = lane >> 2, tt = lane & 3;
    // B fragments of Q^T: column (head) g, k-chunk c = 2v + hh covers dims
    // 32v + 8tt + 4hh + {0,1} (b0) and {2,3} (b1)
    uint32_t qb[NC][2];
#pragma unroll
    for (int c = 0; c < NC; ++c) {
        const int v = c / 2, hh = c % 2;
        const int d0 = 32 * v + 8 * tt + 4 * hh;
        if (g < G) {
            qb[c][0] = pack_bf16(s_q[g][d0], s_q[g][d0 + 1]);
            qb[c][1] = pack_bf16(s_q[g][d0 + 2], s_q[g][d0 + 3]);
        } else {
            qb[c][0] = qb[c][1] = 0u;
        }
    }
    // O^T accumulators: m-tile i = (v, pp): rows 0-7 are dims
    // 32v + 8(row/2) + 2(2pp) + row%2, rows 8-15 the same with 2pp + 1
    float o[NM][4];
#pragma unroll
    for (int i = 0; i < NM; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    // running max / sum of heads 2tt and 2tt + 1 (log2 domain)
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};

    const uint4 *Kb = a.K + (((int64_t)b * a.Hkv + h) * a.S) * (D / 8);
    const uint4 *Vb = a.V + (((int64_t)b * a.Hkv + h) * a.S) * (D / 8);
    for (int64_t kb = r0 + 16 * warp; kb < r1; kb += 16 * kDecWarps) {
        const int64_t key0 = kb + g, key1 = kb + g + 8;
        const bool in0 = key0 < r1, in1 = key1 < r1;
        uint4 kA[NV], kB[NV], vA[NV], vB[NV];
#pragma unroll
        for (int v = 0; v < NV; ++v) {
            const uint4 z = make_uint4(0, 0, 0, 0);
            kA[v] = in0 ? __ldcs(Kb + key0 * (D / 8) + 4 * v + tt) : z;
            kB[v] = in1 ? __ldcs(Kb + key1 * (D / 8) + 4 * v + tt) : z;
            vA[v] = in0 ? __ldcs(Vb + key0 * (D / 8) + 4 * v + tt) : z;
            vB[v] = in1 ? __ldcs(Vb + key1 * (D / 8) + 4 * v + tt) : z;
        }
        // S^T = K Q^T for the 16 keys
        float sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < NC; ++c) {
            const int v = c / 2, hh = c % 2;
            mma16816(sc, word(kA[v], 2 * hh), word(kB[v], 2 * hh), word(kA[v], 2 * hh + 1),
                     word(kB[v], 2 * hh + 1), qb[c][0], qb[c][1]);
        }
        // sc[0..1]: key g, heads 2tt, 2tt+1; sc[2..3]: key g + 8
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
            const float m_new = fmaxf(m_run[e], mx);
            corr[e] = (m_new == -INFINITY) ? 1.f : ex2f_approx(m_run[e] - m_new);
            pv[e] = (m_new == -INFINITY) ? 0.f : ex2f_approx(x[e] - m_new);
            pv[e + 2] = (m_new == -INFINITY) ? 0.f : ex2f_approx(x[e + 2] - m_new);
            l_run[e] = l_run[e] * corr[e] + pv[e] + pv[e + 2];
            m_run[e] = m_new;
        }
        if (__any_sync(0xffffffffu, corr[0] != 1.f || corr[1] != 1.f)) {
#pragma unroll
            for (int i = 0; i < NM; ++i) {
                o[i][0] *= corr[0]; o[i][1] *= corr[1];
                o[i][2] *= corr[0]; o[i][3] *= corr[1];
            }
        }
        // P^T fragments (k = keys, n = heads) by transposing the S^T layout
        const uint32_t pb0 = movtrans(pack_bf16(pv[0], pv[1]));
        const uint32_t pb1 = movtrans(pack_bf16(pv[2], pv[3]));
        // O^T += V^T P^T
#pragma unroll
        for (int i = 0; i < NM; ++i) {
            const int v = i / 2, pp = i % 2;
            mma16816(o[i], movtrans(word(vA[v], 2 * pp)), movtrans(word(vA[v], 2 * pp + 1)),
                     movtrans(word(vB[v], 2 * pp)), movtrans(word(vB[v], 2 * pp + 1)), pb0, pb1);
        }
    }
    // row sums: the lanes of a head share its max, so partial sums add up
#pragma unroll
    for (int e = 0; e < 2; ++e)
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) l_run[e] += __shfl_xor_sync(0xffffffffu, l_run[e], off);
    // scatter this warp's O^T into s_acc[warp][head][dim]
#pragma unroll
    for (int i = 0; i < NM; ++i) {
        const int v = i / 2, pp = i % 2;
        const int dA = 32 * v + 8 * (g / 2) + 2 * (2 * pp) + (g % 2);
        const int dB = dA + 2;
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int head = 2 * tt + e;
            if (head < G) {
                s_acc[warp][head][dA] = o[i][e];
                s_acc[warp][head][dB] = o[i][2 + e];
            }
        }
    }
    if (g == 0) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int head = 2 * tt + e;
            if (head < G) { s_m[warp][head] = m_run[e]; s_l[warp][head] = l_run[e]; }
        }
    }
    __syncthreads();
    float *out = a.part + ((((int64_t)b * a.Hkv + h) * a.nsplit) + split) * (G * (2 + D));
    for (int e = t; e < G * D; e += kDecThreads) {
        int gg = e / D, dd = e % D;
        float mm = -INFINITY;
#pragma unroll
        for (int w2 = 0; w2 < kDecWarps; ++w2) mm = fmaxf(mm, s_m[w2][gg]);
        float ll = 0.f, aa = 0.f;
#pragma unroll
        for (int w2 = 0; w2 < kDecWarps; ++w2) {
            float cf = (mm == -INFINITY) ? 0.f : ex2f_approx(s_m[w2][gg] - mm);
            ll += s_l[w2][gg] * cf;
            aa += s_acc[w2][gg][dd] * cf;
        }
        out[2 * G + gg * D + dd] = aa;
        if (dd == 0) { out[gg] = mm; out[G + gg] = ll; }
    }
}

// Merge the nsplit partial states of each (sequence, kv head) and write o, lse,
// for few splits: one thread per output element walks the splits.
template <int D, int G>
__global__ void __launch_bounds__(256) decode_combine_kernel(DecodeArgs a, __nv_bfloat16 *o, float *lse)
{
    const int h = blockIdx.x, b = blockIdx.y, t = threadIdx.x;
    const int kind = a.kind[b];
    if (kind == KSA_SKIP) return;
    int64_t lo, hi;
    if (!decode_slice(kind, a.state[4 * (int64_t)b], a.state[4 * (int64_t)b + 1], a.k, a.w, &lo, &hi) ||
        hi > a.S)
        return;
    const float *part = a.part + (((int64_t)b * a.Hkv + h) * a.nsplit) * (G * (2 + D));
    const int stride = G * (2 + D);
    for (int e = t; e < G * D; e += blockDim.x) {
        int g = e / D, dd = e % D;
        float mm = -INFINITY;
        for (int s = 0; s < a.nsplit; ++s) mm = fmaxf(mm, part[s * stride + g]);
        float ll = 0.f, aa = 0.f;
        for (int s = 0; s < a.nsplit; ++s) {
            float ms = part[s * stride + g];
            float cf = (ms == -INFINITY) ? 0.f : ex2f_approx(ms - mm);
            ll += part[s * stride + G + g] * cf;
            aa += part[s * stride + 2 * G + g * D + dd] * cf;
        }
        int64_t oi = ((int64_t)b * a.Hq + (int64_t)h * G + g) * D + dd;
        o[oi] = __float2bfloat16_rn(aa / ll);
        if (lse && dd == 0) lse[(int64_t)b * a.Hq + (int64_t)h * G + g] = (mm + log2f(ll)) * 0.69314718055994530942f;
    }
}

// The same merge for many splits (kDecWideCombine or more; a batch of one
// long sequence takes hundreds), where a thread per element walking every
// split in turn waits on one load at a time.  One CTA per (kv head,
// sequence): the G heads' maxima over the splits first
// (threads strided over the splits, then a block reduction), then warp w sums
// splits w, w + 8, ... (each lane 32-strided over the G x D outputs, so a
// split's row of partials is one coalesced read and every lane has
// independent loads in flight), and the eight warps' sums are added at the end.
template <int D, int G>
__global__ void __launch_bounds__(256) decode_combine_wide_kernel(DecodeArgs a, __nv_bfloat16 *o, float *lse)
{
    constexpr int W = 8, E = G * D, EPL = E / 32;
    __shared__ float s_red[W][E + G];   // per warp: the G x D sums, then the G row sums
    __shared__ float s_mx[W][G];
    const int h = blockIdx.x, b = blockIdx.y, t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int kind = a.kind[b];
    if (kind == KSA_SKIP) return;
    int64_t lo, hi;
    if (!decode_slice(kind, a.state[4 * (int64_t)b], a.state[4 * (int64_t)b + 1], a.k, a.w, &lo, &hi) ||
        hi > a.S)
        return;
    const float *part = a.part + (((int64_t)b * a.Hkv + h) * a.nsplit) * (G * (2 + D));
    const int stride = G * (2 + D);
    float mm[G];
#pragma unroll
    for (int g = 0; g < G; ++g) mm[g] = -INFINITY;
    for (int s = t; s < a.nsplit; s += blockDim.x)
#pragma unroll
        for (int g = 0; g < G; ++g) mm[g] = fmaxf(mm[g], part[(int64_t)s * stride + g]);
#pragma unroll
    for (int g = 0; g < G; ++g) {
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mm[g] = fmaxf(mm[g], __shfl_xor_sync(0xffffffffu, mm[g], off));
        if (lane == 0) s_mx[warp][g] = mm[g];
    }
    __syncthreads();
#pragma unroll
    for (int g = 0; g < G; ++g) {
        mm[g] = s_mx[0][g];
#pragma unroll
        for (int w2 = 1; w2 < W; ++w2) mm[g] = fmaxf(mm[g], s_mx[w2][g]);
    }
    float acc[EPL], ll[G];
#pragma unroll
    for (int i = 0; i < EPL; ++i) acc[i] = 0.f;
#pragma unroll
    for (int g = 0; g < G; ++g) ll[g] = 0.f;
    for (int s = warp; s < a.nsplit; s += W) {
        const float *ps = part + (int64_t)s * stride;
        float cf[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float ms = ps[g];
            cf[g] = (ms == -INFINITY) ? 0.f : ex2f_approx(ms - mm[g]);
            ll[g] += ps[G + g] * cf[g];
        }
#pragma unroll
        for (int i = 0; i < EPL; ++i) acc[i] += ps[2 * G + lane + 32 * i] * cf[(32 * i) / D];
    }
#pragma unroll
    for (int i = 0; i < EPL; ++i) s_red[warp][lane + 32 * i] = acc[i];
    if (lane == 0)
#pragma unroll
        for (int g = 0; g < G; ++g) s_red[warp][E + g] = ll[g];
    __syncthreads();
    for (int e = t; e < E; e += blockDim.x) {
        const int g = e / D, dd = e % D;
        float aa = 0.f, lt = 0.f;
#pragma unroll
        for (int w2 = 0; w2 < W; ++w2) {
            aa += s_red[w2][e];
            lt += s_red[w2][E + g];
        }
        const int64_t oi = ((int64_t)b * a.Hq + (int64_t)h * G + g) * D + dd;
        o[oi] = __float2bfloat16_rn(aa / lt);
        if (lse && dd == 0) lse[(int64_t)b * a.Hq + (int64_t)h * G + g] = (mm[g] + log2f(lt)) * 0.69314718055994530942f;
    }
}

constexpr int kDecWideCombine = 16;   // split count from which the wide merge is faster

int decode_splits(const ksa_params *p, int batch, int64_t max_text)
{
    int64_t max_slice = 1 + p->k + (int64_t)p->w * p->k + max_text / p->k;
    int64_t units = (int64_t)batch * p->num_kv_heads;
    // ~8 waves of 4 CTAs per SM, at least 1024 rows per split; but at least
    // two CTAs per SM while splits keep 512 rows or more (small batches)
    const int64_t sms = sm_count();
    int64_t want = (32LL * sms + units - 1) / units;
    int64_t cap = (max_slice + 1023) / 1024;
    int64_t s = want < cap ? want : cap;
    if (s * units < 2 * sms) {
        const int64_t fill = (2 * sms + units - 1) / units, cap512 = (max_slice + 511) / 512;
        const int64_t s2 = fill < cap512 ? fill : cap512;
        if (s2 > s) s = s2;
    }
    if (s < 1) s = 1;
    if (s > 1024) s = 1024;
    return (int)s;
}

size_t decode_split_bytes(const ksa_params *p, int batch)
{
    const int G = p->num_q_heads / p->num_kv_heads;
    return sizeof(float) * (size_t)batch * p->num_kv_heads * G * (2 + p->head_dim);
}

size_t decode_workspace_bytes(const ksa_params *p, int batch, int64_t max_text)
{
    return align_up(decode_split_bytes(p, batch) * (size_t)decode_splits(p, batch, max_text));
}

template <int D, int G>
static int launch_decode_t(const DecodeArgs &a, int batch, __nv_bfloat16 *o, float *lse, cudaStream_t st)
{
    dim3 grid(a.nsplit, a.Hkv, batch);
    decode_split_kernel<D, G><<<grid, kDecThreads, 0, st>>>(a);
    if (a.nsplit >= kDecWideCombine)
        decode_combine_wide_kernel<D, G><<<dim3(a.Hkv, batch), 256, 0, st>>>(a, o, lse);
    else
        decode_combine_kernel<D, G><<<dim3(a.Hkv, batch), 256, 0, st>>>(a, o, lse);
    return cudaGetLastError() == cudaSuccess ? KSA_OK : KSA_ERR_CUDA;
}

int launch_decode(const ksa_params *p, const ksa_cache *c, const int8_t *kind, const void *q,
                  void *o, float *lse, int64_t max_text, void *ws, size_t ws_bytes,
                  cudaStream_t st)
{
    if (c->batch == 0) return KSA_OK;
    if (ws_bytes < decode_workspace_bytes(p, c->batch, max_text)) return KSA_ERR_WORKSPACE;
    return launch_decode_splits(p, c, kind, q, o, lse, decode_splits(p, c->batch, max_text), ws, st);
}

int launch_decode_splits(const ksa_params *p, const ksa_cache *c, const int8_t *kind, const void *q, void *o,
                         float *lse, int nsplit, void *ws, cudaStream_t st)
{
    if (c->batch == 0) return KSA_OK;
    if (nsplit < 1) return KSA_ERR_INVALID;
    DecodeArgs a;
    a.k = p->k; a.w = p->w; a.Hkv = p->num_kv_heads; a.Hq = p->num_q_heads;
    a.nsplit = nsplit;
    a.S = ksa_cache_slots(p, c->cap_summaries);
    float scale = p->scale > 0.f ? p->scale : 1.0f / sqrtf((float)p->head_dim);
    a.scale_log2 = scale * 1.4426950408889634f;
    a.rotate = p->rope_theta > 0.0;
    a.log2_theta = a.rotate ? log2(p->rope_theta) : 0.0;
    a.kind = kind; a.state = c->state;
    a.q = (const __nv_bfloat16 *)q;
    a.K = (const uint4 *)c->k; a.V = (const uint4 *)c->v;
    a.part = (float *)ws;
    const int G = p->num_q_heads / p->num_kv_heads;
    __nv_bfloat16 *ob = (__nv_bfloat16 *)o;
#define KSA_DEC(DD, GG) \
    if (p->head_dim == DD && G == GG) return launch_decode_t<DD, GG>(a, c->batch, ob, lse, st);
    KSA_DEC(128, 1) KSA_DEC(128, 2) KSA_DEC(128, 4) KSA_DEC(128, 8)
    KSA_DEC(64, 1) KSA_DEC(64, 2) KSA_DEC(64, 4) KSA_DEC(64, 8)
#undef KSA_DEC
    return KSA_ERR_UNSUPPORTED;
}

}  // namespace ksa

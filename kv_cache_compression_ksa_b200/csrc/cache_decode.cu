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
        int act = 0;
        if (kind == KSA_TEXT) {
            if (f >= 0 && f < a.k) act = 1; else st[3] = KSA_ERR_STATE;
        } else if (kind == KSA_SUMMARY) {
            if (f != a.k) st[3] = KSA_ERR_STATE;
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
// Decode: split-K over the contiguous slice.
//
// Grid (nsplit, Hkv, B); 4 warps per CTA.  A warp reads KPW = 32/LPK key
// rows per 16-byte load instruction (LPK = d/8 lanes per row), U rows per
// lane group per step, so every load instruction covers KPW*d*2 contiguous
// bytes.  Each lane keeps the G query heads' slice of 8 dims and its own
// running (max, sum, acc) per head; scores are completed with an xor
// butterfly over the LPK lanes of a row.  Softmax runs in the log2 domain
// with the scale folded into q.
// ---------------------------------------------------------------------------
constexpr int kDecWarps = 4;
constexpr int kDecThreads = kDecWarps * 32;
constexpr int kDecU = 4;

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

__device__ __forceinline__ float ex2f_approx(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Slice of one sequence after its append: [lo, hi) in slots.  Returns false
// (and records the error) if the state cannot hold a query of this kind.
__device__ __forceinline__ bool decode_slice(int kind, int64_t n, int64_t m, int k, int w,
                                             int64_t *lo, int64_t *hi)
{
    int64_t f = n - m * k;
    if (kind == KSA_SUMMARY) {
        if (m < 1 || f != 0) return false;
        *lo = 0; *hi = k + 1;
        return true;
    }
    if (f < 1 || f > k) return false;
    int64_t ring = m < w ? m : w;
    int64_t far = m > w ? m - w : 0;
    *lo = k - f + 1;
    *hi = 1 + k + ring * k + far;
    return true;
}

template <int D, int G>
__global__ void __launch_bounds__(kDecThreads, 3) decode_split_kernel(DecodeArgs a)
{
    constexpr int LPK = D / 8;     // lanes per key row (8 dims = 16 bytes each)
    constexpr int KPW = 32 / LPK;  // key rows per warp load instruction
    constexpr int U = (LPK / G) < 4 ? (LPK / G) : 4;  // key rows per lane group per step
    constexpr int NV = U * G;      // scores per lane group per step (<= LPK)
    // after the reduce-scatter each score is complete on LPK/NV lanes: lane
    // c8 holds score number c8 >> SH
    constexpr int SH = (LPK / NV) == 1 ? 0 : (LPK / NV) == 2 ? 1 : (LPK / NV) == 4 ? 2 : 3;
    constexpr int HALF = D / 2;
    static_assert(NV <= LPK && (LPK >> SH) == NV, "score layout");
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
    if (!decode_slice(kind, n, m, a.k, a.w, &lo, &hi)) {
        if (split == 0 && h == 0 && t == 0) a.state[4 * (int64_t)b + 3] = KSA_ERR_STATE;
        return;
    }
    // this split's range
    const int64_t L = hi - lo;
    const int64_t per = (L + a.nsplit - 1) / a.nsplit;
    const int64_t r0 = lo + (int64_t)split * per;
    const int64_t r1 = min(hi, r0 + per);

    // rotated, pre-scaled q of the G heads of this kv head, position n - 1
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
        float xr = __bfloat162float(__float2bfloat16_rn(x * c - y * s));
        float yr = __bfloat162float(__float2bfloat16_rn(y * c + x * s));
        s_q[g][r] = xr * a.scale_log2;
        s_q[g][r + HALF] = yr * a.scale_log2;
    }
    __syncthreads();

    const int sub = lane / LPK;   // which key row of the warp load
    const int c8 = lane % LPK;    // which 8 dims; after the reduce-scatter: score (u*G+g) << SH
    float qf[G][8];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int e = 0; e < 8; ++e) qf[g][e] = s_q[g][c8 * 8 + e];

    // running state: max and sum of this lane's score slot (head my_g), and
    // the accumulators of every head for this lane's 8 dims
    float m_run = -INFINITY, l_run = 0.f, acc[G][8];
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[g][e] = 0.f;

    const uint4 *Kb = a.K + (((int64_t)b * a.Hkv + h) * a.S) * (D / 8) + c8;
    const uint4 *Vb = a.V + (((int64_t)b * a.Hkv + h) * a.S) * (D / 8) + c8;
    constexpr int STEP = kDecWarps * KPW * U;  // rows per CTA step
    auto load = [&](int64_t base, uint4 *kr, uint4 *vr) {
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t row = base + ((int64_t)u * kDecWarps + warp) * KPW + sub;
            if (row < r1) {
                kr[u] = __ldcs(Kb + row * (D / 8));
                vr[u] = __ldcs(Vb + row * (D / 8));
            } else {
                kr[u] = make_uint4(0, 0, 0, 0);
                vr[u] = kr[u];
            }
        }
    };
    uint4 kr[U], vr[U], kn[U], vn[U];
    load(r0, kr, vr);
    for (int64_t base = r0; base < r1; base += STEP) {
        if (base + STEP < r1) load(base + STEP, kn, vn);   // next step's rows in flight
        // partial scores of this lane's 8 dims: v[u*G + g]
        float v[NV];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            float kf[8];
            bf16x8_to_f32(kr[u], kf);
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float s = 0.f;
#pragma unroll
                for (int e = 0; e < 8; ++e) s = fmaf(qf[g][e], kf[e], s);
                v[u * G + g] = s;
            }
        }
        // reduce-scatter over the LPK lanes of a row group (top log2(NV)
        // lane bits), then all-reduce over the remaining SH bits
#pragma unroll
        for (int off = LPK / 2, half = NV / 2; off >= 1; off >>= 1, half = half > 1 ? half / 2 : 0) {
            if (half >= 1) {
                const bool upper = (c8 & off) != 0;
#pragma unroll
                for (int i = 0; i < half; ++i) {
                    const float send = upper ? v[i] : v[i + half];
                    const float keep = upper ? v[i + half] : v[i];
                    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
                }
            } else {
                v[0] += __shfl_xor_sync(0xffffffffu, v[0], off);
            }
        }
        const int my_u = (c8 >> SH) / G;
        const int64_t my_row = base + ((int64_t)my_u * kDecWarps + warp) * KPW + sub;
        float sc = my_row < r1 ? v[0] : -INFINITY;
        // max over the U scores of this lane's head (score bits above log2 G)
        float mx = sc;
#pragma unroll
        for (int off = G << SH; off < LPK; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        const float m_new = fmaxf(m_run, mx);
        const float corr = (m_new == -INFINITY) ? 1.f : ex2f_approx(m_run - m_new);
        const float p = (m_new == -INFINITY) ? 0.f : ex2f_approx(sc - m_new);
        m_run = m_new;
        l_run = l_run * corr + p;
        // every lane needs each head's correction and every (u, g) weight
        const int gbase = lane & ~(LPK - 1);
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float cg = __shfl_sync(0xffffffffu, corr, gbase + (g << SH));
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[g][e] *= cg;
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            float vf[8];
            bf16x8_to_f32(vr[u], vf);
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float pg = __shfl_sync(0xffffffffu, p, gbase + ((u * G + g) << SH));
#pragma unroll
                for (int e = 0; e < 8; ++e) acc[g][e] = fmaf(pg, vf[e], acc[g][e]);
            }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) { kr[u] = kn[u]; vr[u] = vn[u]; }
    }
    // per head: combine the U score slots of the row group (the copies on
    // the low SH lane bits are identical and are not summed)
    {
        float mx = m_run;
#pragma unroll
        for (int off = G << SH; off < LPK; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        float l = (mx == -INFINITY) ? 0.f : l_run * ex2f_approx(m_run - mx);
#pragma unroll
        for (int off = G << SH; off < LPK; off <<= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
        m_run = mx;
        l_run = l;
    }
    // lanes whose score number has head g now hold (m, l) of head g; the
    // accumulators are already relative to each head's m_run
    float mh[G], lh[G];
    {
        const int gbase = lane & ~(LPK - 1);
#pragma unroll
        for (int g = 0; g < G; ++g) {
            mh[g] = __shfl_sync(0xffffffffu, m_run, gbase + (g << SH));
            lh[g] = __shfl_sync(0xffffffffu, l_run, gbase + (g << SH));
        }
    }
    // merge the KPW row groups of the warp (lanes c8 + j*LPK)
#pragma unroll
    for (int off = LPK; off < 32; off <<= 1) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
            float mo = __shfl_xor_sync(0xffffffffu, mh[g], off);
            float lo_ = __shfl_xor_sync(0xffffffffu, lh[g], off);
            float mn = fmaxf(mh[g], mo);
            float ca = (mn == -INFINITY) ? 0.f : ex2f_approx(mh[g] - mn);
            float cb = (mn == -INFINITY) ? 0.f : ex2f_approx(mo - mn);
            lh[g] = lh[g] * ca + lo_ * cb;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                float ao = __shfl_xor_sync(0xffffffffu, acc[g][e], off);
                acc[g][e] = acc[g][e] * ca + ao * cb;
            }
            mh[g] = mn;
        }
    }
    if (sub == 0) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
            if (c8 == 0) { s_m[warp][g] = mh[g]; s_l[warp][g] = lh[g]; }
#pragma unroll
            for (int e = 0; e < 8; ++e) s_acc[warp][g][c8 * 8 + e] = acc[g][e];
        }
    }
    __syncthreads();
    float *out = a.part + ((((int64_t)b * a.Hkv + h) * a.nsplit) + split) * (G * (2 + D));
    for (int e = t; e < G * D; e += kDecThreads) {
        int g = e / D, dd = e % D;
        float mm = -INFINITY;
#pragma unroll
        for (int w2 = 0; w2 < kDecWarps; ++w2) mm = fmaxf(mm, s_m[w2][g]);
        float ll = 0.f, aa = 0.f;
#pragma unroll
        for (int w2 = 0; w2 < kDecWarps; ++w2) {
            float cf = (mm == -INFINITY) ? 0.f : ex2f_approx(s_m[w2][g] - mm);
            ll += s_l[w2][g] * cf;
            aa += s_acc[w2][g][dd] * cf;
        }
        out[2 * G + g * D + dd] = aa;
        if (dd == 0) { out[g] = mm; out[G + g] = ll; }
    }
}

// Merge the nsplit partial states of each (sequence, kv head) and write o, lse.
template <int D, int G>
__global__ void __launch_bounds__(256) decode_combine_kernel(DecodeArgs a, __nv_bfloat16 *o, float *lse)
{
    const int h = blockIdx.x, b = blockIdx.y, t = threadIdx.x;
    const int kind = a.kind[b];
    if (kind == KSA_SKIP) return;
    int64_t lo, hi;
    if (!decode_slice(kind, a.state[4 * (int64_t)b], a.state[4 * (int64_t)b + 1], a.k, a.w, &lo, &hi))
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

static int decode_splits(const ksa_params *p, int batch, int64_t max_text)
{
    int64_t max_slice = 1 + p->k + (int64_t)p->w * p->k + max_text / p->k;
    int64_t units = (int64_t)batch * p->num_kv_heads;
    int64_t want = (32LL * sm_count() + units - 1) / units;  // ~8 waves of 4 CTAs per SM
    int64_t cap = (max_slice + 511) / 512;                      // >= 512 rows per split
    int64_t s = want < cap ? want : cap;
    if (s < 1) s = 1;
    if (s > 1024) s = 1024;
    return (int)s;
}

size_t decode_workspace_bytes(const ksa_params *p, int batch, int64_t max_text)
{
    int G = p->num_q_heads / p->num_kv_heads;
    int s = decode_splits(p, batch, max_text);
    return align_up(sizeof(float) * (size_t)batch * p->num_kv_heads * s * G * (2 + p->head_dim));
}

template <int D, int G>
static int launch_decode_t(const DecodeArgs &a, int batch, __nv_bfloat16 *o, float *lse, cudaStream_t st)
{
    dim3 grid(a.nsplit, a.Hkv, batch);
    decode_split_kernel<D, G><<<grid, kDecThreads, 0, st>>>(a);
    decode_combine_kernel<D, G><<<dim3(a.Hkv, batch), 256, 0, st>>>(a, o, lse);
    return cudaGetLastError() == cudaSuccess ? KSA_OK : KSA_ERR_CUDA;
}

int launch_decode(const ksa_params *p, const ksa_cache *c, const int8_t *kind, const void *q,
                  void *o, float *lse, int64_t max_text, void *ws, size_t ws_bytes,
                  cudaStream_t st)
{
    if (c->batch == 0) return KSA_OK;
    if (ws_bytes < decode_workspace_bytes(p, c->batch, max_text)) return KSA_ERR_WORKSPACE;
    DecodeArgs a;
    a.k = p->k; a.w = p->w; a.Hkv = p->num_kv_heads; a.Hq = p->num_q_heads;
    a.nsplit = decode_splits(p, c->batch, max_text);
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

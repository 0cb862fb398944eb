// rope_interleave.cu -- batch plan and the RoPE + interleave kernel.
//
// Kwai Summary Attention Technical Report, section 2.2.1: the augmented
// sequence of Eq. (1) puts summary s_j after the k text tokens of chunk j,
// and s_j takes the position id of its chunk's last text token.  Table 3
// gives RoPE theta = 1e6.  Keys enter the decode cache already rotated
// (section 2.3.1), so rotation happens once, here, before attention.
//
// Memory-bound: every element is read once and written once.
#include "ksa_internal.cuh"

namespace ksa {

// ---------------------------------------------------------------------------
// Plan: one block scans the batch.  Per sequence n_b = cu[b+1]-cu[b]:
//   chunks ceil(n_b/k), summaries floor(n_b/k), work units
//   ceil(chunks/unit_chunks).  Checks the host-side totals (total_sum < 0:
//   not checked).
// ---------------------------------------------------------------------------
constexpr int kPlanThreads = 1024;

__global__ void __launch_bounds__(kPlanThreads)
plan_kernel(int batch, const int32_t *__restrict__ cu, int k, int unit_chunks,
            int64_t total_text, int64_t total_sum, int64_t aug_rows, Plan pl,
            int32_t *err, int reset_err)
{
    __shared__ int64_t s_chunks[kPlanThreads], s_sums[kPlanThreads], s_tiles[kPlanThreads];
    __shared__ int s_bad;
    const int t = threadIdx.x;
    if (t == 0) {
        if (reset_err) *err = 0;
        s_bad = 0;
    }
    __syncthreads();
    const int per = (batch + kPlanThreads - 1) / kPlanThreads;
    const int b0 = min(batch, t * per), b1 = min(batch, b0 + per);
    int64_t ch = 0, su = 0, ti = 0;
    int bad = 0;
    for (int b = b0; b < b1; ++b) {
        int n = cu[b + 1] - cu[b];
        if (n < 0) bad = 1;
        n = max(n, 0);
        int c = (int)(((int64_t)n + k - 1) / k);   // n may be INT32_MAX
        ch += c;
        su += n / k;
        if (unit_chunks > 0) ti += (c + unit_chunks - 1) / unit_chunks;
    }
    s_chunks[t] = ch; s_sums[t] = su; s_tiles[t] = ti;
    if (bad) s_bad = 1;
    __syncthreads();
    // inclusive scan (Hillis-Steele) over the per-thread sums
    for (int off = 1; off < kPlanThreads; off <<= 1) {
        int64_t a = 0, b2 = 0, c2 = 0;
        if (t >= off) { a = s_chunks[t - off]; b2 = s_sums[t - off]; c2 = s_tiles[t - off]; }
        __syncthreads();
        s_chunks[t] += a; s_sums[t] += b2; s_tiles[t] += c2;
        __syncthreads();
    }
    int64_t ch0 = t ? s_chunks[t - 1] : 0, su0 = t ? s_sums[t - 1] : 0, ti0 = t ? s_tiles[t - 1] : 0;
    for (int b = b0; b < b1; ++b) {
        int n = max(cu[b + 1] - cu[b], 0);
        int c = (int)(((int64_t)n + k - 1) / k);   // n may be INT32_MAX
        pl.chunk_off[b] = (int32_t)ch0;
        pl.sum_off[b] = (int32_t)su0;
        pl.tile_off[b] = (int32_t)ti0;
        ch0 += c;
        su0 += n / k;
        if (unit_chunks > 0) ti0 += (c + unit_chunks - 1) / unit_chunks;
    }
    if (t == kPlanThreads - 1) {
        pl.chunk_off[batch] = (int32_t)s_chunks[t];
        pl.sum_off[batch] = (int32_t)s_sums[t];
        pl.tile_off[batch] = (int32_t)s_tiles[t];
        bool ok = !s_bad && cu[0] == 0 && (int64_t)cu[batch] == total_text &&
                  (total_sum < 0 || s_sums[t] == total_sum) && s_chunks[t] * (int64_t)(k + 1) == aug_rows &&
                  s_chunks[t] < (int64_t)INT32_MAX;
        if (!ok) set_error(err, KSA_ERR_INVALID);
    }
}

int launch_plan(const ksa_params *p, int batch, const int32_t *cu, int64_t total_text,
                int64_t total_sum, int64_t aug_rows, const Plan &pl, int32_t *err,
                int unit_chunks, cudaStream_t st)
{
    plan_kernel<<<1, kPlanThreads, 0, st>>>(batch, cu, p->k, unit_chunks, total_text, total_sum,
                                            aug_rows, pl, err, err == pl.err);
    return cudaGetLastError() == cudaSuccess ? KSA_OK : KSA_ERR_CUDA;
}

// ---------------------------------------------------------------------------
// RoPE + interleave.  One block handles kRows augmented rows; per row the
// d/2 (cos, sin) pairs are computed once in fp64-reduced form and shared by
// all heads.  Work items: Q and K rotate 8 pairs (two 16-byte halves r and
// r + d/2), V copies 16 bytes.  Padding rows are written as zeros.
// ---------------------------------------------------------------------------
constexpr int kRopeThreads = 256;
constexpr int kRows = 4;

struct RopeArgs {
    int batch, k, Hq, Hkv, d;
    int64_t aug_rows;
    double log2_theta;
    int rotate;         // 0: RoPE disabled (theta <= 0)
    const int32_t *cu;
    Plan pl;
    int32_t *err;
    const uint4 *qt, *kt, *vt, *qs, *ks, *vs;
    uint4 *qa, *ka, *va;
};

// BWD: the backward (gradients of the augmented rows -> gradients of the
// text and summary projections).  The rotation is orthogonal, so its
// transpose is the rotation by the opposite angle; V is copied back; padding
// rows have no source and are skipped.  In that mode qa/ka/va are read and
// qt/kt/vt/qs/ks/vs written.
template <bool BWD>
__global__ void __launch_bounds__(kRopeThreads)
interleave_rope_kernel(RopeArgs a)
{
    __shared__ float s_cos[kRows][64], s_sin[kRows][64];
    __shared__ int64_t s_src[kRows];   // source row, -1 = padding
    __shared__ int s_is_sum[kRows];
    __shared__ int64_t s_pos[kRows];
    if (*a.err != 0) return;
    const int64_t row0 = (int64_t)blockIdx.x * kRows;
    const int half = a.d / 2;
    const int t = threadIdx.x;
    if (t < kRows) {
        int64_t R = row0 + t;
        int64_t src = -1;
        int is_sum = 0;
        int64_t pos = 0;
        if (R < a.aug_rows) {
            int64_t g = R / (a.k + 1);
            int r = (int)(R % (a.k + 1));
            // sequence: last b with chunk_off[b] <= g
            int lo = 0, hi = a.batch - 1;
            while (lo < hi) {
                int mid = (lo + hi + 1) >> 1;
                if (a.pl.chunk_off[mid] <= g) lo = mid; else hi = mid - 1;
            }
            int b = lo;
            int64_t c = g - a.pl.chunk_off[b];
            int n = a.cu[b + 1] - a.cu[b];
            if (r < a.k) {
                int64_t i = c * a.k + r;
                if (i < n) { src = a.cu[b] + i; pos = i; }
            } else {
                if (c < n / a.k) { src = a.pl.sum_off[b] + c; pos = c * a.k + a.k - 1; is_sum = 1; }
            }
        }
        s_src[t] = src;
        s_is_sum[t] = is_sum;
        s_pos[t] = pos;
    }
    __syncthreads();
    // (cos, sin) table: kRows * d/2 entries
    for (int e = t; e < kRows * half; e += kRopeThreads) {
        int r = e / half, pr = e % half;
        float c = 1.f, s = 0.f;
        if (a.rotate) rope_cos_sin((double)s_pos[r], pr, a.d, a.log2_theta, &c, &s);
        s_cos[r][pr] = c;
        s_sin[r][pr] = BWD ? -s : s;
    }
    __syncthreads();
    const int qv = a.Hq * a.d / 16;   // rotate items per Q row (8 pairs each)
    const int kv = a.Hkv * a.d / 16;  // rotate items per K row
    const int vv = a.Hkv * a.d / 8;   // 16-byte copy items per V row
    const int per_row = qv + kv + vv;
    const int chunks_half = half / 8;  // 16-byte chunks in one half of a head
    for (int e = t; e < kRows * per_row; e += kRopeThreads) {
        int r = e / per_row, it = e % per_row;
        int64_t R = row0 + r;
        if (R >= a.aug_rows) continue;
        int64_t src = s_src[r];
        const float *cs = s_cos[r], *sn = s_sin[r];
        if (it < qv + kv) {
            bool isq = it < qv;
            int j = isq ? it : it - qv;
            int H = isq ? a.Hq : a.Hkv;
            int h = j / chunks_half, c = j % chunks_half;
            // uint4 index of element (row, h, 8c) with d/8 uint4 per head row
            int64_t base_out = (R * H + h) * (a.d / 8);
            if (BWD) {
                if (src < 0) continue;
                const uint4 *in = isq ? a.qa : a.ka;
                uint4 lo = in[base_out + c], hi = in[base_out + c + chunks_half];
                rope_rot8(lo, hi, cs + 8 * c, sn + 8 * c);
                uint4 *out = const_cast<uint4 *>(isq ? (s_is_sum[r] ? a.qs : a.qt) : (s_is_sum[r] ? a.ks : a.kt));
                int64_t base_in = (src * H + h) * (a.d / 8);
                out[base_in + c] = lo;
                out[base_in + c + chunks_half] = hi;
                continue;
            }
            uint4 lo = make_uint4(0, 0, 0, 0), hi = lo;
            if (src >= 0) {
                const uint4 *in = isq ? (s_is_sum[r] ? a.qs : a.qt) : (s_is_sum[r] ? a.ks : a.kt);
                int64_t base_in = (src * H + h) * (a.d / 8);
                lo = in[base_in + c];
                hi = in[base_in + c + chunks_half];
                rope_rot8(lo, hi, cs + 8 * c, sn + 8 * c);
            }
            uint4 *out = isq ? a.qa : a.ka;
            out[base_out + c] = lo;
            out[base_out + c + chunks_half] = hi;
        } else {
            int j = it - qv - kv;
            int64_t o = R * (int64_t)a.Hkv * (a.d / 8) + j;
            if (BWD) {
                if (src < 0) continue;
                uint4 *out = const_cast<uint4 *>(s_is_sum[r] ? a.vs : a.vt);
                out[src * (int64_t)a.Hkv * (a.d / 8) + j] = a.va[o];
                continue;
            }
            uint4 val = make_uint4(0, 0, 0, 0);
            if (src >= 0) {
                const uint4 *in = s_is_sum[r] ? a.vs : a.vt;
                val = in[src * (int64_t)a.Hkv * (a.d / 8) + j];
            }
            a.va[o] = val;
        }
    }
}

int launch_interleave_rope(const ksa_params *p, int batch, const int32_t *cu, int64_t aug_rows,
                           const void *qt, const void *kt, const void *vt, const void *qs,
                           const void *ks, const void *vs, void *qa, void *ka, void *va,
                           const Plan &pl, int32_t *err, cudaStream_t st)
{
    if (aug_rows == 0) return KSA_OK;
    RopeArgs a;
    a.batch = batch; a.k = p->k; a.Hq = p->num_q_heads; a.Hkv = p->num_kv_heads; a.d = p->head_dim;
    a.aug_rows = aug_rows;
    a.rotate = p->rope_theta > 0.0;
    a.log2_theta = a.rotate ? log2(p->rope_theta) : 0.0;
    a.cu = cu; a.pl = pl; a.err = err;
    a.qt = (const uint4 *)qt; a.kt = (const uint4 *)kt; a.vt = (const uint4 *)vt;
    a.qs = (const uint4 *)qs; a.ks = (const uint4 *)ks; a.vs = (const uint4 *)vs;
    a.qa = (uint4 *)qa; a.ka = (uint4 *)ka; a.va = (uint4 *)va;
    int64_t blocks = (aug_rows + kRows - 1) / kRows;
    if (blocks > INT32_MAX) return KSA_ERR_UNSUPPORTED;
    interleave_rope_kernel<false><<<(unsigned)blocks, kRopeThreads, 0, st>>>(a);
    return cudaGetLastError() == cudaSuccess ? KSA_OK : KSA_ERR_CUDA;
}

int launch_interleave_rope_bwd(const ksa_params *p, int batch, const int32_t *cu, int64_t aug_rows,
                               const void *dqa, const void *dka, const void *dva, void *dqt, void *dkt, void *dvt,
                               void *dqs, void *dks, void *dvs, const Plan &pl, int32_t *err, cudaStream_t st)
{
    if (aug_rows == 0) return KSA_OK;
    RopeArgs a;
    a.batch = batch; a.k = p->k; a.Hq = p->num_q_heads; a.Hkv = p->num_kv_heads; a.d = p->head_dim;
    a.aug_rows = aug_rows;
    a.rotate = p->rope_theta > 0.0;
    a.log2_theta = a.rotate ? log2(p->rope_theta) : 0.0;
    a.cu = cu; a.pl = pl; a.err = err;
    a.qt = (const uint4 *)dqt; a.kt = (const uint4 *)dkt; a.vt = (const uint4 *)dvt;
    a.qs = (const uint4 *)dqs; a.ks = (const uint4 *)dks; a.vs = (const uint4 *)dvs;
    a.qa = (uint4 *)dqa; a.ka = (uint4 *)dka; a.va = (uint4 *)dva;
    int64_t blocks = (aug_rows + kRows - 1) / kRows;
    if (blocks > INT32_MAX) return KSA_ERR_UNSUPPORTED;
    interleave_rope_kernel<true><<<(unsigned)blocks, kRopeThreads, 0, st>>>(a);
    return cudaGetLastError() == cudaSuccess ? KSA_OK : KSA_ERR_CUDA;
}

}  // namespace ksa

// ksa_internal.cuh -- declarations shared by the .cu files of libksa.so.
//
// Kwai Summary Attention Technical Report: section 2.2 (the rule), section
// 2.3 (the block-sparse prefill kernel and the contiguous decode cache).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/ksa.h"

namespace ksa {

// Per-batch offsets derived on the device from cu_seqlens by plan_kernel and
// kept at the head of the prefill workspace.
struct Plan {
    int32_t *err;        // error word used when the caller passes none
    int32_t *chunk_off;  // [B+1] first chunk of each sequence (ceil(n/k) each)
    int32_t *sum_off;    // [B+1] first summary input row (floor(n/k) each)
    int32_t *tile_off;   // [B+1] first prefill work unit of each sequence
};

constexpr size_t kAlign = 256;
inline size_t align_up(size_t x, size_t a = kAlign) { return (x + a - 1) / a * a; }

// Workspace layout of the prefill calls.
inline size_t plan_bytes(int batch)
{
    return align_up(16) + 3 * align_up(sizeof(int32_t) * (size_t)(batch + 1));
}
inline Plan plan_view(void *ws, int batch)
{
    char *p = static_cast<char *>(ws);
    Plan pl;
    pl.err = reinterpret_cast<int32_t *>(p);
    p += align_up(16);
    size_t a = align_up(sizeof(int32_t) * (size_t)(batch + 1));
    pl.chunk_off = reinterpret_cast<int32_t *>(p); p += a;
    pl.sum_off = reinterpret_cast<int32_t *>(p); p += a;
    pl.tile_off = reinterpret_cast<int32_t *>(p);
    return pl;
}

// Chunks covered by one prefill work unit (all rows of a unit share one kv
// head); set by the prefill launcher, 0 for calls that need no tile list.
int prefill_unit_chunks(const ksa_params *p);
int prefill_heads_per_tile(const ksa_params *p);

// Enqueue the plan kernel: validates cu_seqlens against the host totals and
// fills the offsets.  unit_chunks > 0 also fills tile_off.
int launch_plan(const ksa_params *p, int batch, const int32_t *cu, int64_t total_text,
                int64_t total_sum, int64_t aug_rows, const Plan &pl, int32_t *err,
                int unit_chunks, cudaStream_t st);

int launch_interleave_rope(const ksa_params *p, int batch, const int32_t *cu, int64_t aug_rows,
                           const void *qt, const void *kt, const void *vt, const void *qs,
                           const void *ks, const void *vs, void *qa, void *ka, void *va,
                           const Plan &pl, int32_t *err, cudaStream_t st);

int launch_interleave_rope_bwd(const ksa_params *p, int batch, const int32_t *cu, int64_t aug_rows,
                               const void *dqa, const void *dka, const void *dva, void *dqt, void *dkt, void *dvt,
                               void *dqs, void *dks, void *dvs, const Plan &pl, int32_t *err, cudaStream_t st);

// Prefill backward (prefill_bwd.cu).
size_t prefill_bwd_workspace_bytes(const ksa_params *p, int batch, int64_t aug_rows);
int launch_prefill_bwd(const ksa_params *p, int batch, const int32_t *cu, int64_t total_text, int64_t aug_rows,
                       const void *q, const void *k, const void *v, const void *o, const float *lse, const void *dout,
                       void *dq, void *dk, void *dv, void *ws, const Plan &pl, int32_t *err, cudaStream_t st);

// Tensor-core backward of the text query rows (prefill_bwd_sm100.cu): dk, dv
// added into the fp32 accumulators dk32, dv32 ([aug_rows, Hkv, d], zeroed by
// the caller), dq of the text rows written as bf16; ws holds
// prefill_bwd_tc_workspace_bytes.
bool prefill_bwd_tc_supported(const ksa_params *p);
size_t prefill_bwd_tc_workspace_bytes(int batch, int64_t aug_rows);
int launch_prefill_bwd_tc(const ksa_params *p, int batch, const int32_t *cu, int64_t total_text, int64_t aug_rows,
                          const void *q, const void *k, const void *v, const void *dout, const float *lse,
                          const float *dsum, float *dk32, float *dv32, void *dq, void *ws, const Plan &pl,
                          int32_t *err, cudaStream_t st);

// Decode cache from the augmented K/V of a prefilled batch (cache_decode.cu).
int launch_cache_build(const ksa_params *p, const ksa_cache *c, const int32_t *cu, const void *k_aug,
                       const void *v_aug, const Plan &pl, int32_t *err, cudaStream_t st);

// The tensor-core prefill kernel in chunk mode: the text rows of a block of
// new tokens against a decode cache.  The caller (prefill_chunk.cu) gathers
// the block's rotated query rows and its window of text keys into augmented
// buffers ([chunks, k+1, H, d]) and fills the per-sequence arrays; summary
// key tiles are read from the cache's summary slots.
struct ChunkTiles {
    const int32_t *tile_off;   // [B+1] first work unit of each sequence
    const int32_t *cbeg;       // [B] first query chunk (absolute)
    const int32_t *ntot;       // [B] text tokens after the block
    const int32_t *qbase;      // [B] q/o buffer chunk of absolute chunk 0
    const int32_t *kvbase;     // [B] window buffer chunk of absolute chunk 0
    int64_t q_chunks, kv_chunks, max_units;
    const void *qa, *ka, *va;
    void *oa;
    float *lse;
};
int launch_prefill_cache(const ksa_params *p, const ksa_cache *c, const ChunkTiles &t, int32_t *err,
                         cudaStream_t st);

// Chunked prefill against a decode cache (prefill_chunk.cu).
size_t prefill_chunk_workspace_bytes(const ksa_params *p, int batch, int64_t total_text, int64_t total_sum);
int launch_prefill_chunk(const ksa_params *p, const ksa_cache *c, const int32_t *cu_t, int64_t total_t,
                         const int32_t *cu_s, int64_t total_s, const void *qt, const void *kt, const void *vt,
                         const void *qs, const void *ks, const void *vs, void *ot, void *os, float *lt, float *ls,
                         void *ws, int32_t *dev_err, cudaStream_t st);

// Decode over an MLA latent cache (mla_decode.cu).
size_t mla_decode_workspace_bytes(const ksa_mla_params *p, int batch, int64_t max_text);
int launch_mla_append(const ksa_mla_params *p, const ksa_mla_cache *c, const int8_t *kind, const void *x,
                      cudaStream_t st);
int launch_mla_decode(const ksa_mla_params *p, const ksa_mla_cache *c, const int8_t *kind, const void *q, void *o,
                      float *lse, int64_t max_text, void *ws, size_t ws_bytes, cudaStream_t st);

int launch_prefill(const ksa_params *p, int batch, const int32_t *cu, int64_t total_text,
                   int64_t aug_rows, const void *qa, const void *ka, const void *va, void *oa,
                   float *lse, const Plan &pl, int32_t *err, cudaStream_t st);

int launch_cache_append(const ksa_params *p, const ksa_cache *c, const int8_t *kind,
                        const void *k_new, const void *v_new, cudaStream_t st);

size_t decode_workspace_bytes(const ksa_params *p, int batch, int64_t max_text);
// Split-K shape of the decode: the split count it chooses for a batch and
// max_text, and the bytes of partials (m, l, acc) one split needs.
int decode_splits(const ksa_params *p, int batch, int64_t max_text);
size_t decode_split_bytes(const ksa_params *p, int batch);
int launch_decode(const ksa_params *p, const ksa_cache *c, const int8_t *kind, const void *q,
                  void *o, float *lse, int64_t max_text, void *ws, size_t ws_bytes,
                  cudaStream_t st);
// The same decode with an explicit split count; ws holds nsplit splits.
int launch_decode_splits(const ksa_params *p, const ksa_cache *c, const int8_t *kind, const void *q, void *o,
                         float *lse, int nsplit, void *ws, cudaStream_t st);
// The argument checks of ksa_decode (everything but the workspace).
int check_decode_args(const ksa_params *p, const ksa_cache *cache, const int8_t *kind, const void *q,
                      const void *o, const float *lse, int64_t max_text);

// Number of SMs of the current device (cached per device).
int sm_count();

// Record the first error only.
__device__ __forceinline__ void set_error(int32_t *err, int code)
{
    if (err) atomicCAS(err, 0, code);
}

// RoPE angle of pair r (of d/2) at position pos, reduced to [-pi, pi] in
// fp64 so that positions up to millions keep full fp32 accuracy in sincos.
__device__ __forceinline__ void rope_cos_sin(double pos, int r, int d, double log2_theta,
                                             float *c, float *s)
{
    // inv_freq = theta^(-2r/d)
    double inv_freq = exp2(-2.0 * (double)r / (double)d * log2_theta);
    double ang = pos * inv_freq;
    const double two_pi = 6.283185307179586476925286766559;
    ang = ang - two_pi * rint(ang / two_pi);
    double sd, cd;
    sincos(ang, &sd, &cd);
    *c = (float)cd;
    *s = (float)sd;
}

// Rotate-half RoPE of 8 pairs: lo holds x_r .. x_{r+7}, hi holds
// x_{r+d/2} .. x_{r+d/2+7} (bf16); cs / sn the pairs' cos / sin.  fp32
// arithmetic, bf16 round-to-nearest-even.  Every kernel that rotates keys
// uses this one routine, so keys rotated by different calls are identical.
__device__ __forceinline__ void rope_rot8(uint4 &lo, uint4 &hi, const float *cs, const float *sn)
{
    __nv_bfloat162 *a = reinterpret_cast<__nv_bfloat162 *>(&lo);
    __nv_bfloat162 *b = reinterpret_cast<__nv_bfloat162 *>(&hi);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        float2 x = __bfloat1622float2(a[e]);
        float2 y = __bfloat1622float2(b[e]);
        float c0 = cs[2 * e], c1 = cs[2 * e + 1], s0 = sn[2 * e], s1 = sn[2 * e + 1];
        float2 xo = make_float2(x.x * c0 - y.x * s0, x.y * c1 - y.y * s1);
        float2 yo = make_float2(y.x * c0 + x.x * s0, y.y * c1 + x.y * s1);
        a[e] = __float22bfloat162_rn(xo);
        b[e] = __float22bfloat162_rn(yo);
    }
}

// Slice of one sequence after its append: [lo, hi) in slots.  Returns false
// if the state cannot hold a query of this kind (the caller records the error).
// Host-callable too, for CPU tests against a reference cache.
__host__ __device__ __forceinline__ bool decode_slice(int kind, int64_t n, int64_t m, int k, int w,
                                             int64_t *lo, int64_t *hi)
{
    if (n < 0 || m < 0) return false;   // no sequence of appends reaches it
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

// (j + w + 1) k clamped to n: the first text position that sees summary j,
// which is also one past the last text query that sees the text keys of
// chunk j.  Taken in 64 bits: on a sequence of close to 2^31 tokens the
// 32-bit product would pass INT32_MAX (w + 1) k alone may be 2^30.
__host__ __device__ __forceinline__ int window_end(int64_t j, int w, int k, int n)
{
    const int64_t e = (j + w + 1) * (int64_t)k;
    return e < n ? (int)e : n;
}

}  // namespace ksa

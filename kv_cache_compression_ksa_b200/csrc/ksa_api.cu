// ksa_api.cu -- the extern "C" entry points of libksa.so: argument checks on
// the host, then the kernels of rope_interleave.cu, prefill_sm100.cu and
// cache_decode.cu.  Nothing here allocates device or host memory.
#include <math.h>
#include <string.h>

#include "ksa_internal.cuh"

namespace ksa {

int sm_count()
{
    static int cached[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (dev < 0 || dev >= 64) return 148;
    if (!cached[dev]) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cached[dev] = n;
    }
    return cached[dev];
}

static bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Shape checks shared by every call.
// The window the kernels index in 32-bit arithmetic: (w + 1) k text tokens.
// A larger w (e.g. INT32_MAX for "every chunk") is refused, not wrapped;
// w = the chunk count of the longest sequence gives full attention.
constexpr int64_t kMaxWindowTokens = 1LL << 30;

static bool window_fits(int k, int w) { return ((int64_t)w + 1) * (int64_t)k <= kMaxWindowTokens; }

static int check_params(const ksa_params *p)
{
    if (!p) return KSA_ERR_INVALID;
    if (p->k < 1 || p->w < 0 || p->num_q_heads < 1 || p->num_kv_heads < 1) return KSA_ERR_INVALID;
    if (!window_fits(p->k, p->w)) return KSA_ERR_UNSUPPORTED;
    if (p->num_q_heads % p->num_kv_heads != 0) return KSA_ERR_INVALID;
    if (!(p->scale >= 0.f) || isinf(p->scale)) return KSA_ERR_INVALID;
    if (isnan(p->rope_theta)) return KSA_ERR_INVALID;
    if (p->head_dim != 64 && p->head_dim != 128) return KSA_ERR_UNSUPPORTED;
    if (p->num_q_heads / p->num_kv_heads > 8) return KSA_ERR_UNSUPPORTED;
    return KSA_OK;
}

static int check_prefill_shape(const ksa_params *p)
{
    // query tiles hold min(G, 128/k) heads of k slots; G must split evenly
    if (prefill_heads_per_tile(p) < 1) return KSA_ERR_UNSUPPORTED;
    const int G = p->num_q_heads / p->num_kv_heads;
    if (G != 1 && G != 2 && G != 4 && G != 8) return KSA_ERR_UNSUPPORTED;   // summary-row kernel
    return KSA_OK;
}

static int check_mla(const ksa_mla_params *p, const ksa_mla_cache *c, const int8_t *kind)
{
    if (!p || !c) return KSA_ERR_INVALID;
    if (p->k < 1 || p->w < 0 || p->num_heads < 1 || p->kv_lora_rank < 1 || p->rope_dim < 0) return KSA_ERR_INVALID;
    if (!window_fits(p->k, p->w)) return KSA_ERR_UNSUPPORTED;
    if (!(p->scale >= 0.f) || isinf(p->scale) || isnan(p->rope_theta)) return KSA_ERR_INVALID;
    if (p->kv_lora_rank != 512 || p->rope_dim != 64) return KSA_ERR_UNSUPPORTED;
    if (c->batch < 0 || c->cap_summaries < 0) return KSA_ERR_INVALID;
    if (c->batch > 0 && (!c->latent || !c->state || !kind || !aligned16(c->latent))) return KSA_ERR_INVALID;
    if (c->batch > 65535) return KSA_ERR_UNSUPPORTED;
    if ((c->cap_summaries + 1) * (int64_t)p->k > INT32_MAX) return KSA_ERR_UNSUPPORTED;
    return KSA_OK;
}

}  // namespace ksa

using namespace ksa;

extern "C" {

const char *ksa_status_string(int s)
{
    switch (s) {
    case KSA_OK: return "ok";
    case KSA_ERR_INVALID: return "invalid argument";
    case KSA_ERR_UNSUPPORTED: return "unsupported shape";
    case KSA_ERR_CAPACITY: return "capacity exceeded";
    case KSA_ERR_CUDA: return "CUDA error";
    case KSA_ERR_TIMEOUT: return "device wait timed out";
    case KSA_ERR_WORKSPACE: return "workspace too small";
    case KSA_ERR_STATE: return "decode cache order violated";
    default: return "unknown status";
    }
}

int64_t ksa_aug_rows(const ksa_params *p, int32_t batch, const int32_t *seqlens_host)
{
    if (check_params(p) != KSA_OK || batch < 0 || (batch > 0 && !seqlens_host)) return -1;
    int64_t chunks = 0;
    for (int b = 0; b < batch; ++b) {
        if (seqlens_host[b] < 0) return -1;
        chunks += ((int64_t)seqlens_host[b] + p->k - 1) / p->k;
    }
    return chunks * (p->k + 1);
}

size_t ksa_prefill_workspace_size(const ksa_params *p, int32_t batch, int64_t total_text)
{
    (void)p; (void)total_text;
    if (batch < 0) return 0;
    return plan_bytes(batch);
}

static int check_prefill_common(const ksa_params *p, int32_t batch, const int32_t *cu, int64_t total_text,
                                int64_t aug_rows, void *ws, size_t ws_bytes)
{
    int rc = check_params(p);
    if (rc != KSA_OK) return rc;
    if (batch < 1 || !cu || total_text < 0 || aug_rows < 0 || aug_rows % (p->k + 1) != 0) return KSA_ERR_INVALID;
    if (total_text > INT32_MAX || aug_rows / (p->k + 1) > INT32_MAX) return KSA_ERR_UNSUPPORTED;
    if (aug_rows < total_text) return KSA_ERR_INVALID;
    if (!ws) return KSA_ERR_INVALID;
    if (ws_bytes < plan_bytes(batch)) return KSA_ERR_WORKSPACE;
    if (!aligned16(ws)) return KSA_ERR_INVALID;
    return KSA_OK;
}

int ksa_interleave_rope(const ksa_params *p, int32_t batch, const int32_t *cu_seqlens, int64_t total_text,
                        int64_t total_sum, int64_t aug_rows, const void *q_text, const void *k_text,
                        const void *v_text, const void *q_sum, const void *k_sum, const void *v_sum, void *q_aug,
                        void *k_aug, void *v_aug, void *workspace, size_t workspace_bytes, int32_t *dev_err,
                        void *stream)
{
    int rc = check_prefill_common(p, batch, cu_seqlens, total_text, aug_rows, workspace, workspace_bytes);
    if (rc != KSA_OK) return rc;
    if (total_sum < 0 || total_sum > total_text / p->k) return KSA_ERR_INVALID;
    if (total_text > 0 && (!q_text || !k_text || !v_text)) return KSA_ERR_INVALID;
    if (total_sum > 0 && (!q_sum || !k_sum || !v_sum)) return KSA_ERR_INVALID;
    if (aug_rows > 0 && (!q_aug || !k_aug || !v_aug)) return KSA_ERR_INVALID;
    const void *ptrs[] = {q_text, k_text, v_text, q_sum, k_sum, v_sum, q_aug, k_aug, v_aug};
    for (const void *q : ptrs)
        if (q && !aligned16(q)) return KSA_ERR_INVALID;
    if (reinterpret_cast<uintptr_t>(dev_err) & 3u) return KSA_ERR_INVALID;
    cudaStream_t st = (cudaStream_t)stream;
    Plan pl = plan_view(workspace, batch);
    int32_t *err = dev_err ? dev_err : pl.err;
    rc = launch_plan(p, batch, cu_seqlens, total_text, total_sum, aug_rows, pl, err, 0, st);
    if (rc != KSA_OK) return rc;
    return launch_interleave_rope(p, batch, cu_seqlens, aug_rows, q_text, k_text, v_text, q_sum, k_sum, v_sum,
                                  q_aug, k_aug, v_aug, pl, err, st);
}

int ksa_interleave_rope_bwd(const ksa_params *p, int32_t batch, const int32_t *cu_seqlens, int64_t total_text,
                            int64_t total_sum, int64_t aug_rows, const void *dq_aug, const void *dk_aug,
                            const void *dv_aug, void *dq_text, void *dk_text, void *dv_text, void *dq_sum,
                            void *dk_sum, void *dv_sum, void *workspace, size_t workspace_bytes, int32_t *dev_err,
                            void *stream)
{
    int rc = check_prefill_common(p, batch, cu_seqlens, total_text, aug_rows, workspace, workspace_bytes);
    if (rc != KSA_OK) return rc;
    if (total_sum < 0 || total_sum > total_text / p->k) return KSA_ERR_INVALID;
    if (total_text > 0 && (!dq_text || !dk_text || !dv_text)) return KSA_ERR_INVALID;
    if (total_sum > 0 && (!dq_sum || !dk_sum || !dv_sum)) return KSA_ERR_INVALID;
    if (aug_rows > 0 && (!dq_aug || !dk_aug || !dv_aug)) return KSA_ERR_INVALID;
    const void *ptrs[] = {dq_text, dk_text, dv_text, dq_sum, dk_sum, dv_sum, dq_aug, dk_aug, dv_aug};
    for (const void *q : ptrs)
        if (q && !aligned16(q)) return KSA_ERR_INVALID;
    if (reinterpret_cast<uintptr_t>(dev_err) & 3u) return KSA_ERR_INVALID;
    cudaStream_t st = (cudaStream_t)stream;
    Plan pl = plan_view(workspace, batch);
    int32_t *err = dev_err ? dev_err : pl.err;
    rc = launch_plan(p, batch, cu_seqlens, total_text, total_sum, aug_rows, pl, err, 0, st);
    if (rc != KSA_OK) return rc;
    return launch_interleave_rope_bwd(p, batch, cu_seqlens, aug_rows, dq_aug, dk_aug, dv_aug, dq_text, dk_text,
                                      dv_text, dq_sum, dk_sum, dv_sum, pl, err, st);
}

int ksa_prefill_fwd(const ksa_params *p, int32_t batch, const int32_t *cu_seqlens, int64_t total_text,
                    int64_t aug_rows, const void *q_aug, const void *k_aug, const void *v_aug, void *o_aug,
                    float *lse, void *workspace, size_t workspace_bytes, int32_t *dev_err, void *stream)
{
    int rc = check_prefill_common(p, batch, cu_seqlens, total_text, aug_rows, workspace, workspace_bytes);
    if (rc != KSA_OK) return rc;
    rc = check_prefill_shape(p);
    if (rc != KSA_OK) return rc;
    if (aug_rows > 0 && (!q_aug || !k_aug || !v_aug || !o_aug)) return KSA_ERR_INVALID;
    const void *ptrs[] = {q_aug, k_aug, v_aug, o_aug};
    for (const void *q : ptrs)
        if (q && !aligned16(q)) return KSA_ERR_INVALID;
    if ((reinterpret_cast<uintptr_t>(lse) & 3u) || (reinterpret_cast<uintptr_t>(dev_err) & 3u))
        return KSA_ERR_INVALID;
    cudaStream_t st = (cudaStream_t)stream;
    Plan pl = plan_view(workspace, batch);
    int32_t *err = dev_err ? dev_err : pl.err;
    // the summary count is implied by cu_seqlens here: -1 skips that check
    rc = launch_plan(p, batch, cu_seqlens, total_text, -1, aug_rows, pl, err, prefill_unit_chunks(p), st);
    if (rc != KSA_OK) return rc;
    return launch_prefill(p, batch, cu_seqlens, total_text, aug_rows, q_aug, k_aug, v_aug, o_aug, lse, pl, err, st);
}

size_t ksa_prefill_bwd_workspace_size(const ksa_params *p, int32_t batch, int64_t aug_rows)
{
    if (check_params(p) != KSA_OK || batch < 0 || aug_rows < 0) return 0;
    return prefill_bwd_workspace_bytes(p, batch, aug_rows);
}

int ksa_prefill_bwd(const ksa_params *p, int32_t batch, const int32_t *cu_seqlens, int64_t total_text,
                    int64_t aug_rows, const void *q_aug, const void *k_aug, const void *v_aug, const void *o_aug,
                    const float *lse, const void *do_aug, void *dq_aug, void *dk_aug, void *dv_aug, void *workspace,
                    size_t workspace_bytes, int32_t *dev_err, void *stream)
{
    int rc = check_prefill_common(p, batch, cu_seqlens, total_text, aug_rows, workspace, workspace_bytes);
    if (rc != KSA_OK) return rc;
    if (workspace_bytes < prefill_bwd_workspace_bytes(p, batch, aug_rows)) return KSA_ERR_WORKSPACE;
    if (aug_rows > 0) {
        const void *ptrs[] = {q_aug, k_aug, v_aug, o_aug, do_aug, dq_aug, dk_aug, dv_aug};
        for (const void *x : ptrs)
            if (!x || !aligned16(x)) return KSA_ERR_INVALID;
        if (!lse || (reinterpret_cast<uintptr_t>(lse) & 3u)) return KSA_ERR_INVALID;
    }
    if (reinterpret_cast<uintptr_t>(dev_err) & 3u) return KSA_ERR_INVALID;
    cudaStream_t st = (cudaStream_t)stream;
    Plan pl = plan_view(workspace, batch);
    int32_t *err = dev_err ? dev_err : pl.err;
    rc = launch_plan(p, batch, cu_seqlens, total_text, -1, aug_rows, pl, err, 0, st);
    if (rc != KSA_OK) return rc;
    return launch_prefill_bwd(p, batch, cu_seqlens, total_text, aug_rows, q_aug, k_aug, v_aug, o_aug, lse, do_aug,
                              dq_aug, dk_aug, dv_aug, workspace, pl, err, st);
}

int64_t ksa_cache_slots(const ksa_params *p, int64_t cap_summaries)
{
    if (!p || p->k < 1 || p->w < 0 || cap_summaries < 0) return -1;
    return 1 + (int64_t)p->k + (int64_t)p->w * p->k + cap_summaries;
}

static int check_cache(const ksa_params *p, const ksa_cache *c, const int8_t *kind)
{
    int rc = check_params(p);
    if (rc != KSA_OK) return rc;
    if (!c || c->batch < 0 || c->cap_summaries < 0) return KSA_ERR_INVALID;
    if (c->batch > 0 && (!c->k || !c->v || !c->state || !kind)) return KSA_ERR_INVALID;
    if (c->batch > 0 && (!aligned16(c->k) || !aligned16(c->v))) return KSA_ERR_INVALID;
    if (c->batch > 65535) return KSA_ERR_UNSUPPORTED;
    // int32 state: text positions must stay representable
    if ((c->cap_summaries + 1) * (int64_t)p->k > INT32_MAX) return KSA_ERR_UNSUPPORTED;
    return KSA_OK;
}

int ksa_cache_append(const ksa_params *p, const ksa_cache *cache, const int8_t *kind, const void *k_new,
                     const void *v_new, void *stream)
{
    int rc = check_cache(p, cache, kind);
    if (rc != KSA_OK) return rc;
    if (cache->batch > 0 && (!k_new || !v_new || !aligned16(k_new) || !aligned16(v_new))) return KSA_ERR_INVALID;
    return launch_cache_append(p, cache, kind, k_new, v_new, (cudaStream_t)stream);
}

int ksa_cache_from_prefill(const ksa_params *p, const ksa_cache *cache, const int32_t *cu_seqlens,
                           int64_t total_text, int64_t aug_rows, const void *k_aug, const void *v_aug,
                           void *workspace, size_t workspace_bytes, int32_t *dev_err, void *stream)
{
    int rc = check_params(p);
    if (rc != KSA_OK) return rc;
    if (!cache || cache->batch < 0 || cache->cap_summaries < 0) return KSA_ERR_INVALID;
    if (cache->batch == 0) return KSA_OK;
    if (!cache->k || !cache->v || !cache->state || !aligned16(cache->k) || !aligned16(cache->v)) return KSA_ERR_INVALID;
    if (cache->batch > 65535) return KSA_ERR_UNSUPPORTED;
    if ((cache->cap_summaries + 1) * (int64_t)p->k > INT32_MAX) return KSA_ERR_UNSUPPORTED;
    rc = check_prefill_common(p, cache->batch, cu_seqlens, total_text, aug_rows, workspace, workspace_bytes);
    if (rc != KSA_OK) return rc;
    if (aug_rows > 0 && (!k_aug || !v_aug || !aligned16(k_aug) || !aligned16(v_aug))) return KSA_ERR_INVALID;
    if (reinterpret_cast<uintptr_t>(dev_err) & 3u) return KSA_ERR_INVALID;
    cudaStream_t st = (cudaStream_t)stream;
    Plan pl = plan_view(workspace, cache->batch);
    int32_t *err = dev_err ? dev_err : pl.err;
    rc = launch_plan(p, cache->batch, cu_seqlens, total_text, -1, aug_rows, pl, err, 0, st);
    if (rc != KSA_OK) return rc;
    return launch_cache_build(p, cache, cu_seqlens, k_aug, v_aug, pl, err, st);
}

size_t ksa_prefill_chunk_workspace_size(const ksa_params *p, int32_t batch, int64_t total_text, int64_t total_sum)
{
    if (check_params(p) != KSA_OK || batch < 0 || total_text < 0 || total_sum < 0) return 0;
    return prefill_chunk_workspace_bytes(p, batch, total_text, total_sum);
}

int ksa_prefill_chunk(const ksa_params *p, const ksa_cache *cache, const int32_t *cu_text, int64_t total_text,
                      const int32_t *cu_sum, int64_t total_sum, const void *q_text, const void *k_text,
                      const void *v_text, const void *q_sum, const void *k_sum, const void *v_sum, void *o_text,
                      void *o_sum, float *lse_text, float *lse_sum, void *workspace, size_t workspace_bytes,
                      int32_t *dev_err, void *stream)
{
    int rc = check_params(p);
    if (rc != KSA_OK) return rc;
    if (!cache || cache->batch < 0 || cache->cap_summaries < 0) return KSA_ERR_INVALID;
    if (total_text < 0 || total_sum < 0) return KSA_ERR_INVALID;
    if (total_text > INT32_MAX || total_sum > INT32_MAX) return KSA_ERR_UNSUPPORTED;
    if (cache->batch == 0) return KSA_OK;
    if (!cache->k || !cache->v || !cache->state || !aligned16(cache->k) || !aligned16(cache->v)) return KSA_ERR_INVALID;
    if (cache->batch > 65535) return KSA_ERR_UNSUPPORTED;
    if ((cache->cap_summaries + 1) * (int64_t)p->k > INT32_MAX) return KSA_ERR_UNSUPPORTED;
    if (!cu_text || !cu_sum || !workspace || !aligned16(workspace)) return KSA_ERR_INVALID;
    const void *need_t[] = {q_text, k_text, v_text, o_text};
    const void *need_s[] = {q_sum, k_sum, v_sum, o_sum};
    for (const void *x : need_t)
        if (total_text > 0 && (!x || !aligned16(x))) return KSA_ERR_INVALID;
    for (const void *x : need_s)
        if (total_sum > 0 && (!x || !aligned16(x))) return KSA_ERR_INVALID;
    if ((reinterpret_cast<uintptr_t>(lse_text) & 3u) || (reinterpret_cast<uintptr_t>(lse_sum) & 3u) ||
        (reinterpret_cast<uintptr_t>(dev_err) & 3u))
        return KSA_ERR_INVALID;
    if (workspace_bytes < prefill_chunk_workspace_bytes(p, cache->batch, total_text, total_sum))
        return KSA_ERR_WORKSPACE;
    return launch_prefill_chunk(p, cache, cu_text, total_text, cu_sum, total_sum, q_text, k_text, v_text, q_sum,
                                k_sum, v_sum, o_text, o_sum, lse_text, lse_sum, workspace, dev_err,
                                (cudaStream_t)stream);
}

size_t ksa_decode_workspace_size(const ksa_params *p, int32_t batch, int64_t max_text)
{
    if (check_params(p) != KSA_OK || batch < 0 || max_text < 0) return 0;
    return decode_workspace_bytes(p, batch, max_text);
}

}  // extern "C"

namespace ksa {
int check_decode_args(const ksa_params *p, const ksa_cache *cache, const int8_t *kind, const void *q,
                      const void *o, const float *lse, int64_t max_text)
{
    int rc = check_cache(p, cache, kind);
    if (rc != KSA_OK) return rc;
    if (max_text < 0) return KSA_ERR_INVALID;
    if (cache->batch > 0) {
        if (!q || !o || !aligned16(q) || !aligned16(o)) return KSA_ERR_INVALID;
        if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return KSA_ERR_INVALID;
    }
    return KSA_OK;
}
}  // namespace ksa

extern "C" {

int ksa_decode(const ksa_params *p, const ksa_cache *cache, const int8_t *kind, const void *q, void *o, float *lse,
               int64_t max_text, void *workspace, size_t workspace_bytes, void *stream)
{
    int rc = check_decode_args(p, cache, kind, q, o, lse, max_text);
    if (rc != KSA_OK) return rc;
    if (cache->batch > 0 && (!workspace || !aligned16(workspace))) return KSA_ERR_INVALID;
    return launch_decode(p, cache, kind, q, o, lse, max_text, workspace, workspace_bytes, (cudaStream_t)stream);
}

int64_t ksa_mla_cache_slots(const ksa_mla_params *p, int64_t cap_summaries)
{
    if (!p || p->k < 1 || p->w < 0 || cap_summaries < 0) return -1;
    return 1 + (int64_t)p->k + (int64_t)p->w * p->k + cap_summaries;
}

int ksa_mla_cache_append(const ksa_mla_params *p, const ksa_mla_cache *cache, const int8_t *kind, const void *x,
                         void *stream)
{
    int rc = check_mla(p, cache, kind);
    if (rc != KSA_OK) return rc;
    if (cache->batch > 0 && (!x || !aligned16(x))) return KSA_ERR_INVALID;
    return launch_mla_append(p, cache, kind, x, (cudaStream_t)stream);
}

size_t ksa_mla_decode_workspace_size(const ksa_mla_params *p, int32_t batch, int64_t max_text)
{
    if (!p || p->k < 1 || p->w < 0 || p->num_heads < 1 || batch < 0 || max_text < 0) return 0;
    if (!window_fits(p->k, p->w) || p->kv_lora_rank != 512 || p->rope_dim != 64) return 0;
    return mla_decode_workspace_bytes(p, batch, max_text);
}

int ksa_mla_decode(const ksa_mla_params *p, const ksa_mla_cache *cache, const int8_t *kind, const void *q, void *o,
                   float *lse, int64_t max_text, void *workspace, size_t workspace_bytes, void *stream)
{
    int rc = check_mla(p, cache, kind);
    if (rc != KSA_OK) return rc;
    if (max_text < 0) return KSA_ERR_INVALID;
    if (cache->batch > 0) {
        if (!q || !o || !workspace || !aligned16(q) || !aligned16(o) || !aligned16(workspace)) return KSA_ERR_INVALID;
        if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return KSA_ERR_INVALID;
    }
    return launch_mla_decode(p, cache, kind, q, o, lse, max_text, workspace, workspace_bytes, (cudaStream_t)stream);
}

int ksa_get_device_error(int32_t *dev_err, void *stream)
{
    if (!dev_err) return KSA_ERR_INVALID;
    cudaStream_t st = (cudaStream_t)stream;
    int32_t v = 0;
    if (cudaMemcpyAsync(&v, dev_err, sizeof(v), cudaMemcpyDeviceToHost, st) != cudaSuccess) return KSA_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return KSA_ERR_CUDA;
    if (v != KSA_OK) {
        if (cudaMemsetAsync(dev_err, 0, sizeof(int32_t), st) != cudaSuccess) return KSA_ERR_CUDA;
        if (cudaStreamSynchronize(st) != cudaSuccess) return KSA_ERR_CUDA;
    }
    return v;
}

}  // extern "C"

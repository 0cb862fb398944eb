/*
 * ksa.h -- C ABI of the B200 (sm_100a) Kwai Summary Attention hot path.
 *
 * What is computed ("Kwai Summary Attention Technical Report"):
 *   - the augmented sequence: after every k text tokens comes one summary
 *     token s_j (section 2.2.1, Eq. (1));
 *   - a summary token attends to the k text tokens of its own chunk and to
 *     itself; its RoPE position is that of its chunk's last text token
 *     (section 2.2.1, rules after Eq. (1); Figure 4c for the self key);
 *   - a text token t_i attends causally to the text of chunks
 *     floor(i/k)-w .. floor(i/k) (Sliding Chunk Attention, Eq. (2)) and to
 *     the summaries s_0 .. s_{floor(i/k)-w-1} of the chunks that have left
 *     that window (Eq. (3)); in-window summaries are not attended
 *     (section 2.2.2);
 *   - softmax(Q K^T * scale + M_KSA) V with scale = 1/sqrt(d) (Eq. (10));
 *   - decode reads one contiguous slice of a cache made of a scratch slot,
 *     the current chunk (filled right to left), a ring of w sliding chunks
 *     and an append-only summary buffer (section 2.3.1, Figure 4 (a)-(e)).
 *
 * Conventions for every entry point:
 *   - Tensor pointers are DEVICE pointers owned by the caller, row-major and
 *     contiguous; "bf16" is IEEE bfloat16 (2 bytes).  Base pointers must be
 *     16-byte aligned.
 *   - The library allocates no device or host memory and never synchronises
 *     the stream inside a compute call; all work is enqueued on `stream`
 *     (cudaStream_t passed as void*, NULL = legacy default stream).
 *   - Errors found on the host (bad sizes, null pointers, small workspace,
 *     unsupported shapes) are returned before anything is launched.  Errors
 *     found on the device (inconsistent cu_seqlens, cache order violations,
 *     a full summary buffer, a pipeline wait that ran out) never trap: the
 *     kernel records a KSA_ERR_* code in a device error word and skips the
 *     affected work.  ksa_get_device_error() reads and clears such a word.
 *   - Supported: head_dim 64 or 128; num_q_heads % num_kv_heads == 0 with
 *     at most 8 q heads per kv head; k >= 1; w >= 0; for prefill k <= 128
 *     and 1, 2, 4 or 8 q heads per kv head (when (q heads per kv head) * k
 *     exceeds 128 rows, a kv head's q heads are split over several query
 *     tiles, each reading the same key/value tiles).
 */
#ifndef KSA_H
#define KSA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KSA_API __attribute__((visibility("default")))
#else
#define KSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Shape and method parameters shared by all calls. */
typedef struct ksa_params {
    int32_t k;            /* chunk size: text tokens per chunk (>= 1)           */
    int32_t w;            /* sliding chunk number C of Eqs. (2)-(3) (>= 0;      *
                           * (w+1)*k <= 2^30, else KSA_ERR_UNSUPPORTED)        */
    int32_t num_q_heads;  /* Hq                                                 */
    int32_t num_kv_heads; /* Hkv; q head h reads kv head h / (Hq/Hkv)           */
    int32_t head_dim;     /* d: 64 or 128                                       */
    float scale;          /* softmax scale; 0 selects 1/sqrt(d) (Eq. (10))      */
    double rope_theta;    /* RoPE base (Table 3 uses 1e6); <= 0 disables RoPE   */
} ksa_params;

/* Status codes. */
enum {
    KSA_OK = 0,
    KSA_ERR_INVALID = -1,     /* bad argument (null pointer, negative size ...)  */
    KSA_ERR_UNSUPPORTED = -2, /* valid but not implemented (e.g. head_dim 96)   */
    KSA_ERR_CAPACITY = -3,    /* summary buffer full / output too small          */
    KSA_ERR_CUDA = -4,        /* a CUDA runtime or driver call failed            */
    KSA_ERR_TIMEOUT = -5,     /* a bounded device-side wait gave up              */
    KSA_ERR_WORKSPACE = -6,   /* workspace smaller than the *_workspace_size()   */
    KSA_ERR_STATE = -7        /* decode-cache order violated (see ksa_cache_append) */
};

/* Per-sequence step kinds for the decode calls. */
enum { KSA_TEXT = 0, KSA_SUMMARY = 1, KSA_SKIP = 2 };

/* ------------------------------------------------------------------------
 * Augmented layout (prefill).
 *
 * Each sequence b (n_b text tokens, cu_seqlens[b+1]-cu_seqlens[b]) owns
 * nc_b = ceil(n_b / k) whole chunks of k+1 rows, in the order of Eq. (1):
 * rows k*... t_{jk} .. t_{jk+k-1}, s_j.  Sequence b starts at row
 * (k+1) * sum_{b'<b} nc_{b'}.  A trailing partial chunk (n_b % k != 0) has
 * no summary (the report assumes k | n); its unused text rows and its
 * summary row are padding, written as zeros by ksa_interleave_rope and left
 * unspecified in the attention output.  Total rows = ksa_aug_rows().
 * Summary inputs are packed per sequence: sequence b contributes
 * floor(n_b / k) summary rows.
 * ------------------------------------------------------------------------ */

/* Rows of the augmented layout for host-side sequence lengths
 * seqlens_host[0 .. batch-1].  Returns -1 on invalid input. */
KSA_API int64_t ksa_aug_rows(const ksa_params *p, int32_t batch, const int32_t *seqlens_host);

/* Workspace bytes needed by ksa_interleave_rope / ksa_prefill_fwd for a
 * batch of `batch` sequences (holds the per-sequence offsets and the tile
 * list the kernels derive from cu_seqlens on the device). */
KSA_API size_t ksa_prefill_workspace_size(const ksa_params *p, int32_t batch, int64_t total_text);

/* RoPE + interleave (Eq. (1); RoPE positions of section 2.2.1).
 *
 * q_text [total_text, Hq, d], k_text/v_text [total_text, Hkv, d]: bf16 text
 *   projections, packed by sequence along cu_seqlens (device int32 [batch+1],
 *   cu_seqlens[0] = 0, non-decreasing, cu_seqlens[batch] = total_text).
 * q_sum [total_sum, Hq, d], k_sum/v_sum [total_sum, Hkv, d]: bf16 summary
 *   projections, total_sum = sum_b floor(n_b / k), packed the same way.
 * q_aug [aug_rows, Hq, d], k_aug/v_aug [aug_rows, Hkv, d]: bf16 outputs in
 *   the augmented layout; aug_rows = ksa_aug_rows(...).
 * Q and K of text t_i are rotated at position i (local to its sequence),
 * those of s_j at position jk+k-1 (rotate-half pairs (r, r+d/2), angle
 * pos * theta^(-2r/d), computed in fp64); V is copied.  Padding rows are
 * zeroed.  dev_err: device int32 error word (may be NULL: the workspace's
 * own word is used).  An inconsistent cu_seqlens sets KSA_ERR_INVALID there
 * and writes nothing. */
KSA_API int ksa_interleave_rope(const ksa_params *p, int32_t batch, const int32_t *cu_seqlens,
                        int64_t total_text, int64_t total_sum, int64_t aug_rows,
                        const void *q_text, const void *k_text, const void *v_text,
                        const void *q_sum, const void *k_sum, const void *v_sum,
                        void *q_aug, void *k_aug, void *v_aug,
                        void *workspace, size_t workspace_bytes, int32_t *dev_err,
                        void *stream);

/* Backward of ksa_interleave_rope: from the gradients of the augmented rows
 * (dq_aug [aug_rows, Hq, d], dk_aug / dv_aug [aug_rows, Hkv, d], e.g. from
 * ksa_prefill_bwd) to the gradients of the text and summary projections,
 * laid out as the forward's inputs (dq_text [total_text, Hq, d] ...,
 * dq_sum [total_sum, Hq, d] ...).  The rotation is orthogonal: q and k
 * gradients are rotated by the opposite angle at the same positions; v
 * gradients are copied.  Padding rows are ignored.  Arguments otherwise as
 * for ksa_interleave_rope. */
KSA_API int ksa_interleave_rope_bwd(const ksa_params *p, int32_t batch, const int32_t *cu_seqlens,
                            int64_t total_text, int64_t total_sum, int64_t aug_rows,
                            const void *dq_aug, const void *dk_aug, const void *dv_aug,
                            void *dq_text, void *dk_text, void *dv_text,
                            void *dq_sum, void *dk_sum, void *dv_sum,
                            void *workspace, size_t workspace_bytes, int32_t *dev_err, void *stream);

/* KSA prefill forward (Eqs. (2), (3), (10); block-sparse kernel of
 * section 2.3).  q_aug/k_aug/v_aug: the augmented layout (bf16, rotated).
 * o_aug [aug_rows, Hq, d] bf16: attention output of every real row (text
 * and summary); lse [aug_rows, Hq] fp32 natural-log sum of exp of the
 * scaled scores, or NULL to skip it.  Padding rows of o_aug/lse are not
 * written.  Text rows run on the tcgen05 tensor cores, skipping every key
 * tile the rule masks out entirely; summary rows (k+1 keys each) run on
 * CUDA cores. */
KSA_API int ksa_prefill_fwd(const ksa_params *p, int32_t batch, const int32_t *cu_seqlens,
                    int64_t total_text, int64_t aug_rows,
                    const void *q_aug, const void *k_aug, const void *v_aug,
                    void *o_aug, float *lse,
                    void *workspace, size_t workspace_bytes, int32_t *dev_err,
                    void *stream);

/* Workspace bytes for ksa_prefill_bwd: the batch plan, block offsets, an
 * fp32 [aug_rows, Hq] buffer for rowsum(dO * O), fp32 [aug_rows, Hkv, d]
 * accumulators for dk and dv (a key tile's query range is split over
 * several CTAs that add their shares) and the key-tile work list of the
 * tensor-core kernels. */
KSA_API size_t ksa_prefill_bwd_workspace_size(const ksa_params *p, int32_t batch, int64_t aug_rows);

/* KSA prefill backward: gradients of Eq. (10) under the KSA mask (sections
 * 2.2.1-2.2.2, Eqs. (2)-(3)) with respect to the augmented, rotated inputs
 * of ksa_prefill_fwd.  q_aug, k_aug, v_aug, o_aug, lse: as given to and
 * returned by ksa_prefill_fwd (lse is required); do_aug [aug_rows, Hq, d]
 * bf16: the gradient of the loss with respect to o_aug.  Writes
 * dq_aug [aug_rows, Hq, d], dk_aug / dv_aug [aug_rows, Hkv, d] (bf16) for
 * every real row (text and summary); padding rows are not written.  dk and
 * dv sum over the q heads that share a kv head.  The text query rows run on
 * the tcgen05 tensor cores (dk, dv key-stationary over 128-key tiles; dq
 * query-stationary over 128-query tiles), skipping every tile pair the rule
 * masks out entirely; the summary query rows (k+1 keys each) run on CUDA
 * cores, fused with the conversion of the fp32 accumulators.  Shapes with
 * 128 % k != 0 or d not in {64, 128} run every row on the warp-level MMA.
 * The padding rows of k_aug and v_aug must hold finite values (as
 * ksa_interleave_rope leaves them: zeros); those of q_aug and do_aug are
 * never read into a result.  dev_err and cu_seqlens as for
 * ksa_prefill_fwd. */
KSA_API int ksa_prefill_bwd(const ksa_params *p, int32_t batch, const int32_t *cu_seqlens,
                    int64_t total_text, int64_t aug_rows,
                    const void *q_aug, const void *k_aug, const void *v_aug,
                    const void *o_aug, const float *lse, const void *do_aug,
                    void *dq_aug, void *dk_aug, void *dv_aug,
                    void *workspace, size_t workspace_bytes, int32_t *dev_err, void *stream);

/* ------------------------------------------------------------------------
 * Decode cache (section 2.3.1, Figure 4).
 *
 * k, v: [batch, Hkv, slots, d] bf16, slots = ksa_cache_slots(p, cap).
 * Slot map of one (sequence, kv head):
 *   0                          scratch: the newest summary's own K/V (4c)
 *   1 .. k                     current chunk, token r at slot k - r (4b)
 *   k+1+b*k .. k+(b+1)*k       ring block b = chunk index mod w (4d)
 *   1 + k + w*k + j            summary s_j, append-only (4e)
 * state: device int32 [batch, 4] = {n_text, m, 0, err}: text tokens and
 * summaries appended so far, and the sequence's last device error.  A
 * fresh cache is all-zero state.  f = n_text - m*k tokens sit in the open
 * chunk; f == k means it waits for its summary.
 * ------------------------------------------------------------------------ */
typedef struct ksa_cache {
    void *k;
    void *v;
    int32_t *state;
    int32_t batch;
    int64_t cap_summaries;
} ksa_cache;

/* 1 + k + w*k + cap_summaries, or -1 on invalid input. */
KSA_API int64_t ksa_cache_slots(const ksa_params *p, int64_t cap_summaries);

/* Append one token per sequence.  kind: device int8 [batch] of KSA_TEXT,
 * KSA_SUMMARY or KSA_SKIP.  k_new, v_new: [batch, Hkv, d] bf16, NOT
 * rotated: K is rotated here at the token's position (text: n_text;
 * summary: n_text - 1, its chunk's last text token) unless RoPE is off.
 *   TEXT    (needs f < k): K/V into slot k - f; n_text += 1.       (4b)
 *   SUMMARY (needs f == k): K/V into slot 0 (4c); slots 1..k copied over
 *           ring block m mod w (4d); K/V into slot 1+k+w*k+m (4e); m += 1.
 * A violated precondition, or a state no sequence of appends reaches
 * (negative counts), sets state[b].err = KSA_ERR_STATE, a full summary
 * buffer KSA_ERR_CAPACITY; that sequence is left unchanged. */
KSA_API int ksa_cache_append(const ksa_params *p, const ksa_cache *cache, const int8_t *kind,
                     const void *k_new, const void *v_new, void *stream);

/* Build the decode cache of a prefilled batch in one pass: the hand-off from
 * prefill to decode (the report fills the cache token by token, Figure 4;
 * this writes the state that sequence of appends reaches, section 2.3.1).
 * k_aug, v_aug: the augmented K/V that ksa_interleave_rope wrote for the same
 * cu_seqlens (device int32 [cache->batch + 1]), i.e. already rotated.  For
 * sequence b with n_b text tokens, m_b = floor(n_b / k) summaries and
 * f_b = n_b - m_b k open tokens it writes: summary s_j at slot 1+k+w*k+j;
 * chunk c of its last min(m_b, w) complete chunks at ring block c mod w,
 * token r at slot k+1+(c mod w)*k+(k-1-r); open token r at slot k - r; and
 * state[b] = {n_b, m_b, 0, 0}.  Other slots are left as they are (they hold
 * nothing a later decode reads).  A sequence with m_b > cap_summaries is
 * not written and gets state[b].err = KSA_ERR_CAPACITY.  workspace:
 * ksa_prefill_workspace_size(p, batch, total_text) bytes; dev_err as for
 * ksa_interleave_rope (an inconsistent cu_seqlens sets KSA_ERR_INVALID
 * there and nothing is written). */
KSA_API int ksa_cache_from_prefill(const ksa_params *p, const ksa_cache *cache, const int32_t *cu_seqlens,
                           int64_t total_text, int64_t aug_rows, const void *k_aug, const void *v_aug,
                           void *workspace, size_t workspace_bytes, int32_t *dev_err, void *stream);

/* Workspace bytes for ksa_prefill_chunk: per-sequence snapshots and block
 * offsets, and the rotated q and k of the block (total_text + total_sum
 * rows of Hq + Hkv heads, bf16). */
KSA_API size_t ksa_prefill_chunk_workspace_size(const ksa_params *p, int32_t batch, int64_t total_text,
                                                int64_t total_sum);

/* Chunked prefill: a block of new text tokens per sequence, attended against
 * the sequence's decode cache, then appended to it.  The rows are the
 * prefill's (Eq. (10) under the rule of sections 2.2.1-2.2.2) for text
 * positions n0 .. n0+T_b-1 and summaries m0 .. m0+S_b-1 of sequence b, whose
 * first n0 tokens and m0 summaries are in the cache (state {n0, m0}); the
 * older keys are read from the slots of section 2.3.1 (Figure 4).
 * cu_text / cu_sum: device int32 [cache->batch + 1], the new text tokens and
 * new summaries per sequence (prefix sums; the totals are total_text and
 * total_sum).  S_b must be floor((f0 + T_b) / k), f0 = n0 - m0 k: each chunk
 * the block completes brings its summary.  Inputs (bf16, NOT rotated; rotated
 * here at those positions, a summary at its chunk's last text position):
 * q_text [total_text, Hq, d], k_text / v_text [total_text, Hkv, d], and the
 * summary tensors likewise with total_sum rows.  Outputs: o_text
 * [total_text, Hq, d], o_sum [total_sum, Hq, d] (bf16); lse_text
 * [total_text, Hq], lse_sum [total_sum, Hq] (fp32, natural log) or NULL.
 * Afterwards the cache holds what the token-by-token appends (ksa_cache_append)
 * of the same tokens would leave in every slot a later decode reads, and
 * state[b] = {n0 + T_b, m0 + S_b}.  A sequence whose state has an error, an
 * f0 outside [0, k] or the wrong S_b gets state[b].err = KSA_ERR_STATE (too
 * many summaries for cap_summaries: KSA_ERR_CAPACITY) and neither its rows
 * nor its cache are written.  Inconsistent cu arrays set *dev_err (or the
 * workspace's own word when dev_err is NULL) to KSA_ERR_INVALID and nothing
 * is written.  Supported: d in {64, 128}, any G <= 8, k >= 1, w >= 0.
 * The text rows run on the tcgen05 prefill kernel when its shape rules hold
 * (1, 2, 4 or 8 q heads per kv head), reading summary keys straight from
 * the cache in tiles of 128 slots, so every slot of cache->k / cache->v must
 * hold finite values (zero the cache once when allocating it); the block's
 * summaries are written to the cache before its text rows are attended.
 * Other shapes and the summary rows use the warp-level tensor-core MMA. */
KSA_API int ksa_prefill_chunk(const ksa_params *p, const ksa_cache *cache, const int32_t *cu_text,
                              int64_t total_text, const int32_t *cu_sum, int64_t total_sum, const void *q_text,
                              const void *k_text, const void *v_text, const void *q_sum, const void *k_sum,
                              const void *v_sum, void *o_text, void *o_sum, float *lse_text, float *lse_sum,
                              void *workspace, size_t workspace_bytes, int32_t *dev_err, void *stream);

/* Workspace bytes for ksa_decode when no sequence has more than max_text
 * text tokens. */
KSA_API size_t ksa_decode_workspace_size(const ksa_params *p, int32_t batch, int64_t max_text);

/* One decode step per sequence, after that step's ksa_cache_append.
 * q: [batch, Hq, d] bf16, NOT rotated (rotated here at position n_text-1).
 * TEXT reads slots [k-f+1, 1+k+min(m,w)*k+max(0,m-w)) with f = n_text-m*k;
 * SUMMARY reads slots [0, k+1); SKIP writes nothing.  Each is one
 * contiguous slice.  o: [batch, Hq, d] bf16; lse: [batch, Hq] fp32 or NULL.
 * max_text bounds n_text over the batch (it sizes the split-K grid and
 * must match the workspace query).  A sequence whose state cannot hold a
 * query of its kind (negative counts, f outside [1, k] for TEXT, f != 0 or
 * m = 0 for SUMMARY, a slice past the cache's slots) gets state[b].err =
 * KSA_ERR_STATE and no output. */
KSA_API int ksa_decode(const ksa_params *p, const ksa_cache *cache, const int8_t *kind, const void *q,
               void *o, float *lse, int64_t max_text,
               void *workspace, size_t workspace_bytes, void *stream);

/* ksa_decode without a workspace, for callers that cannot allocate device
 * memory: a host program that owns all of the GPU's memory (for example a
 * serving engine that reserves HBM for its own KV pools up front) or a
 * custom op that is handed only its inputs and outputs has no allocator to
 * take a workspace from, and a cudaMalloc of its own would break that
 * ownership and stall the device in the middle of its decode loop.
 * Arguments, argument checks and results are those of ksa_decode minus the
 * workspace; the split-K partials go to a 4 MiB device array that the
 * library keeps on every GPU that loads it, until the process exits.  The
 * first call made on a device looks up that array's device address, with
 * that device current; make this first call before any stream capture.
 * One split of the partials takes 4 * batch * num_q_heads * (head_dim + 2)
 * bytes; the call uses as many of ksa_decode's splits as fit in 4 MiB
 * (fewer splits only lengthen each split's share of the slice), and returns
 * KSA_ERR_CAPACITY, launching nothing, when a single split does not fit
 * (batch * num_q_heads * (head_dim + 2) > 1048576).  Every call shares the
 * one array and it keeps the last call's contents (nothing in it needs to
 * start at zero); calls whose kernels can overlap on the GPU (other
 * streams, other host threads) race on it, so the caller must order them.
 * The report has no counterpart to this call: it serves the library's
 * callers, not the method. */
KSA_API int ksa_decode_noalloc(const ksa_params *p, const ksa_cache *cache, const int8_t *kind,
                               const void *q, void *o, float *lse, int64_t max_text, void *stream);

/* ------------------------------------------------------------------------
 * KSA over an MLA latent cache (section 3.2, Eq. (6); MLA as described in
 * section 3.1: a d_c latent block holding the non-RoPE keys and values and a
 * decoupled d_r RoPE key block per cached token).
 *
 * The cache keeps the slot map of section 2.3.1 above, one latent row of
 * d_c + d_r bf16 values per slot: latent [batch, slots, d_c + d_r], state as
 * for ksa_cache.  Decoding uses the absorbed form of MLA: the caller folds
 * the key up-projection into the query (q_c, d_c values per head) and maps
 * the d_c-dim output through the value up-projection afterwards.  A head's
 * score against slot j is scale * (q_c . c_j + q_r . r_j), its output
 * sum_j softmax_j c_j: multi-query attention over the latent rows.
 * Supported: d_c = 512, d_r = 64, any num_heads.
 * ------------------------------------------------------------------------ */
typedef struct ksa_mla_params {
    int32_t k;            /* chunk size (>= 1)                                   */
    int32_t w;            /* sliding chunk number (>= 0; (w+1)*k <= 2^30)        */
    int32_t num_heads;    /* query heads (all read the same latent rows)         */
    int32_t kv_lora_rank; /* d_c: 512                                            */
    int32_t rope_dim;     /* d_r: 64                                             */
    float scale;          /* softmax scale; 0 selects 1/sqrt(d_c + d_r)          */
    double rope_theta;    /* RoPE base of the d_r part; <= 0 disables RoPE       */
} ksa_mla_params;

typedef struct ksa_mla_cache {
    void *latent;          /* [batch, slots, d_c + d_r] bf16                     */
    int32_t *state;        /* [batch, 4] {n_text, m, 0, err} as for ksa_cache    */
    int32_t batch;
    int64_t cap_summaries;
} ksa_mla_cache;

/* 1 + k + w*k + cap_summaries, or -1 on invalid input. */
KSA_API int64_t ksa_mla_cache_slots(const ksa_mla_params *p, int64_t cap_summaries);

/* Append one token per sequence to a latent cache: as ksa_cache_append,
 * with x [batch, d_c + d_r] bf16 the new latent rows (c, then r NOT
 * rotated; r is rotated here, rotate-half over its d_r dims, at the token's
 * position: text n_text, summary n_text - 1). */
KSA_API int ksa_mla_cache_append(const ksa_mla_params *p, const ksa_mla_cache *cache, const int8_t *kind,
                                 const void *x, void *stream);

/* Workspace bytes for ksa_mla_decode (split shares of each slice: fp32
 * partial outputs and softmax statistics). */
KSA_API size_t ksa_mla_decode_workspace_size(const ksa_mla_params *p, int32_t batch, int64_t max_text);

/* One decode step per sequence over its latent slice, after that step's
 * ksa_mla_cache_append.  q: [batch, num_heads, d_c + d_r] bf16 (q_c, then
 * q_r NOT rotated; rotated here at position n_text - 1).  Slices and kinds
 * as for ksa_decode.  o: [batch, num_heads, d_c] bf16, the latent output;
 * lse: [batch, num_heads] fp32 (natural log) or NULL.  max_text bounds
 * n_text over the batch and must match the workspace query.  When
 * num_heads is a multiple of 128 each group of 128 heads runs on tcgen05 in
 * clusters of two CTAs (split-K over the slice, the latent dims split
 * between the pair); other head counts run on the warp-level MMA.  A
 * pipeline wait that times out on the tcgen05 path records KSA_ERR_TIMEOUT
 * in the sequence's state[3], like the other per-sequence errors. */
KSA_API int ksa_mla_decode(const ksa_mla_params *p, const ksa_mla_cache *cache, const int8_t *kind, const void *q,
                           void *o, float *lse, int64_t max_text, void *workspace, size_t workspace_bytes,
                           void *stream);

/* Synchronise `stream`, return the device error word (KSA_OK if clear) and
 * reset it to KSA_OK.  dev_err: device int32. */
KSA_API int ksa_get_device_error(int32_t *dev_err, void *stream);

/* Self-check of the bounded-wait error path of the tensor-core pipelines
 * (the prefill, its backward, the chunked prefill and the MLA decode): every mbarrier wait
 * there gives up after a bounded number of polls or sleeps, records
 * KSA_ERR_TIMEOUT in the caller's error word, makes the CTA's other roles
 * stop waiting, and the CTA frees its tensor memory and exits, so the
 * context stays usable.  This call launches one CTA of 128 threads that
 * allocates all 512 TMEM columns of its SM and waits, with those same
 * routines, on two mbarriers that nothing ever completes: one waiter polls
 * (at most poll_limit polls, 1 .. 2^22), one sleeps in try_wait (at most
 * sleep_limit sleeps of up to 20 us, 1 .. 2^17).  Afterwards *dev_err holds
 * KSA_ERR_TIMEOUT (read it with ksa_get_device_error) and the TMEM is
 * free again.  No passage of the report corresponds to it: it checks the
 * library's own failure handling.  dev_err: device int32, 4-byte aligned.
 * Returns KSA_ERR_INVALID for a limit out of range or a bad error word. */
KSA_API int ksa_selftest_wait_timeout(uint32_t poll_limit, uint32_t sleep_limit, int32_t *dev_err,
                                      void *stream);

/* Human-readable name of a status code (static storage). */
KSA_API const char *ksa_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* KSA_H */

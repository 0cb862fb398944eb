/*
 * ksa_oracle.c -- the fp64 CPU oracle for Kwai Summary Attention (KSA).
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, plain, obviously correct
 * statement of what the KSA hot path computes.  It exists to check the CUDA
 * library against.  Only the tests, the smoke check and the benchmark's CPU
 * baseline may load it.  It shares no code, header, table or helper with the
 * CUDA path under kv_cache_compression_ksa_b200/, and it never reads anything
 * the CUDA path wrote except as the value under test.
 *
 * Everything is fp64.  Inputs arrive as fp64 arrays (the test harness widens
 * bf16 exactly).  There is no blocking, no fusion and no reordering beyond
 * the definitions cited below.
 *
 * Sources (all in "Kwai Summary Attention Technical Report"):
 *   - augmented sequence, one summary s_j after each chunk of k text tokens:
 *     section 2.2.1, Eq. (1);
 *   - a summary token sees only the text tokens of its own chunk; its
 *     position id equals that of its chunk's last text token: section 2.2.1,
 *     the two bullet rules after Eq. (1);
 *   - a text token i sees the text of chunks floor(i/k)-C .. floor(i/k)
 *     causally (Sliding Chunk Attention, Eq. (2)) plus the distant summaries
 *     s_0 .. s_{floor(i/k)-C-1} (Eq. (3)); summaries inside the window are
 *     not seen: section 2.2.2;
 *   - masked softmax attention with scale 1/sqrt(d): section 4 (distillation),
 *     Eq. (10);
 *   - the decode cache (current chunk filled right to left, scratch slot on
 *     its left, ring of sliding chunks, append-only summary buffer) and its
 *     update order on chunk completion: section 2.3.1 and Figure 4 (a)-(e);
 *   - RoPE theta = 1e6: Table 3.
 *
 * Readings where the pages are silent (each one is listed with its reason
 * in the design notes of the repository):
 *   - a summary token also sees itself (its own K/V sits in the scratch slot
 *     that summary attention reads, Figure 4c);
 *   - RoPE is the rotate-half form, applied to Q and K only, positions are
 *     the local text index; summaries take the position of their chunk's
 *     last text token;
 *   - a trailing partial chunk (n not divisible by k) gets no summary; its
 *     text tokens follow Eq. (3) unchanged;
 *   - GQA: q head h reads kv head floor(h / (Hq/Hkv)).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_API __attribute__((visibility("default")))

/* ------------------------------------------------------------------------ */
/* RoPE (rotate-half), fp64.                                                 */
/* x, out: [rows, heads, d]; pos: [rows].  out may alias x.                  */
/* For pair index r < d/2: angle = pos * theta^(-2r/d);                      */
/*   out[r]       = x[r] cos - x[r+d/2] sin                                  */
/*   out[r+d/2]   = x[r+d/2] cos + x[r] sin                                  */
/* ------------------------------------------------------------------------ */
ORACLE_API void oracle_rope(int64_t rows, int heads, int d, const double *x,
                            const int64_t *pos, double theta, double *out)
{
    const int half = d / 2;
    for (int64_t t = 0; t < rows; ++t) {
        for (int r = 0; r < half; ++r) {
            double inv_freq = pow(theta, -2.0 * (double)r / (double)d);
            double ang = (double)pos[t] * inv_freq;
            double c = cos(ang), s = sin(ang);
            for (int h = 0; h < heads; ++h) {
                const double *src = x + (t * heads + h) * (int64_t)d;
                double *dst = out + (t * heads + h) * (int64_t)d;
                double a = src[r], b = src[r + half];
                dst[r] = a * c - b * s;
                dst[r + half] = b * c + a * s;
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Visibility predicate, straight from the rules of sections 2.2.1-2.2.2.    */
/* Tokens are named by kind (0 = text, 1 = summary) and index within their   */
/* kind: text t_i, summary s_j.  n = text tokens in the sequence.            */
/* Returns 1 if the query may attend to the key.                             */
/* ------------------------------------------------------------------------ */
ORACLE_API int oracle_visible(int64_t n, int k, int C, int q_kind, int64_t q_idx,
                              int key_kind, int64_t key_idx)
{
    const int64_t m = n / k; /* complete chunks = summaries */
    if (q_kind == 1) {
        /* s_j sees t_{jk} .. t_{jk+k-1} and itself, nothing else. */
        const int64_t j = q_idx;
        if (j < 0 || j >= m) return 0;
        if (key_kind == 1) return key_idx == j;
        return key_idx >= j * k && key_idx < j * k + k;
    }
    /* text query t_i, chunk c = floor(i/k) */
    const int64_t i = q_idx;
    if (i < 0 || i >= n) return 0;
    const int64_t c = i / k;
    if (key_kind == 1) {
        /* distant summaries s_0 .. s_{c-C-1} (Eq. 3, left term) */
        return key_idx >= 0 && key_idx < m && key_idx <= c - C - 1;
    }
    /* sliding chunk text t_{(c-C)k} .. t_i (Eq. 2 / Eq. 3, right term);
       a negative start index means "from the first token". */
    int64_t lo = (c - C) * (int64_t)k;
    if (lo < 0) lo = 0;
    return key_idx >= lo && key_idx <= i;
}

/* Dense mask over the augmented sequence of Eq. (1), for small cases.
 * Row/column a -> token: chunk j = a / (k+1), slot r = a % (k+1);
 * r < k is text t_{jk+r}, r == k is summary s_j.  Trailing partial chunk:
 * its text rows follow, no summary row.  L = n + floor(n/k).
 * mask: [L, L] bytes, 1 = visible. */
ORACLE_API int64_t oracle_aug_len(int64_t n, int k) { return n + n / k; }

static void aug_token(int64_t a, int k, int *kind, int64_t *idx)
{
    int64_t j = a / (k + 1), r = a % (k + 1);
    if (r == k) { *kind = 1; *idx = j; }
    else { *kind = 0; *idx = j * k + r; }
}

ORACLE_API void oracle_dense_mask(int64_t n, int k, int C, uint8_t *mask)
{
    const int64_t L = n + n / k;
    for (int64_t a = 0; a < L; ++a) {
        int qk; int64_t qi;
        aug_token(a, k, &qk, &qi);
        for (int64_t b = 0; b < L; ++b) {
            int kk; int64_t ki;
            aug_token(b, k, &kk, &ki);
            mask[a * L + b] = (uint8_t)oracle_visible(n, k, C, qk, qi, kk, ki);
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Masked softmax attention of one query over an explicit key list.          */
/* scores_i = scale * q . k_i; o = sum_i softmax(scores)_i v_i;              */
/* lse = log(sum_i exp(scores_i)).  Eq. (10) restricted to visible keys.     */
/* keys/vals: pointers to the d-vectors of each visible key (kv head fixed). */
/* ------------------------------------------------------------------------ */
static void attend(int d, double scale, const double *q, int64_t nk,
                   const double *const *keys, const double *const *vals,
                   double *scores, double *o, double *lse)
{
    double mx = -INFINITY;
    for (int64_t t = 0; t < nk; ++t) {
        double s = 0.0;
        for (int e = 0; e < d; ++e) s += q[e] * keys[t][e];
        s *= scale;
        scores[t] = s;
        if (s > mx) mx = s;
    }
    double sum = 0.0;
    for (int64_t t = 0; t < nk; ++t) {
        scores[t] = exp(scores[t] - mx);
        sum += scores[t];
    }
    for (int e = 0; e < d; ++e) o[e] = 0.0;
    for (int64_t t = 0; t < nk; ++t) {
        double p = scores[t] / sum;
        for (int e = 0; e < d; ++e) o[e] += p * vals[t][e];
    }
    *lse = mx + log(sum);
}

/* ------------------------------------------------------------------------ */
/* The visible key set of a text query t_i as Eq. (3) writes it: the         */
/* summaries s_0 .. s_{c-C-1} and the text t_{(c-C)k} .. t_i, c = floor(i/k). */
/* Returns the summary count [0, *n_sum) and the first window text index.   */
/* ------------------------------------------------------------------------ */
static void text_query_keys(int64_t n, int k, int C, int64_t i, int64_t *n_sum, int64_t *t_lo)
{
    const int64_t m = n / k;
    const int64_t c = i / k;
    int64_t s = c - C;          /* s_0 .. s_{c-C-1}: c - C of them */
    if (s < 0) s = 0;
    if (s > m) s = m;
    int64_t lo = (c - C) * (int64_t)k;
    if (lo < 0) lo = 0;
    *n_sum = s;
    *t_lo = lo;
}

/* Number of visible (query, key) pairs per head over the whole augmented
 * sequence, from the same key sets the attention below uses. */
ORACLE_API int64_t oracle_count_pairs(int64_t n, int k, int C)
{
    int64_t tot = 0;
    for (int64_t i = 0; i < n; ++i) {
        int64_t ns, lo;
        text_query_keys(n, k, C, i, &ns, &lo);
        tot += ns + (i - lo + 1);
    }
    return tot + (n / k) * (int64_t)(k + 1);
}

/* ------------------------------------------------------------------------ */
/* KSA attention for one sequence, for a chosen set of query rows.           */
/*   qt [n, Hq, d], kt/vt [n, Hkv, d]: RoPE'd text Q/K/V                     */
/*   qs [m, Hq, d], ks/vs [m, Hkv, d]: RoPE'd summary Q/K/V, m = floor(n/k)  */
/*   tq_idx[n_tq]: text query indices (NULL: all n, in order)                */
/*   sq_idx[n_sq]: summary query indices (NULL: all m, in order)             */
/*   ot [n_tq, Hq, d], lse_t [n_tq, Hq]; os [n_sq, Hq, d], lse_s [n_sq, Hq]  */
/* The visible key list of each query is Eq. (3) (text) or the summary rule. */
/* ------------------------------------------------------------------------ */
ORACLE_API void oracle_ksa_attention(
    int64_t n, int k, int C, int Hq, int Hkv, int d, double scale,
    const double *qt, const double *kt, const double *vt,
    const double *qs, const double *ks, const double *vs,
    int64_t n_tq, const int64_t *tq_idx, int64_t n_sq, const int64_t *sq_idx,
    double *ot, double *lse_t, double *os, double *lse_s)
{
    const int64_t m = n / k;
    const int G = Hq / Hkv;
    const int64_t max_keys = n + m + 1;

    #pragma omp parallel
    {
        const double **keys = (const double **)malloc(sizeof(double *) * max_keys);
        const double **vals = (const double **)malloc(sizeof(double *) * max_keys);
        double *scores = (double *)malloc(sizeof(double) * max_keys);

        #pragma omp for schedule(dynamic, 1)
        for (int64_t u = 0; u < n_tq * Hq; ++u) {
            const int64_t qq = u / Hq;
            const int h = (int)(u % Hq), hk = h / G;
            const int64_t i = tq_idx ? tq_idx[qq] : qq;
            int64_t ns, lo, nk = 0;
            text_query_keys(n, k, C, i, &ns, &lo);
            /* distant summaries s_0 .. s_{c-C-1} */
            for (int64_t j = 0; j < ns; ++j) {
                keys[nk] = ks + (j * Hkv + hk) * (int64_t)d;
                vals[nk] = vs + (j * Hkv + hk) * (int64_t)d;
                ++nk;
            }
            /* sliding chunk text t_{(c-C)k} .. t_i */
            for (int64_t p = lo; p <= i; ++p) {
                keys[nk] = kt + (p * Hkv + hk) * (int64_t)d;
                vals[nk] = vt + (p * Hkv + hk) * (int64_t)d;
                ++nk;
            }
            attend(d, scale, qt + (i * Hq + h) * (int64_t)d, nk, keys, vals, scores,
                   ot + (qq * Hq + h) * (int64_t)d, lse_t + qq * Hq + h);
        }

        #pragma omp for schedule(dynamic, 4)
        for (int64_t u = 0; u < n_sq * Hq; ++u) {
            const int64_t qq = u / Hq;
            const int h = (int)(u % Hq), hk = h / G;
            const int64_t j = sq_idx ? sq_idx[qq] : qq;
            int64_t nk = 0;
            for (int64_t p = j * k; p < j * k + k; ++p) {
                keys[nk] = kt + (p * Hkv + hk) * (int64_t)d;
                vals[nk] = vt + (p * Hkv + hk) * (int64_t)d;
                ++nk;
            }
            keys[nk] = ks + (j * Hkv + hk) * (int64_t)d; /* itself */
            vals[nk] = vs + (j * Hkv + hk) * (int64_t)d;
            ++nk;
            attend(d, scale, qs + (j * Hq + h) * (int64_t)d, nk, keys, vals, scores,
                   os + (qq * Hq + h) * (int64_t)d, lse_s + qq * Hq + h);
        }
        free(keys); free(vals); free(scores);
    }
}

/* ------------------------------------------------------------------------ */
/* Decode cache model (section 2.3.1, Figure 4).                             */
/*                                                                           */
/* One sequence's cache is an array of S = 1 + k + C*k + cap slots, each     */
/* slot holding one [Hkv, d] K row and one V row.  Slot map:                 */
/*   slot 0                       scratch: the newest summary's own K/V      */
/*   slots 1 .. k                 current chunk; its token r (0-based) sits  */
/*                                at slot k - r (filled right to left, right */
/*                                edge against the ring)                     */
/*   slots k+1+b*k .. k+(b+1)*k   ring block b; chunk c lives in block c % C */
/*                                as a block copy of the current chunk       */
/*   slot 1 + k + C*k + j         summary s_j (append-only, grows right)     */
/*                                                                           */
/* State: n_text (text tokens appended), m (summaries appended).             */
/* f = n_text - m*k tokens sit in the open chunk; f == k means the chunk is  */
/* complete and waits for its summary.                                       */
/* ------------------------------------------------------------------------ */
typedef struct {
    int k, C, Hkv, d;
    int64_t cap, n_text, m;
    double *K, *V; /* [S, Hkv, d] */
} oracle_cache;

ORACLE_API int64_t oracle_cache_slots(int k, int C, int64_t cap)
{
    return 1 + (int64_t)k + (int64_t)C * k + cap;
}

ORACLE_API oracle_cache *oracle_cache_new(int k, int C, int Hkv, int d, int64_t cap)
{
    oracle_cache *c = (oracle_cache *)calloc(1, sizeof(oracle_cache));
    int64_t S = oracle_cache_slots(k, C, cap);
    c->k = k; c->C = C; c->Hkv = Hkv; c->d = d; c->cap = cap;
    c->K = (double *)calloc((size_t)(S * Hkv * d), sizeof(double));
    c->V = (double *)calloc((size_t)(S * Hkv * d), sizeof(double));
    return c;
}

ORACLE_API void oracle_cache_free(oracle_cache *c)
{
    if (!c) return;
    free(c->K); free(c->V); free(c);
}

ORACLE_API double *oracle_cache_k(oracle_cache *c) { return c->K; }
ORACLE_API double *oracle_cache_v(oracle_cache *c) { return c->V; }
ORACLE_API int64_t oracle_cache_n_text(oracle_cache *c) { return c->n_text; }
ORACLE_API int64_t oracle_cache_m(oracle_cache *c) { return c->m; }

static void put_slot(oracle_cache *c, int64_t slot, const double *k_row, const double *v_row)
{
    const int64_t w = (int64_t)c->Hkv * c->d;
    memcpy(c->K + slot * w, k_row, sizeof(double) * w);
    memcpy(c->V + slot * w, v_row, sizeof(double) * w);
}

/* Figure 4b: write a new text token's K/V into the next free slot of the
 * current chunk.  k_row/v_row: [Hkv, d] (already RoPE'd).
 * Returns 0, or -1 if the open chunk is already complete. */
ORACLE_API int oracle_cache_append_text(oracle_cache *c, const double *k_row, const double *v_row)
{
    int64_t f = c->n_text - c->m * c->k;
    if (f >= c->k) return -1;
    put_slot(c, c->k - f, k_row, v_row);
    c->n_text += 1;
    return 0;
}

/* Figure 4c-4e, in the order of section 2.3.1 (i)-(iii):
 *   (i)   the summary's K/V goes to the scratch slot;
 *   (ii)  the finished chunk (slots 1..k) is copied over ring block m % C;
 *   (iii) the summary's K/V is appended to the summary buffer.
 * Returns 0, -1 if the chunk is not complete, -3 if the buffer is full. */
ORACLE_API int oracle_cache_append_summary(oracle_cache *c, const double *k_row, const double *v_row)
{
    int64_t f = c->n_text - c->m * c->k;
    if (f != c->k) return -1;
    if (c->m >= c->cap) return -3;
    const int64_t w = (int64_t)c->Hkv * c->d;
    put_slot(c, 0, k_row, v_row);
    if (c->C > 0) {
        int64_t b = c->m % c->C;
        int64_t dst = 1 + c->k + b * c->k;
        memcpy(c->K + dst * w, c->K + 1 * w, sizeof(double) * w * c->k);
        memcpy(c->V + dst * w, c->V + 1 * w, sizeof(double) * w * c->k);
    }
    put_slot(c, 1 + c->k + (int64_t)c->C * c->k + c->m, k_row, v_row);
    c->m += 1;
    return 0;
}

/* The single contiguous slice [lo, hi) a decode query reads (section 2.3.1:
 * "every KV read during decoding corresponds to a contiguous slice").
 * kind 0 (text): the newest text token, after its append; f' = n_text - m*k
 *   tokens of the open chunk are visible (slots k-f'+1 .. k), then the ring
 *   blocks holding chunks max(0,m-C) .. m-1, then summaries s_0 .. s_{m-C-1}.
 * kind 1 (summary): the newest summary, after its append: scratch + the
 *   k slots of the chunk it summarises. */
ORACLE_API void oracle_cache_slice(oracle_cache *c, int kind, int64_t *lo, int64_t *hi)
{
    const int64_t k = c->k, C = c->C, m = c->m;
    if (kind == 1) { *lo = 0; *hi = k + 1; return; }
    int64_t fp = c->n_text - m * k;
    int64_t ring = m < C ? m : C;
    int64_t far = m - C > 0 ? m - C : 0;
    *lo = k - fp + 1;
    *hi = 1 + k + ring * k + far;
}

/* Decode: Eq. (10) for one query vector per q head against the cache slice.
 * q: [Hq, d] (already RoPE'd); o: [Hq, d]; lse: [Hq]. */
ORACLE_API void oracle_cache_decode(oracle_cache *c, int kind, int Hq, double scale,
                                    const double *q, double *o, double *lse)
{
    int64_t lo, hi;
    oracle_cache_slice(c, kind, &lo, &hi);
    const int d = c->d, Hkv = c->Hkv, G = Hq / Hkv;
    const int64_t nk = hi - lo;
    /* the query heads are independent: one per thread, each with its own
     * key lists and score buffer (the per-head arithmetic is unchanged) */
    #pragma omp parallel
    {
        const double **keys = (const double **)malloc(sizeof(double *) * (nk + 1));
        const double **vals = (const double **)malloc(sizeof(double *) * (nk + 1));
        double *scores = (double *)malloc(sizeof(double) * (nk + 1));
        #pragma omp for schedule(static)
        for (int h = 0; h < Hq; ++h) {
            int hk = h / G;
            for (int64_t t = 0; t < nk; ++t) {
                keys[t] = c->K + ((lo + t) * Hkv + hk) * (int64_t)d;
                vals[t] = c->V + ((lo + t) * Hkv + hk) * (int64_t)d;
            }
            attend(d, scale, q + (int64_t)h * d, nk, keys, vals, scores, o + (int64_t)h * d, lse + h);
        }
        free(keys); free(vals); free(scores);
    }
}

/* Decode over an externally held cache image laid out [S, Hkv, d] (the
 * same slot map), for checking a cache the oracle did not build.  The
 * state (n_text, m) says which slots are live. */
ORACLE_API void oracle_decode_image(int k, int C, int Hkv, int d, int64_t cap,
                                    int64_t n_text, int64_t m, int kind,
                                    const double *K, const double *V,
                                    int Hq, double scale, const double *q,
                                    double *o, double *lse)
{
    oracle_cache c;
    c.k = k; c.C = C; c.Hkv = Hkv; c.d = d; c.cap = cap;
    c.n_text = n_text; c.m = m;
    c.K = (double *)K; c.V = (double *)V;
    oracle_cache_decode(&c, kind, Hq, scale, q, o, lse);
}

// prefill_bwd.cu -- backward of the KSA prefill attention: dq, dk, dv of the
// augmented (rotated) Q, K, V given dO, O and the forward's LSE.
//
// Kwai Summary Attention Technical Report: the forward is Eq. (10),
// softmax(Q K^T / sqrt(d) + M_KSA) V, with the mask of section 2.2.1 (a
// summary sees its chunk's k text tokens and itself) and section 2.2.2,
// Eqs. (2)-(3) (text t_i sees text chunks c-w .. c causally and the
// summaries s_0 .. s_{c-w-1}).  The gradients are the textbook ones under the
// same mask: P = exp(S - lse), dP = dO V^T, D = rowsum(dO * O),
// dS = P * (dP - D), dq = scale dS K, dk = scale dS^T Q, dv = P^T dO.
//
// launch_prefill_bwd runs D = rowsum(dO * O), then, where the shape allows
// (k divides 128, d of 64 or 128), the tensor-core kernels of
// prefill_bwd_sm100.cu for the text query rows and bwd_sum_rows_kernel for
// the summary query rows fused with the fp32 -> bf16 conversion; every other
// shape runs on the warp-level kernels below.
//
// Warp-level path.  Work is cut the way the forward skips tiles: a block
// holds 64 rows of one kind (64 consecutive text tokens or 64 consecutive
// summaries of one sequence), and a query block only meets the key blocks its
// rows can see (summaries 0 .. c_last-w-1 and the text of chunks c_first-w ..
// c_last), and a key block only the query blocks that can see it.  Inside a
// pair of blocks the mask is evaluated per element from the rows' coordinates.
//
//   bwd_dot_kernel   D = rowsum(dO * O)                          (HBM)
//   bwd_sum_rows_kernel  tensor-core path: the summary query rows (k+1 keys
//                    each) on CUDA cores, added into the accumulators as they
//                    are converted to bf16
//   bwd_dq_kernel    query-stationary: dq of 64 rows of one q head
//   bwd_dkv_kernel   key-stationary: dk, dv of 64 rows of one kv head, over
//                    all q heads of its group and (grid z) a share of at
//                    most 16 of the query blocks that see them, added into
//                    fp32 accumulators (the first summaries are seen by every
//                    later text row, so their query ranges are split)
//   bwd_dkv_out_kernel  accumulators -> bf16
// Both attention kernels use the warp-level tensor-core MMA (m16n8k16, bf16
// in, fp32 accumulate) with operands staged in shared memory and read with
// ldmatrix; each warp owns 16 rows of its block.  dq rows belong to exactly
// one block and are written once.
#include <math.h>

#include "ksa_internal.cuh"
#include "warp_mma.cuh"

namespace ksa {
namespace bw {

constexpr int RB = 64;          // rows per block
constexpr int kThreads = 128;   // 4 warps x 16 rows
constexpr int TEXT_ROWS = 0, SUM_ROWS = 1;
constexpr int QB_SPLIT = 16;    // query blocks per dk/dv CTA: long query ranges are split

struct Args {
    int k, w, Hq, Hkv, G, batch;
    float scale, scale_log2;
    const int32_t *cu;
    Plan pl;
    const int32_t *tb_off, *sb_off;   // [B+1] first text / summary block of each sequence
    int32_t *err;
    const __nv_bfloat16 *q, *kk, *v, *o, *dout;
    const float *lse;                 // [rows, Hq] natural log
    float *dsum;                      // [rows, Hq] D = rowsum(dO * O)
    float *dk32, *dv32;               // [rows, Hkv, d] fp32 accumulators of the split dk/dv pass
    int nblk;                         // upper bound of the block count (grid x)
    __nv_bfloat16 *dq, *dk, *dv;
};

// A block: rows of one kind of sequence b.
struct Blk {
    int b, kind, idx0, cnt, n, m;
    int64_t c0;    // first chunk of the sequence in the augmented layout
};

__device__ __forceinline__ int64_t aug_row(const Args &a, const Blk &B, int idx)
{
    return B.kind == TEXT_ROWS ? (B.c0 + idx / a.k) * (a.k + 1) + idx % a.k : (B.c0 + idx) * (a.k + 1) + a.k;
}

__device__ __forceinline__ int find_seq(const int32_t *off, int batch, int id)
{
    int lo = 0, hi = batch - 1;
    while (lo < hi) {
        int mid = (lo + hi + 1) >> 1;
        if (off[mid] <= id) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// block id -> (sequence, kind, rows): text blocks of all sequences first
__device__ __forceinline__ bool block_of(const Args &a, int id, Blk &B)
{
    const int nt = a.tb_off[a.batch];
    int b, kind, j;
    if (id < nt) {
        b = find_seq(a.tb_off, a.batch, id); kind = TEXT_ROWS; j = id - a.tb_off[b];
    } else {
        id -= nt;
        if (id >= a.sb_off[a.batch]) return false;
        b = find_seq(a.sb_off, a.batch, id); kind = SUM_ROWS; j = id - a.sb_off[b];
    }
    B.b = b; B.kind = kind;
    B.n = a.cu[b + 1] - a.cu[b];
    B.m = B.n / a.k;
    B.c0 = a.pl.chunk_off[b];
    B.idx0 = j * RB;
    B.cnt = min(RB, (kind == TEXT_ROWS ? B.n : B.m) - B.idx0);
    return B.cnt > 0;
}

// 64 rows x D bf16 of one head into shared memory, rows padded by 16 bytes
// (row pitch D + 8 elements keeps ldmatrix's 8-row reads conflict-free);
// rows at or beyond cnt are zero.
template <int D>
__device__ __forceinline__ void load_rows(__nv_bfloat16 (*dst)[D + 8], const __nv_bfloat16 *src, int H, int head,
                                          const Args &a, const Blk &B, int first, int cnt)
{
    constexpr int V8 = D / 8;
    for (int e = threadIdx.x; e < RB * V8; e += kThreads) {
        const int r = e / V8, c8 = e % V8;
        uint4 val = make_uint4(0, 0, 0, 0);
        if (r < cnt) val = reinterpret_cast<const uint4 *>(src + (aug_row(a, B, first + r) * H + head) * D)[c8];
        *reinterpret_cast<uint4 *>(&dst[r][c8 * 8]) = val;
    }
}

// the same, issued as 16-byte cp.async copies (one commit group per call);
// zero rows are written directly
template <int D>
__device__ __forceinline__ void load_rows_async(__nv_bfloat16 (*dst)[D + 8], const __nv_bfloat16 *src, int H, int head,
                                                const Args &a, const Blk &B, int first, int cnt)
{
    constexpr int V8 = D / 8;
    for (int e = threadIdx.x; e < RB * V8; e += kThreads) {
        const int r = e / V8, c8 = e % V8;
        if (r < cnt) {
            const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(&dst[r][c8 * 8]));
            const void *g = reinterpret_cast<const uint4 *>(src + (aug_row(a, B, first + r) * H + head) * D) + c8;
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(g) : "memory");
        } else {
            *reinterpret_cast<uint4 *>(&dst[r][c8 * 8]) = make_uint4(0, 0, 0, 0);
        }
    }
}

using wm::cp_commit;
using wm::cp_wait;
using wm::frag_a;
using wm::frag_b_kn;
using wm::frag_b_nk;

// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) bwd_dot_kernel(Args a, int64_t cells)
{
    // D = dO . O over d for each (row, head) cell: D / 8 consecutive lanes
    // take one cell, 16 bytes each, so that a warp's loads are contiguous
    constexpr int L = D / 8;
    const int64_t t = (int64_t)blockIdx.x * 256 + threadIdx.x;
    const int64_t cell = t / L;
    const bool live = cell < cells;
    float s = 0.f;
    if (live) {
        const uint4 u = reinterpret_cast<const uint4 *>(a.dout)[t], w = reinterpret_cast<const uint4 *>(a.o)[t];
        const uint32_t uu[4] = {u.x, u.y, u.z, u.w}, ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            s = fmaf(__uint_as_float(uu[i] << 16), __uint_as_float(ww[i] << 16), s);
            s = fmaf(__uint_as_float(uu[i] & 0xffff0000u), __uint_as_float(ww[i] & 0xffff0000u), s);
        }
    }
#pragma unroll
    for (int off = L / 2; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (live && (t % L) == 0) a.dsum[cell] = s;
}

// ---------------------------------------------------------------------------
// dq: one CTA = one query block x one q head.
template <int D>
__global__ void __launch_bounds__(kThreads) bwd_dq_kernel(Args a)
{
    constexpr int KC = D / 16, NT = D / 8;
    using Row = __nv_bfloat16[D + 8];
    extern __shared__ __align__(16) uint8_t bw_smem[];
    // Q, dO, then two buffers of (K, V)
    Row *sQ = reinterpret_cast<Row *>(bw_smem), *sO = sQ + RB, *sKV = sO + RB;
    if (*a.err != 0) return;
    Blk Q;
    // text blocks late in a sequence see the most summaries: reverse order
    // puts them first
    const int nreal = a.tb_off[a.batch] + a.sb_off[a.batch];
    const int id = (int)blockIdx.x < nreal ? nreal - 1 - (int)blockIdx.x : (int)blockIdx.x;
    if (!block_of(a, id, Q)) return;
    const int h = blockIdx.y, g = h / a.G;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gr = lane >> 2, tt = lane & 3;
    load_rows<D>(sQ, a.q, a.Hq, h, a, Q, Q.idx0, Q.cnt);
    load_rows<D>(sO, a.dout, a.Hq, h, a, Q, Q.idx0, Q.cnt);
    // this warp's two rows per lane: 16 warp + gr and + 8
    float lse2[2], dd[2];
    int qi[2];
    bool live[2];
#pragma unroll
    for (int x = 0; x < 2; ++x) {
        const int r = 16 * warp + gr + 8 * x;
        live[x] = r < Q.cnt;
        qi[x] = Q.idx0 + r;
        const int64_t row = live[x] ? aug_row(a, Q, qi[x]) : 0;
        lse2[x] = live[x] ? a.lse[row * a.Hq + h] * 1.4426950408889634f : 0.f;
        dd[x] = live[x] ? a.dsum[row * a.Hq + h] : 0.f;
    }
    __syncthreads();
    uint32_t qf[KC][4], of[KC][4];
#pragma unroll
    for (int c = 0; c < KC; ++c) {
        frag_a<D>(qf[c], sQ, 16 * warp, 16 * c);
        frag_a<D>(of[c], sO, 16 * warp, 16 * c);
    }
    float acc[NT][4];
#pragma unroll
    for (int i = 0; i < NT; ++i) acc[i][0] = acc[i][1] = acc[i][2] = acc[i][3] = 0.f;
    // per row, the keys it sees: text [lt_lo, lt_hi], summaries [ls_lo, ls_hi)
    int lt_lo[2], lt_hi[2], ls_lo[2], ls_hi[2];
#pragma unroll
    for (int x = 0; x < 2; ++x) {
        if (!live[x]) {
            lt_lo[x] = 1; lt_hi[x] = 0; ls_lo[x] = ls_hi[x] = 0;
        } else if (Q.kind == TEXT_ROWS) {
            const int c = qi[x] / a.k;
            lt_lo[x] = max(0, c - a.w) * a.k; lt_hi[x] = qi[x];
            ls_lo[x] = 0; ls_hi[x] = max(0, min(c - a.w, Q.m));
        } else {
            lt_lo[x] = qi[x] * a.k; lt_hi[x] = qi[x] * a.k + a.k - 1;
            ls_lo[x] = qi[x]; ls_hi[x] = qi[x] + 1;
        }
    }

    // the key blocks these rows can see
    int nsb = 0, t_lo = 0, t_hi = 0, s_lo = 0;
    if (Q.kind == TEXT_ROWS) {
        const int ca = Q.idx0 / a.k, cb = (Q.idx0 + Q.cnt - 1) / a.k;
        const int ns = max(0, min(cb - a.w, Q.m));
        nsb = (ns + RB - 1) / RB;            // summary key blocks [0, ns)
        t_lo = max(0, ca - a.w) * a.k;       // text keys [t_lo, t_hi)
        t_hi = Q.idx0 + Q.cnt;
    } else {
        t_lo = Q.idx0 * a.k;
        t_hi = (Q.idx0 + Q.cnt) * a.k;
        nsb = 1;                             // the block's own summaries (each sees itself)
        s_lo = Q.idx0;
    }
    const int ntb = (t_hi - t_lo + RB - 1) / RB;
    const int s_end = Q.kind == TEXT_ROWS ? max(0, min((Q.idx0 + Q.cnt - 1) / a.k - a.w, Q.m)) : Q.idx0 + Q.cnt;
    auto key_block = [&](int kb) {
        Blk K = Q;
        if (kb < nsb) {
            K.kind = SUM_ROWS; K.idx0 = s_lo + kb * RB; K.cnt = min(RB, s_end - K.idx0);
        } else {
            K.kind = TEXT_ROWS; K.idx0 = t_lo + (kb - nsb) * RB; K.cnt = min(RB, t_hi - K.idx0);
        }
        return K;
    };
    auto prefetch = [&](int kb) {   // key block kb -> buffer kb % 2 (one commit group)
        const Blk K = key_block(kb);
        Row *b = sKV + (kb & 1) * 2 * RB;
        load_rows_async<D>(b, a.kk, a.Hkv, g, a, K, K.idx0, K.cnt);
        load_rows_async<D>(b + RB, a.v, a.Hkv, g, a, K, K.idx0, K.cnt);
        cp_commit();
    };
    const int nkb = nsb + ntb;
    if (nkb > 0) prefetch(0);
    for (int kb = 0; kb < nkb; ++kb) {
        const Blk K = key_block(kb);
        if (kb + 1 < nkb) {
            prefetch(kb + 1);
            cp_wait<1>();
        } else {
            cp_wait<0>();
        }
        __syncthreads();   // key block kb has landed for every thread
        Row *sK = sKV + (kb & 1) * 2 * RB, *sV = sK + RB;
        // a whole key block inside every text row's range needs no mask
        bool full = K.cnt == RB && Q.kind == TEXT_ROWS;
        if (full) {
            const int ia = Q.idx0, ib = Q.idx0 + Q.cnt - 1, ca = ia / a.k, cb = ib / a.k;
            full = K.kind == SUM_ROWS ? K.idx0 + K.cnt - 1 < min(ca - a.w, Q.m)
                                      : (K.idx0 + K.cnt - 1 <= ia && K.idx0 >= max(0, cb - a.w) * a.k);
        }
        // S = Q K^T and dP = dO V^T: 16 rows x 64 keys
        float s[8][4], dp[8][4];
#pragma unroll
        for (int i = 0; i < 8; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = dp[i][0] = dp[i][1] = dp[i][2] = dp[i][3] = 0.f;
#pragma unroll
        for (int c = 0; c < KC; ++c)
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                uint32_t bk[4], bv[4];
                frag_b_nk<D>(bk, sK, 16 * np, 16 * c);
                frag_b_nk<D>(bv, sV, 16 * np, 16 * c);
                wm::mma16816(s[2 * np], qf[c][0], qf[c][1], qf[c][2], qf[c][3], bk[0], bk[1]);
                wm::mma16816(s[2 * np + 1], qf[c][0], qf[c][1], qf[c][2], qf[c][3], bk[2], bk[3]);
                wm::mma16816(dp[2 * np], of[c][0], of[c][1], of[c][2], of[c][3], bv[0], bv[1]);
                wm::mma16816(dp[2 * np + 1], of[c][0], of[c][1], of[c][2], of[c][3], bv[2], bv[3]);
            }
        // dS = P * (dP - D), P = exp(S - lse) on visible pairs, as bf16 A fragments
        uint32_t dsf[4][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            float e[4];
#pragma unroll
            for (int z = 0; z < 4; ++z) {
                const int x = z >> 1, col = 8 * nt + 2 * tt + (z & 1), key = K.idx0 + col;
                const bool vis = full || (col < K.cnt && (K.kind == TEXT_ROWS ? key >= lt_lo[x] && key <= lt_hi[x]
                                                                                : key >= ls_lo[x] && key < ls_hi[x]));
                const float p = vis ? wm::ex2(s[nt][z] * a.scale_log2 - lse2[x]) : 0.f;
                e[z] = p * (dp[nt][z] - dd[x]);
            }
            const int j = nt >> 1;
            if ((nt & 1) == 0) { dsf[j][0] = wm::pack2(e[0], e[1]); dsf[j][1] = wm::pack2(e[2], e[3]); }
            else { dsf[j][2] = wm::pack2(e[0], e[1]); dsf[j][3] = wm::pack2(e[2], e[3]); }
        }
        // dq += dS K (k = keys, n = dims)
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int np = 0; np < NT / 2; ++np) {
                uint32_t bk[4];
                frag_b_kn<D>(bk, sK, 16 * j, 16 * np);
                wm::mma16816(acc[2 * np], dsf[j][0], dsf[j][1], dsf[j][2], dsf[j][3], bk[0], bk[1]);
                wm::mma16816(acc[2 * np + 1], dsf[j][0], dsf[j][1], dsf[j][2], dsf[j][3], bk[2], bk[3]);
            }
        __syncthreads();   // buffer kb % 2 is read: the next prefetch may overwrite it
    }
    // dq rows: acc[nt] holds (row gr, dims 8nt + 2tt, +1) and (row gr + 8, same dims)
#pragma unroll
    for (int x = 0; x < 2; ++x) {
        if (!live[x]) continue;
        __nv_bfloat16 *dst = a.dq + (aug_row(a, Q, qi[x]) * a.Hq + h) * D;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
            *reinterpret_cast<uint32_t *>(dst + 8 * nt + 2 * tt) =
                wm::pack2(acc[nt][2 * x] * a.scale, acc[nt][2 * x + 1] * a.scale);
    }
}

// ---------------------------------------------------------------------------
// dk, dv: one CTA = one key block x one kv head, over the q heads of its group.
template <int D>
__global__ void __launch_bounds__(kThreads) bwd_dkv_kernel(Args a)
{
    constexpr int KC = D / 16, NT = D / 8;
    using Row = __nv_bfloat16[D + 8];
    extern __shared__ __align__(16) uint8_t bw_smem[];
    // K, V, then two buffers of (Q, dO), then two buffers of (LSE, D)
    Row *sK = reinterpret_cast<Row *>(bw_smem), *sV = sK + RB, *sQO = sV + RB;
    float *sLD = reinterpret_cast<float *>(sQO + 4 * RB);
    if (*a.err != 0) return;
    Blk K;
    if (!block_of(a, blockIdx.x, K)) return;
    const int g = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gr = lane >> 2, tt = lane & 3;
    int ki[2];
    bool live[2];
    // per key row, the queries that see it (the rule inverted): text
    // queries [qt_lo, qt_hi], summary queries [qs_lo, qs_hi).  Text key p of
    // chunk c_p: text queries p .. (c_p + w + 1) k - 1 and summary c_p (if
    // that chunk is complete); summary key j: text queries from
    // (j + w + 1) k on and summary j.
    int qt_lo[2], qt_hi[2], qs_lo[2], qs_hi[2];
#pragma unroll
    for (int x = 0; x < 2; ++x) {
        const int r = 16 * warp + gr + 8 * x;
        live[x] = r < K.cnt;
        ki[x] = K.idx0 + r;
        if (!live[x]) {
            qt_lo[x] = 1; qt_hi[x] = 0; qs_lo[x] = qs_hi[x] = 0;
        } else if (K.kind == TEXT_ROWS) {
            const int cp = ki[x] / a.k;
            qt_lo[x] = ki[x]; qt_hi[x] = window_end(cp, a.w, a.k, K.n) - 1;
            qs_lo[x] = cp; qs_hi[x] = cp < K.m ? cp + 1 : cp;
        } else {
            qt_lo[x] = window_end(ki[x], a.w, a.k, K.n); qt_hi[x] = INT32_MAX;
            qs_lo[x] = ki[x]; qs_hi[x] = ki[x] + 1;
        }
    }
    float dk[NT][4], dv[NT][4];
#pragma unroll
    for (int i = 0; i < NT; ++i) dk[i][0] = dk[i][1] = dk[i][2] = dk[i][3] = dv[i][0] = dv[i][1] = dv[i][2] = dv[i][3] = 0.f;

    // the query blocks that can see these keys
    int t_lo, t_hi, s_lo, s_hi;
    if (K.kind == TEXT_ROWS) {
        const int ca = K.idx0 / a.k, cb = (K.idx0 + K.cnt - 1) / a.k;
        t_lo = K.idx0;
        t_hi = window_end(cb, a.w, a.k, K.n);
        s_lo = ca;
        s_hi = min(cb + 1, K.m);
    } else {
        t_lo = window_end(K.idx0, a.w, a.k, K.n);
        t_hi = K.n;
        s_lo = K.idx0;
        s_hi = K.idx0 + K.cnt;
    }
    const int ntb = (t_hi - t_lo + RB - 1) / RB;
    const int nsb = s_hi > s_lo ? 1 : 0;   // at most 64 summaries see this block's keys
    // this CTA's share of the query blocks (split z of ceil((ntb + nsb) / QB_SPLIT))
    const int qb_lo = (int)blockIdx.z * QB_SPLIT, qb_hi = min(ntb + nsb, qb_lo + QB_SPLIT);
    if (qb_lo >= ntb + nsb) return;   // an empty share (block-uniform), before any load
    load_rows<D>(sK, a.kk, a.Hkv, g, a, K, K.idx0, K.cnt);
    load_rows<D>(sV, a.v, a.Hkv, g, a, K, K.idx0, K.cnt);
    const int nq = qb_hi - qb_lo;   // query blocks per head in this share
    auto query_block = [&](int qb) {
        Blk Q = K;
        if (qb < ntb) {
            Q.kind = TEXT_ROWS; Q.idx0 = t_lo + qb * RB; Q.cnt = min(RB, t_hi - Q.idx0);
        } else {
            Q.kind = SUM_ROWS; Q.idx0 = s_lo; Q.cnt = s_hi - s_lo;
        }
        return Q;
    };
    auto prefetch = [&](int it) {   // step it = (head, query block) -> buffer it % 2
        const int h = g * a.G + it / nq;
        const Blk Q = query_block(qb_lo + it % nq);
        Row *b = sQO + (it & 1) * 2 * RB;
        load_rows_async<D>(b, a.q, a.Hq, h, a, Q, Q.idx0, Q.cnt);
        load_rows_async<D>(b + RB, a.dout, a.Hq, h, a, Q, Q.idx0, Q.cnt);
        float *ld = sLD + (it & 1) * 2 * RB;
        for (int r = threadIdx.x; r < RB; r += kThreads) {
            const bool ok = r < Q.cnt;
            const int64_t row = ok ? aug_row(a, Q, Q.idx0 + r) : 0;
            ld[r] = ok ? a.lse[row * a.Hq + h] * 1.4426950408889634f : 0.f;
            ld[RB + r] = ok ? a.dsum[row * a.Hq + h] : 0.f;
        }
        cp_commit();
    };
    const int nsteps = a.G * nq;
    prefetch(0);
    for (int it = 0; it < nsteps; ++it) {
        {
            const Blk Q = query_block(qb_lo + it % nq);
            if (it + 1 < nsteps) {
                prefetch(it + 1);
                cp_wait<1>();
            } else {
                cp_wait<0>();
            }
            __syncthreads();   // step it has landed for every thread
            Row *sQ = sQO + (it & 1) * 2 * RB, *sO = sQ + RB;
            const float *sL = sLD + (it & 1) * 2 * RB, *sD = sL + RB;
            // a whole text query block that sees every live key of the block
            bool full = Q.cnt == RB && Q.kind == TEXT_ROWS;
            if (full) {
                const int k_last = K.idx0 + K.cnt - 1;
                full = K.kind == SUM_ROWS ? Q.idx0 >= window_end(k_last, a.w, a.k, K.n)
                                          : (Q.idx0 >= k_last && Q.idx0 + RB - 1 <= window_end(K.idx0 / a.k, a.w, a.k, K.n) - 1);
            }
            // two halves of 32 queries: S^T = K Q^T, dP^T = V dO^T (16 keys x 32 queries)
#pragma unroll 1
            for (int hq = 0; hq < 2; ++hq) {
                const int q0 = 32 * hq;
                if (q0 >= Q.cnt) break;
                float s[4][4], dp[4][4];
#pragma unroll
                for (int i = 0; i < 4; ++i) s[i][0] = s[i][1] = s[i][2] = s[i][3] = dp[i][0] = dp[i][1] = dp[i][2] = dp[i][3] = 0.f;
#pragma unroll
                for (int c = 0; c < KC; ++c) {
                    uint32_t ak[4], av[4];
                    frag_a<D>(ak, sK, 16 * warp, 16 * c);
                    frag_a<D>(av, sV, 16 * warp, 16 * c);
#pragma unroll
                    for (int np = 0; np < 2; ++np) {
                        uint32_t bq[4], bo[4];
                        frag_b_nk<D>(bq, sQ, q0 + 16 * np, 16 * c);
                        frag_b_nk<D>(bo, sO, q0 + 16 * np, 16 * c);
                        wm::mma16816(s[2 * np], ak[0], ak[1], ak[2], ak[3], bq[0], bq[1]);
                        wm::mma16816(s[2 * np + 1], ak[0], ak[1], ak[2], ak[3], bq[2], bq[3]);
                        wm::mma16816(dp[2 * np], av[0], av[1], av[2], av[3], bo[0], bo[1]);
                        wm::mma16816(dp[2 * np + 1], av[0], av[1], av[2], av[3], bo[2], bo[3]);
                    }
                }
                // P^T and dS^T as bf16 A fragments (16 keys x 32 queries = 2 k-chunks)
                uint32_t pf[2][4], dsf[2][4];
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) {
                    float pe[4], de[4];
#pragma unroll
                    for (int z = 0; z < 4; ++z) {
                        const int x = z >> 1, col = q0 + 8 * nt + 2 * tt + (z & 1), qi = Q.idx0 + col;
                        const bool vis = full || (col < Q.cnt && (Q.kind == TEXT_ROWS ? qi >= qt_lo[x] && qi <= qt_hi[x]
                                                                                      : qi >= qs_lo[x] && qi < qs_hi[x]));
                        const float p = vis ? wm::ex2(s[nt][z] * a.scale_log2 - sL[col]) : 0.f;
                        pe[z] = p;
                        de[z] = p * (dp[nt][z] - sD[col]);
                    }
                    const int j = nt >> 1;
                    if ((nt & 1) == 0) {
                        pf[j][0] = wm::pack2(pe[0], pe[1]); pf[j][1] = wm::pack2(pe[2], pe[3]);
                        dsf[j][0] = wm::pack2(de[0], de[1]); dsf[j][1] = wm::pack2(de[2], de[3]);
                    } else {
                        pf[j][2] = wm::pack2(pe[0], pe[1]); pf[j][3] = wm::pack2(pe[2], pe[3]);
                        dsf[j][2] = wm::pack2(de[0], de[1]); dsf[j][3] = wm::pack2(de[2], de[3]);
                    }
                }
                // dv += P^T dO, dk += dS^T Q (k = queries, n = dims)
#pragma unroll
                for (int j = 0; j < 2; ++j)
#pragma unroll
                    for (int np = 0; np < NT / 2; ++np) {
                        uint32_t bo[4], bq[4];
                        frag_b_kn<D>(bo, sO, q0 + 16 * j, 16 * np);
                        frag_b_kn<D>(bq, sQ, q0 + 16 * j, 16 * np);
                        wm::mma16816(dv[2 * np], pf[j][0], pf[j][1], pf[j][2], pf[j][3], bo[0], bo[1]);
                        wm::mma16816(dv[2 * np + 1], pf[j][0], pf[j][1], pf[j][2], pf[j][3], bo[2], bo[3]);
                        wm::mma16816(dk[2 * np], dsf[j][0], dsf[j][1], dsf[j][2], dsf[j][3], bq[0], bq[1]);
                        wm::mma16816(dk[2 * np + 1], dsf[j][0], dsf[j][1], dsf[j][2], dsf[j][3], bq[2], bq[3]);
                    }
            }
            __syncthreads();   // buffer it % 2 is read: the next prefetch may overwrite it
        }
    }
    // partial sums of this split into the fp32 accumulators
#pragma unroll
    for (int x = 0; x < 2; ++x) {
        if (!live[x]) continue;
        const int64_t row = aug_row(a, K, ki[x]);
        float *pk = a.dk32 + (row * a.Hkv + g) * D;
        float *pv = a.dv32 + (row * a.Hkv + g) * D;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            atomicAdd(pk + 8 * nt + 2 * tt, dk[nt][2 * x] * a.scale);
            atomicAdd(pk + 8 * nt + 2 * tt + 1, dk[nt][2 * x + 1] * a.scale);
            atomicAdd(pv + 8 * nt + 2 * tt, dv[nt][2 * x]);
            atomicAdd(pv + 8 * nt + 2 * tt + 1, dv[nt][2 * x + 1]);
        }
    }
}

// fp32 accumulators -> bf16 dk, dv of the real rows (padding rows untouched)
__global__ void __launch_bounds__(256) bwd_dkv_out_kernel(Args a, int D)
{
    if (*a.err != 0) return;   // the plan found cu_seqlens inconsistent: its rows may lie outside the buffers
    Blk K;
    if (!block_of(a, blockIdx.x, K)) return;
    const int g = blockIdx.y;
    for (int e = threadIdx.x; e < K.cnt * (D / 2); e += 256) {
        const int r = e / (D / 2), c2 = e % (D / 2);
        const int64_t off = (aug_row(a, K, K.idx0 + r) * a.Hkv + g) * D + 2 * c2;
        *reinterpret_cast<uint32_t *>(a.dk + off) = wm::pack2(a.dk32[off], a.dk32[off + 1]);
        *reinterpret_cast<uint32_t *>(a.dv + off) = wm::pack2(a.dv32[off], a.dv32[off + 1]);
    }
}

// The summary query rows of the tensor-core path and the output conversion,
// fused: one warp per (chunk, kv head).  Summary s_j (section 2.2.1, Figure
// 4c) attends to the k text rows of chunk j and to itself, i.e. exactly the
// k + 1 rows of the chunk; its G q heads give P and dS over those rows
// (CUDA cores, warp-wide dot products), dq of s_j = scale dS K, and the rows'
// dk += scale dS^T q_sj, dv += P^T dO_sj are added to the fp32 accumulators
// of the text query rows as they are converted to bf16.  Lane l holds
// columns [D/32 l, D/32 (l + 1)).  sm: [4 warps][P, dS][G][k + 1] floats.
template <int D>
__global__ void __launch_bounds__(128) bwd_sum_rows_kernel(Args a, int64_t chunks)
{
    constexpr int CPL = D / 32;
    extern __shared__ float bw_sum_sm[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t gc = (int64_t)blockIdx.x * 4 + warp;
    if (*a.err != 0 || gc >= chunks) return;   // warp-uniform; only warp-level syncs below
    const int g = blockIdx.y, K1 = a.k + 1, G = a.G;
    float *sP = bw_sum_sm + (size_t)warp * 2 * G * K1, *sS = sP + G * K1;
    const int b = find_seq(a.pl.chunk_off, a.batch, (int)gc);
    const int j = (int)(gc - a.pl.chunk_off[b]);
    const int n = a.cu[b + 1] - a.cu[b], m = n / a.k;
    if (j * a.k >= n) return;                  // past the sequence (a padding chunk cannot occur)
    const bool has_sum = j < m;
    const int64_t row0 = gc * K1, srow = row0 + a.k;
    const int col0 = lane * CPL;
    auto ld = [&](const __nv_bfloat16 *p, float *f) {
        if constexpr (CPL == 4) {
            const uint2 u = *reinterpret_cast<const uint2 *>(p);
            f[0] = __uint_as_float(u.x << 16); f[1] = __uint_as_float(u.x & 0xffff0000u);
            f[2] = __uint_as_float(u.y << 16); f[3] = __uint_as_float(u.y & 0xffff0000u);
        } else {
            const uint32_t u = *reinterpret_cast<const uint32_t *>(p);
            f[0] = __uint_as_float(u << 16); f[1] = __uint_as_float(u & 0xffff0000u);
        }
    };
    auto st = [&](__nv_bfloat16 *p, const float *f) {
        if constexpr (CPL == 4)
            *reinterpret_cast<uint2 *>(p) = make_uint2(wm::pack2(f[0], f[1]), wm::pack2(f[2], f[3]));
        else
            *reinterpret_cast<uint32_t *>(p) = wm::pack2(f[0], f[1]);
    };
    if (has_sum) {
        for (int r = 0; r < K1; ++r) {
            float kr[CPL], vr[CPL];
            ld(a.kk + ((row0 + r) * a.Hkv + g) * D + col0, kr);
            ld(a.v + ((row0 + r) * a.Hkv + g) * D + col0, vr);
            for (int hh = 0; hh < G; ++hh) {
                const int h = g * G + hh;
                float qv[CPL], ov[CPL];
                ld(a.q + (srow * a.Hq + h) * D + col0, qv);
                ld(a.dout + (srow * a.Hq + h) * D + col0, ov);
                float sc = 0.f, dp = 0.f;
#pragma unroll
                for (int c = 0; c < CPL; ++c) {
                    sc = fmaf(qv[c], kr[c], sc);
                    dp = fmaf(ov[c], vr[c], dp);
                }
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) {
                    sc += __shfl_xor_sync(0xffffffffu, sc, off);
                    dp += __shfl_xor_sync(0xffffffffu, dp, off);
                }
                const float pr = wm::ex2(sc * a.scale_log2 - a.lse[srow * a.Hq + h] * 1.4426950408889634f);
                if (lane == 0) {
                    sP[hh * K1 + r] = pr;
                    sS[hh * K1 + r] = pr * (dp - a.dsum[srow * a.Hq + h]);
                }
            }
        }
        __syncwarp();
        // dq of s_j, head by head
        for (int hh = 0; hh < G; ++hh) {
            float acc[CPL] = {};
            for (int r = 0; r < K1; ++r) {
                float kr[CPL];
                ld(a.kk + ((row0 + r) * a.Hkv + g) * D + col0, kr);
                const float w = sS[hh * K1 + r];
#pragma unroll
                for (int c = 0; c < CPL; ++c) acc[c] = fmaf(w, kr[c], acc[c]);
            }
#pragma unroll
            for (int c = 0; c < CPL; ++c) acc[c] *= a.scale;
            st(a.dq + (srow * a.Hq + g * G + hh) * D + col0, acc);
        }
    }
    // dk, dv of the chunk's real rows: its text rows, then s_j
    const int ntext = min(a.k, n - j * a.k);
    for (int r = 0; r < K1; ++r) {
        if (r < a.k ? r >= ntext : !has_sum) continue;
        const int64_t off = ((row0 + r) * a.Hkv + g) * D + col0;
        float dk[CPL], dv[CPL];
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            dk[c] = a.dk32[off + c];
            dv[c] = a.dv32[off + c];
        }
        if (has_sum) {
            for (int hh = 0; hh < G; ++hh) {
                const int h = g * G + hh;
                float qv[CPL], ov[CPL];
                ld(a.q + (srow * a.Hq + h) * D + col0, qv);
                ld(a.dout + (srow * a.Hq + h) * D + col0, ov);
                const float ws = sS[hh * K1 + r] * a.scale, wp = sP[hh * K1 + r];
#pragma unroll
                for (int c = 0; c < CPL; ++c) {
                    dk[c] = fmaf(ws, qv[c], dk[c]);
                    dv[c] = fmaf(wp, ov[c], dv[c]);
                }
            }
        }
        st(a.dk + off, dk);
        st(a.dv + off, dv);
    }
}

// The same for a compile-time G, in one pass over the chunk's rows: the
// summary row's q and dO of the G heads stay in registers, and each row r
// (loaded once, with its fp32 dk, dv accumulators) gives the G heads' P and
// dS, adds their dk, dv terms and its dS K term to the summary row's dq, and
// is written out.  The G heads' dot products reduce together (independent
// shuffle chains), and the next row's loads are issued before this row's
// arithmetic.
template <int D, int G>
__global__ void __launch_bounds__(128) bwd_sum_rows_g_kernel(Args a, int64_t chunks)
{
    constexpr int CPL = D / 32;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t gc = (int64_t)blockIdx.x * 4 + warp;
    if (*a.err != 0 || gc >= chunks) return;   // warp-uniform; only warp-level syncs below
    const int g = blockIdx.y, K1 = a.k + 1;
    const int b = find_seq(a.pl.chunk_off, a.batch, (int)gc);
    const int j = (int)(gc - a.pl.chunk_off[b]);
    const int n = a.cu[b + 1] - a.cu[b], m = n / a.k;
    if (j * a.k >= n) return;                  // past the sequence (a padding chunk cannot occur)
    const bool has_sum = j < m;
    const int ntext = min(a.k, n - j * a.k);
    const int64_t row0 = gc * K1, srow = row0 + a.k;
    const int col0 = lane * CPL;
    auto ld = [&](const __nv_bfloat16 *p, float *f) {
        if constexpr (CPL == 4) {
            const uint2 u = *reinterpret_cast<const uint2 *>(p);
            f[0] = __uint_as_float(u.x << 16); f[1] = __uint_as_float(u.x & 0xffff0000u);
            f[2] = __uint_as_float(u.y << 16); f[3] = __uint_as_float(u.y & 0xffff0000u);
        } else {
            const uint32_t u = *reinterpret_cast<const uint32_t *>(p);
            f[0] = __uint_as_float(u << 16); f[1] = __uint_as_float(u & 0xffff0000u);
        }
    };
    auto ld32 = [&](const float *p, float *f) {
        if constexpr (CPL == 4) {
            const float4 v = *reinterpret_cast<const float4 *>(p);
            f[0] = v.x; f[1] = v.y; f[2] = v.z; f[3] = v.w;
        } else {
            const float2 v = *reinterpret_cast<const float2 *>(p);
            f[0] = v.x; f[1] = v.y;
        }
    };
    auto st = [&](__nv_bfloat16 *p, const float *f) {
        if constexpr (CPL == 4)
            *reinterpret_cast<uint2 *>(p) = make_uint2(wm::pack2(f[0], f[1]), wm::pack2(f[2], f[3]));
        else
            *reinterpret_cast<uint32_t *>(p) = wm::pack2(f[0], f[1]);
    };
    // the summary row's q, dO, LSE (log2 units) and D of the G heads
    float qs[G][CPL], os[G][CPL], l2[G], dd[G], dq[G][CPL];
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
        const int h = g * G + hh;
#pragma unroll
        for (int c = 0; c < CPL; ++c) qs[hh][c] = os[hh][c] = dq[hh][c] = 0.f;
        l2[hh] = dd[hh] = 0.f;
        if (has_sum) {
            ld(a.q + (srow * a.Hq + h) * D + col0, qs[hh]);
            ld(a.dout + (srow * a.Hq + h) * D + col0, os[hh]);
            l2[hh] = a.lse[srow * a.Hq + h] * 1.4426950408889634f;
            dd[hh] = a.dsum[srow * a.Hq + h];
        }
    }
    // rows of the chunk that exist: its text rows, then s_j
    auto real = [&](int r) { return r < a.k ? r < ntext : has_sum; };
    float kr[CPL], vr[CPL], dkr[CPL], dvr[CPL];
    auto load_row = [&](int r) {
        const int64_t off = ((row0 + r) * a.Hkv + g) * D + col0;
        ld32(a.dk32 + off, dkr);
        ld32(a.dv32 + off, dvr);
        if (has_sum) {
            ld(a.kk + off, kr);
            ld(a.v + off, vr);
        }
    };
    int r = 0;
    while (r < K1 && !real(r)) ++r;
    if (r < K1) load_row(r);
    while (r < K1) {
        float k0[CPL], v0[CPL], dk0[CPL], dv0[CPL];
#pragma unroll
        for (int c = 0; c < CPL; ++c) { k0[c] = kr[c]; v0[c] = vr[c]; dk0[c] = dkr[c]; dv0[c] = dvr[c]; }
        int rn = r + 1;
        while (rn < K1 && !real(rn)) ++rn;
        if (rn < K1) load_row(rn);   // the next row's loads ahead of this row's arithmetic
        if (has_sum) {
            float sc[G], dp[G];
#pragma unroll
            for (int hh = 0; hh < G; ++hh) {
                sc[hh] = dp[hh] = 0.f;
#pragma unroll
                for (int c = 0; c < CPL; ++c) {
                    sc[hh] = fmaf(qs[hh][c], k0[c], sc[hh]);
                    dp[hh] = fmaf(os[hh][c], v0[c], dp[hh]);
                }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1)
#pragma unroll
                for (int hh = 0; hh < G; ++hh) {
                    sc[hh] += __shfl_xor_sync(0xffffffffu, sc[hh], off);
                    dp[hh] += __shfl_xor_sync(0xffffffffu, dp[hh], off);
                }
#pragma unroll
            for (int hh = 0; hh < G; ++hh) {
                const float pr = wm::ex2(sc[hh] * a.scale_log2 - l2[hh]);
                const float ds = pr * (dp[hh] - dd[hh]);
                const float ws = ds * a.scale;
#pragma unroll
                for (int c = 0; c < CPL; ++c) {
                    dq[hh][c] = fmaf(ds, k0[c], dq[hh][c]);
                    dk0[c] = fmaf(ws, qs[hh][c], dk0[c]);
                    dv0[c] = fmaf(pr, os[hh][c], dv0[c]);
                }
            }
        }
        const int64_t off = ((row0 + r) * a.Hkv + g) * D + col0;
        st(a.dk + off, dk0);
        st(a.dv + off, dv0);
        r = rn;
    }
    if (has_sum)
#pragma unroll
        for (int hh = 0; hh < G; ++hh) {
#pragma unroll
            for (int c = 0; c < CPL; ++c) dq[hh][c] *= a.scale;
            st(a.dq + (srow * a.Hq + g * G + hh) * D + col0, dq[hh]);
        }
}

// per-sequence block counts: text blocks ceil(n/64), summary blocks ceil(m/64)
__global__ void bwd_blocks_kernel(int batch, const int32_t *cu, int k, int32_t *tb_off, int32_t *sb_off)
{
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    int t = 0, s = 0;
    for (int b = 0; b < batch; ++b) {
        tb_off[b] = t;
        sb_off[b] = s;
        const int n = max(cu[b + 1] - cu[b], 0);
        t += (n + RB - 1) / RB;
        s += (n / k + RB - 1) / RB;
    }
    tb_off[batch] = t;
    sb_off[batch] = s;
}

}  // namespace bw

// four 64-row tiles of D + 8 bf16 per row (+ per-query LSE and D for dk, dv)
// Summary query rows and the output conversion after the tensor-core kernels.
template <int D>
static int bw_sum_launch(const bw::Args &a, int64_t chunks, cudaStream_t st)
{
    const size_t smem = (size_t)4 * 2 * a.G * (a.k + 1) * sizeof(float);
    if (smem > 48 * 1024) {
        static size_t attr = 0;
        if (smem > attr) {
            if (cudaFuncSetAttribute(bw::bwd_sum_rows_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)smem) != cudaSuccess)
                return KSA_ERR_UNSUPPORTED;
            attr = smem;
        }
    }
    const dim3 grid((unsigned)((chunks + 3) / 4), a.Hkv);
    switch (a.G) {
    case 1: bw::bwd_sum_rows_g_kernel<D, 1><<<grid, 128, 0, st>>>(a, chunks); break;
    case 2: bw::bwd_sum_rows_g_kernel<D, 2><<<grid, 128, 0, st>>>(a, chunks); break;
    case 4: bw::bwd_sum_rows_g_kernel<D, 4><<<grid, 128, 0, st>>>(a, chunks); break;
    case 8: bw::bwd_sum_rows_g_kernel<D, 8><<<grid, 128, 0, st>>>(a, chunks); break;
    default: bw::bwd_sum_rows_kernel<D><<<grid, 128, smem, st>>>(a, chunks); break;
    }
    return KSA_OK;
}

template <int D>
static int bw_launch(const bw::Args &a, int64_t nblk, int64_t zsplits, cudaStream_t st)
{
    const int tiles = 6 * bw::RB * (D + 8) * 2;              // Q, dO + two (K, V) / K, V + two (Q, dO)
    const int dkv = tiles + 2 * 2 * bw::RB * 4;               // + two (LSE, D)
    static bool attr[2] = {false, false};
    if (!attr[D == 128]) {
        if (cudaFuncSetAttribute(bw::bwd_dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, tiles) !=
                cudaSuccess ||
            cudaFuncSetAttribute(bw::bwd_dkv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, dkv) != cudaSuccess)
            return KSA_ERR_CUDA;
        attr[D == 128] = true;
    }
    bw::bwd_dq_kernel<D><<<dim3((unsigned)nblk, a.Hq), bw::kThreads, tiles, st>>>(a);
    bw::bwd_dkv_kernel<D><<<dim3((unsigned)nblk, a.Hkv, (unsigned)zsplits), bw::kThreads, dkv, st>>>(a);
    bw::bwd_dkv_out_kernel<<<dim3((unsigned)nblk, a.Hkv), 256, 0, st>>>(a, D);
    return KSA_OK;
}

size_t prefill_bwd_workspace_bytes(const ksa_params *p, int batch, int64_t aug_rows)
{
    return plan_bytes(batch) + 2 * align_up(sizeof(int32_t) * (size_t)(batch + 1)) +
           align_up(sizeof(float) * (size_t)aug_rows * p->num_q_heads) +
           2 * align_up(sizeof(float) * (size_t)aug_rows * p->num_kv_heads * p->head_dim) +
           prefill_bwd_tc_workspace_bytes(batch, aug_rows);
}

int launch_prefill_bwd(const ksa_params *p, int batch, const int32_t *cu, int64_t total_text, int64_t aug_rows,
                       const void *q, const void *k, const void *v, const void *o, const float *lse, const void *dout,
                       void *dq, void *dk, void *dv, void *ws, const Plan &pl, int32_t *err, cudaStream_t st)
{
    if (aug_rows == 0) return KSA_OK;
    char *w = static_cast<char *>(ws) + plan_bytes(batch);
    const size_t ab = align_up(sizeof(int32_t) * (size_t)(batch + 1));
    bw::Args a;
    a.tb_off = reinterpret_cast<int32_t *>(w);
    a.sb_off = reinterpret_cast<int32_t *>(w + ab);
    a.dsum = reinterpret_cast<float *>(w + 2 * ab);
    const size_t dsb = align_up(sizeof(float) * (size_t)aug_rows * p->num_q_heads);
    const size_t accb = align_up(sizeof(float) * (size_t)aug_rows * p->num_kv_heads * p->head_dim);
    a.dk32 = reinterpret_cast<float *>(w + 2 * ab + dsb);
    a.dv32 = reinterpret_cast<float *>(w + 2 * ab + dsb + accb);
    if (cudaMemsetAsync(a.dk32, 0, 2 * accb, st) != cudaSuccess) return KSA_ERR_CUDA;
    a.k = p->k; a.w = p->w; a.Hq = p->num_q_heads; a.Hkv = p->num_kv_heads; a.G = a.Hq / a.Hkv; a.batch = batch;
    a.scale = p->scale > 0.f ? p->scale : 1.0f / sqrtf((float)p->head_dim);
    a.scale_log2 = a.scale * 1.4426950408889634f;
    a.cu = cu; a.pl = pl; a.err = err;
    a.q = (const __nv_bfloat16 *)q; a.kk = (const __nv_bfloat16 *)k; a.v = (const __nv_bfloat16 *)v;
    a.o = (const __nv_bfloat16 *)o; a.dout = (const __nv_bfloat16 *)dout; a.lse = lse;
    a.dq = (__nv_bfloat16 *)dq; a.dk = (__nv_bfloat16 *)dk; a.dv = (__nv_bfloat16 *)dv;
    bw::bwd_blocks_kernel<<<1, 32, 0, st>>>(batch, cu, p->k, const_cast<int32_t *>(a.tb_off),
                                            const_cast<int32_t *>(a.sb_off));
    const int64_t cells = aug_rows * a.Hq;
    if (p->head_dim == 128)
        bw::bwd_dot_kernel<128><<<(unsigned)((cells * 16 + 255) / 256), 256, 0, st>>>(a, cells);
    else
        bw::bwd_dot_kernel<64><<<(unsigned)((cells * 8 + 255) / 256), 256, 0, st>>>(a, cells);
    // upper bound of the block count; CTAs past the real count exit
    const int64_t nblk = total_text / bw::RB + (total_text / p->k) / bw::RB + 2LL * batch;
    if (nblk > 0x7fffffffLL) return KSA_ERR_UNSUPPORTED;
    a.nblk = (int)nblk;
    // query blocks any key block can meet: at most total_text/64 + 2 (text + one summary block)
    const int64_t zsplits = (total_text / bw::RB + 2 + bw::QB_SPLIT - 1) / bw::QB_SPLIT;
    if (zsplits > 65535) return KSA_ERR_UNSUPPORTED;
    // dq, dk, dv of the text query rows on the tensor-core kernels where the
    // shape allows, then the summary query rows fused with the conversion;
    // otherwise the warp-level passes take every row
    if (prefill_bwd_tc_supported(p)) {
        const int r = launch_prefill_bwd_tc(p, batch, cu, total_text, aug_rows, q, k, v, dout, lse, a.dsum, a.dk32,
                                            a.dv32, dq, w + 2 * ab + dsb + 2 * accb, pl, err, st);
        if (r != KSA_OK) return r;
        const int64_t chunks = aug_rows / (p->k + 1);
        const int rs = p->head_dim == 128 ? bw_sum_launch<128>(a, chunks, st) : bw_sum_launch<64>(a, chunks, st);
        if (rs != KSA_OK) return rs;
        return cudaGetLastError() == cudaSuccess ? KSA_OK : KSA_ERR_CUDA;
    }
    if (p->head_dim == 128) {
        if (bw_launch<128>(a, nblk, zsplits, st) != KSA_OK) return KSA_ERR_CUDA;
    } else if (p->head_dim == 64) {
        if (bw_launch<64>(a, nblk, zsplits, st) != KSA_OK) return KSA_ERR_CUDA;
    } else {
        return KSA_ERR_UNSUPPORTED;
    }
    return cudaGetLastError() == cudaSuccess ? KSA_OK : KSA_ERR_CUDA;
}

}  // namespace ksa

// warp_mma.cuh -- warp-level tensor-core helpers shared by the decode, the
// summary-row, the backward and the chunked-prefill kernels (mma.sync
// m16n8k16, bf16 inputs, fp32 accumulate; ldmatrix and cp.async staging).
//
// Fragment layout of m16n8k16 (row.col), lane = 4 g + t:
//   A (16x16): a0 = (row g, cols 2t, 2t+1), a1 = (row g+8, same cols),
//              a2 = (row g, cols 2t+8, 2t+9), a3 = (row g+8, cols 2t+8, 2t+9);
//   B (16x8):  b0 = (rows 2t, 2t+1, col g), b1 = (rows 2t+8, 2t+9, col g);
//   C (16x8):  c0, c1 = (row g, cols 2t, 2t+1), c2, c3 = (row g+8, same cols).
// The lower half of each 32-bit register holds the element of lower index.
#pragma once

#include <cuda_bf16.h>
#include <stdint.h>

namespace ksa {
namespace wm {

// D += A B
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// 8x8 b16 transpose across the warp, in registers
__device__ __forceinline__ uint32_t movtrans(uint32_t x)
{
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

__device__ __forceinline__ uint32_t word(const uint4 &u, int i)
{
    return i == 0 ? u.x : i == 1 ? u.y : i == 2 ? u.z : u.w;
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// ---- shared-memory staging -------------------------------------------------
__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gmem_src)
{
    const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void *p)
{
    const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(p));
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(a));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void *p)
{
    const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(p));
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(a));
}

// Tiles in shared memory are row-major bf16 with a row pitch of D + 8
// elements: the 16-byte pad keeps ldmatrix's 8-row reads conflict-free.

// A fragment (16 rows x 16 cols) at (row0, col0) of a row-major tile
template <int D>
__device__ __forceinline__ void frag_a(uint32_t (&r)[4], const __nv_bfloat16 (*t)[D + 8], int row0, int col0)
{
    const int l = threadIdx.x & 31;
    ldsm_x4(r, &t[row0 + (l & 7) + 8 * ((l >> 3) & 1)][col0 + 8 * (l >> 4)]);
}

// B fragments of two n-tiles from a tile stored [n][k] (rows = n): n-tiles
// n0 .. n0+7 and n0+8 .. n0+15, k-chunk k0 .. k0+15.  r = {b0, b1 of the
// first n-tile, b0, b1 of the second}.
template <int D>
__device__ __forceinline__ void frag_b_nk(uint32_t (&r)[4], const __nv_bfloat16 (*t)[D + 8], int n0, int k0)
{
    const int l = threadIdx.x & 31;
    ldsm_x4(r, &t[n0 + (l & 7) + 8 * (l >> 4)][k0 + 8 * ((l >> 3) & 1)]);
}

// B fragments of two n-tiles from a tile stored [k][n] (rows = k): k-chunk
// k0 .. k0+15, n-tiles n0 .. n0+7 and n0+8 .. n0+15 (transposing load).
template <int D>
__device__ __forceinline__ void frag_b_kn(uint32_t (&r)[4], const __nv_bfloat16 (*t)[D + 8], int k0, int n0)
{
    const int l = threadIdx.x & 31;
    ldsm_x4_t(r, &t[k0 + (l & 7) + 8 * ((l >> 3) & 1)][n0 + 8 * (l >> 4)]);
}

}  // namespace wm
}  // namespace ksa

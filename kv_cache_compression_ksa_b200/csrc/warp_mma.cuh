// warp_mma.cuh -- warp-level tensor-core helpers shared by the decode and the
// summary-row kernels (mma.sync m16n8k16, bf16 inputs, fp32 accumulate).
//
// Fragment layout of m16n8k16 (row.col), lane = 4 g + t:
//   A (16x16): a0 = (row g, cols 2t, 2t+1), a1 = (row g+8, same cols),
//              a2 = (row g, cols 2t+8, 2t+9), a3 = (row g+8, cols 2t+8, 2t+9);
//   B (16x8):  b0 = (rows 2t, 2t+1, col g), b1 = (rows 2t+8, 2t+9, col g);
//   C (16x8):  c0, c1 = (row g, cols 2t, 2t+1), c2, c3 = (row g+8, same cols).
// The lower half of each 32-bit register holds the element of lower index.
#pragma once

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

}  // namespace wm
}  // namespace ksa

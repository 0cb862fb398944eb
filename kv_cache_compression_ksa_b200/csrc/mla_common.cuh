// mla_common.cuh -- what the two MLA decode kernels share: the latent row
// shape, the launch arguments, and the tensor-core kernel's entry point.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ksa {
namespace mla {

constexpr int DC = 512, DR = 64, DL = DC + DR;   // latent, RoPE key, row

struct Args {
    int k, w, H, batch, splits;
    int64_t S, per;                  // slots per sequence; slots per share (multiple of the kernel's block)
    float scale_log2;
    double log2_theta;
    int rotate;
    const int8_t *kind;
    int32_t *state;
    const __nv_bfloat16 *lat;        // [B, S, DL]
    const __nv_bfloat16 *q;          // [B, H, DL], d_r part not rotated
    float *part_o;                   // [splits, B, H, DC]
    float *part_ml;                  // [splits, B, H, 2] (max in log2 units, sum)
    __nv_bfloat16 *o;                // [B, H, DC]
    float *lse;                      // [B, H] or null
};

// Slots per block of the tensor-core kernel (a share is a multiple of it).
constexpr int kTcBlock = 64;

// The tensor-core kernel for head groups of 128 (H a multiple of 128):
// grid (2 x splits, H / 128, batch) in clusters of two CTAs.
int launch_mla_tc(const Args &a, cudaStream_t st);

}  // namespace mla
}  // namespace ksa

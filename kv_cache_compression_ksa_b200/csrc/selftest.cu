// selftest.cu -- ksa_selftest_wait_timeout: runs the library's bounded-wait
// error path on the GPU, on purpose.
//
// Every pipeline wait of the tensor-core kernels (prefill, backward, MLA
// decode) is bounded: when a phase does not complete in time the waiting
// role records KSA_ERR_TIMEOUT in the caller's error word, raises the CTA's
// abort flag so the other roles stop waiting too, and the CTA frees its
// tensor memory and exits, leaving the context usable.  This kernel builds
// the same situation in miniature with the same wait routines: one CTA
// allocates the full 512 TMEM columns (as the prefill does), two roles wait
// on mbarriers that nothing ever arrives on -- one polling, one sleeping in
// mbarrier.try_wait -- with small limits, and the CTA then tears down
// exactly as the pipelines do.  A caller (the GPU test) checks that the call
// returns, that the error word says KSA_ERR_TIMEOUT, and that a following
// prefill, which needs all of an SM's TMEM, runs.
//
// Grid: one CTA of 128 threads.  Its waits end after at most poll_limit
// polls and sleep_limit sleeps of at most 20 us each (both capped at the
// pipelines' own limits).
#include "ksa_internal.cuh"
#include "tc_sm100.cuh"

namespace ksa {

namespace st {

constexpr int kThreads = 128;
constexpr uint32_t kTmemCols = 512;

__global__ void __launch_bounds__(kThreads, 1) wait_timeout_kernel(int32_t *err, uint32_t poll_limit,
                                                                    uint32_t sleep_limit)
{
    __shared__ __align__(8) uint64_t bars[2];
    __shared__ uint32_t tmem_slot;
    __shared__ int abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int *abort = &abort_flag;
    if (threadIdx.x == 0) {
        tc::mbar_init(tc::smem_u32(&bars[0]), 1);
        tc::mbar_init(tc::smem_u32(&bars[1]), 1);
        *abort = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         tc::smem_u32(&tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    const uint32_t tmem = tmem_slot;
    if (warp == 1 && lane == 0) {
        // a consumer polling for a phase that never completes
        tc::mbar_wait(tc::smem_u32(&bars[0]), 0, abort, err, poll_limit);
    } else if (warp == 2 && lane == 0) {
        // a producer sleeping in try_wait: it leaves on the abort flag the
        // first role raised, or at its own limit
        tc::mbar_wait_sleep(tc::smem_u32(&bars[1]), 0, abort, err, sleep_limit);
    }
    // teardown, as in the pipelines: every role is out of its loop
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    if (warp == 0) {
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                     : "memory");
    }
}

}  // namespace st

}  // namespace ksa

using namespace ksa;

extern "C" KSA_API int ksa_selftest_wait_timeout(uint32_t poll_limit, uint32_t sleep_limit, int32_t *dev_err,
                                                 void *stream)
{
    if (!dev_err || (reinterpret_cast<uintptr_t>(dev_err) & 3u)) return KSA_ERR_INVALID;
    if (poll_limit < 1 || poll_limit > tc::kSpinLimit) return KSA_ERR_INVALID;
    if (sleep_limit < 1 || sleep_limit > tc::kWaitLimit) return KSA_ERR_INVALID;
    st::wait_timeout_kernel<<<1, st::kThreads, 0, (cudaStream_t)stream>>>(dev_err, poll_limit, sleep_limit);
    return cudaGetLastError() == cudaSuccess ? KSA_OK : KSA_ERR_CUDA;
}

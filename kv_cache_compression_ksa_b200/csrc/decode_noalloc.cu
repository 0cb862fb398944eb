// decode_noalloc.cu -- ksa_decode_noalloc: the split-K decode with its
// scratch in a fixed device array of this library, for callers that cannot
// allocate device memory.
//
// Who needs it: a decode step plugged into a host program that owns all
// device memory (a serving engine that reserves the GPU's HBM for its KV
// pools up front, or a framework custom op that is handed only its inputs
// and outputs) has nowhere to get a workspace from, and a cudaMalloc of its
// own would both break that ownership and synchronise the device in the
// middle of the decode loop.  This entry point takes the same inputs and
// outputs as ksa_decode but no workspace: the split-K partial results live
// in kScratchBytes of device memory that the library holds as a static
// array, present on every GPU that loads the library until the process exits.
//
// The report has no counterpart to this call; it exists for callers of the
// library, not for the method.
#include <mutex>

#include "ksa_internal.cuh"

namespace ksa {

// 4 MiB.  One split of the partials (m, l and the d-wide accumulator of
// every q head) takes 4 B x batch x Hq x (d + 2): 1.02 MiB for 64 sequences
// x 32 q heads at d = 128, 0.25 MiB for 16 of them.  The call keeps as many
// of ksa_decode's splits as fit (3 and 15 for those two batches) and
// refuses only a batch whose single split does not fit (batch x Hq x (d + 2)
// above 1 Mi floats).
constexpr size_t kScratchBytes = 4u << 20;

static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

// Device address of g_decode_scratch on each device, looked up once per
// device (with that device current) on the first call made on it.
static void *g_scratch_ptr[64];
static std::mutex g_scratch_mu;

static int scratch_for_current_device(void **out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return KSA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_decode_scratch) != cudaSuccess || !p) return KSA_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return KSA_OK;
}

}  // namespace ksa

using namespace ksa;

extern "C" KSA_API int ksa_decode_noalloc(const ksa_params *p, const ksa_cache *cache, const int8_t *kind,
                                          const void *q, void *o, float *lse, int64_t max_text, void *stream)
{
    // the same argument checks, in the same order, as ksa_decode
    int rc = check_decode_args(p, cache, kind, q, o, lse, max_text);
    if (rc != KSA_OK) return rc;
    if (cache->batch == 0) return KSA_OK;
    // as many of ksa_decode's splits as the fixed scratch holds
    const size_t per_split = decode_split_bytes(p, cache->batch);
    if (per_split > kScratchBytes) return KSA_ERR_CAPACITY;
    int nsplit = decode_splits(p, cache->batch, max_text);
    if ((size_t)nsplit * per_split > kScratchBytes) nsplit = (int)(kScratchBytes / per_split);
    void *scratch = nullptr;
    rc = scratch_for_current_device(&scratch);
    if (rc != KSA_OK) return rc;
    return launch_decode_splits(p, cache, kind, q, o, lse, nsplit, scratch, (cudaStream_t)stream);
}

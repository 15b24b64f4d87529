// nvfp4_kv_append_noalloc: the quantize-append for callers that cannot
// allocate device memory.
//
// The regular nvfp4_kv_append needs one small caller-allocated scratch plane,
// cache->amax, where the first append reduces the chunk's per-head absolute
// maximum before the global scales are fixed.  Some callers cannot create
// even that: an inference-engine plugin whose enqueue step is not allowed to
// allocate, or a process whose device memory is entirely owned by another
// allocator.  This entry point takes the same inputs and outputs but keeps the
// amax scratch in a fixed-size array that lives in the library's own device
// image (loaded with the library; every GPU that loads it keeps the array
// until the process exits).  It calls no cudaMalloc / cudaFree.
//
// Limits and rules:
//  - at most 256 (b, h) pairs: B * H <= 256
//    (2 * 256 words = 2 KiB of scratch);
//  - the first call on each device looks up the array's device address
//    (cudaGetSymbolAddress) with that device current and keeps it for the
//    process; make that first call before any stream capture.  A
//    cudaDeviceReset of that device invalidates the kept address (the module
//    may load elsewhere in the new context): do not call this entry point
//    again on that device after a reset;
//  - every call on a device shares the one array and leaves its last contents
//    there; a scale-fixing (first) append clears it before use.  Calls whose
//    work overlaps on the GPU (two streams, or two threads) race on it:
//    serialise them.
// Validation, slot assignment, the launch and the ring update are those of
// nvfp4_kv_append (the shared host path), with the array as the scratch.
#include <mutex>

#include "nvkv_internal.h"

namespace {

constexpr int kMaxHeads = 256;
constexpr int kMaxDevices = 64;

static __device__ __align__(256) uint32_t g_amax_scratch[2 * kMaxHeads];

std::mutex g_setup_mu;
uint32_t *g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device; set up on the
// first call per device.
cudaError_t scratch_for_current_device(uint32_t **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_setup_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_amax_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_ptr[dev] = static_cast<uint32_t *>(p);
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" nvkv_status nvfp4_kv_append_noalloc(const nvkv_desc *desc, const nvkv_cache *cache,
                                               nvkv_ring *ring, const void *k, const void *v,
                                               nvkv_stream stream)
{
    if (!desc) return NVKV_ERR_INVALID_ARG;
    if ((int64_t)desc->B * desc->H > kMaxHeads) return NVKV_ERR_UNSUPPORTED;
    uint32_t *scratch = nullptr;
    if (scratch_for_current_device(&scratch) != cudaSuccess) return NVKV_ERR_CUDA;
    // the launcher clears the scratch before a scale-fixing append uses it
    return nvkv::nvfp4_append_with_scratch(desc, cache, ring, k, v, (cudaStream_t)stream, scratch);
}

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
//  - at most NVKV_NOALLOC_MAX_HEADS (b, h) pairs: B * H <= 256
//    (2 * 256 words = 2 KiB of scratch);
//  - the first call on each device looks up the array's device address
//    (cudaGetSymbolAddress) with that device current; make that first call
//    before any stream capture;
//  - every call on a device shares the one array and leaves its last contents
//    there; a scale-fixing (first) append clears it before use.  Calls whose
//    work overlaps on the GPU (two streams, or two threads) race on it:
//    serialise them.
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

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" nvkv_status nvfp4_kv_append_noalloc(const nvkv_desc *desc, const nvkv_cache *cache,
                                               nvkv_ring *ring, const void *k, const void *v,
                                               nvkv_stream stream)
{
    if (!desc || !ring) return NVKV_ERR_INVALID_ARG;
    if (desc->magic != NVKV_MAGIC || desc->version != NVKV_VERSION) return NVKV_ERR_STATE;
    if (desc->kv_dtype != NVKV_KV_NVFP4) return NVKV_ERR_STATE;
    if ((int64_t)desc->B * desc->H > kMaxHeads) return NVKV_ERR_UNSUPPORTED;
    if (!cache || !k || !v || !cache->k_data || !cache->v_data || !cache->k_scales ||
        !cache->v_scales || !cache->s_g)
        return NVKV_ERR_INVALID_ARG;
    if (!aligned16(k) || !aligned16(v) || !aligned16(cache->k_data) ||
        !aligned16(cache->v_data) || !aligned16(cache->k_scales) || !aligned16(cache->v_scales))
        return NVKV_ERR_ALIGNMENT;

    // the ring update an append performs, on a copy (validates desc and ring)
    nvkv_ring next = *ring;
    int32_t slots[NVKV_MAX_BATCH * NVKV_MAX_CHUNK];
    const int first = ring->scales_fixed ? 0 : 1;
    nvkv_status st = nvkv_ring_push_chunk(desc, &next, slots);
    if (st != NVKV_OK) return st;

    uint32_t *scratch = nullptr;
    if (scratch_for_current_device(&scratch) != cudaSuccess) return NVKV_ERR_CUDA;

    nvkv::AppendLaunch a{};
    for (int i = 0; i < desc->B * desc->C; ++i) a.slot[i] = slots[i];
    a.k = k;
    a.v = v;
    a.k_data = cache->k_data;
    a.v_data = cache->v_data;
    a.k_scales = cache->k_scales;
    a.v_scales = cache->v_scales;
    a.amax = scratch;                 // cleared by the launcher when first != 0
    a.s_g = cache->s_g;
    a.B = desc->B;
    a.H = desc->H;
    a.T = desc->grid_h * desc->grid_w;
    a.Lq = desc->C * a.T;
    a.Ts = nvkv::shard_tokens(desc);
    a.tok_off = nvkv::shard_first_token(desc);
    a.R = a.Ts * (desc->S + desc->W);
    a.C = desc->C;
    a.first = first;
    if (nvkv::launch_nvfp4_append(a, (cudaStream_t)stream) != cudaSuccess) return NVKV_ERR_CUDA;
    *ring = next;
    return NVKV_OK;
}

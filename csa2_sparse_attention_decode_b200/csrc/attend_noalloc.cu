// csa2_attend_noalloc: the attention call for callers that cannot allocate
// device memory.
//
// csa2_attend needs a caller-provided workspace for the per-split partial
// results.  Some callers have no way to provide one: code embedded in a host
// framework that owns every byte of device memory through its own pool and
// offers plugins no allocation hook, or a serving loop that must not allocate
// once it is running (an allocation can synchronise the device and stall
// every stream).  This entry point keeps the partials in a fixed array that
// is part of the library itself, so the caller passes only inputs and
// outputs.  It launches the attention variant that exchanges its split
// partials through global memory (csa2_attend merges them on chip instead).
#include <mutex>

#include "common.cuh"
#include "index.cuh"

namespace {

constexpr size_t kPartO = (size_t)CSA2_ATTEND_NOALLOC_MAX_ROWS * csa2::ATT_SPLITS * CSA2_LATENT;

// One copy per GPU that loads the library, held until the process exits.
// Host code must not use this name as a pointer: on the host it is only a
// stand-in, and its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) float g_attend_scratch[kPartO];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
float *g_scratch_addr[kMaxDevices] = {};

bool aligned_to(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

// Device address of the scratch array on the current device, resolved once
// per device with that device current.
cudaError_t scratch_address(float **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_scratch_addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_attend_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev] = static_cast<float *>(p);
    }
    *out = g_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" csa2_status csa2_attend_noalloc(const csa2_cache *cache, int32_t heads, const uint16_t *q,
                                           const int32_t *topk, float scale, void *out, int32_t out_is_fp32,
                                           csa2_stream_t stream)
{
    CSA2_TRACE("csa2_attend_noalloc");
    const csa2_status st = csa2::check_cache(cache);
    if (st != CSA2_OK) return st;
    if (heads <= 0 || heads > 128 || !q || !topk || !out || !aligned_to(out, 16) || !aligned_to(q, 16))
        return CSA2_ERR_INVALID_ARG;
    // The fixed array holds the partials of at most this many (request, head) rows.
    if ((int64_t)cache->batch * heads > CSA2_ATTEND_NOALLOC_MAX_ROWS) return CSA2_ERR_UNSUPPORTED;
    float *scratch = nullptr;
    if (scratch_address(&scratch) != cudaSuccess) return CSA2_ERR_CUDA;
    // Every partial the combine step reads is written by this same call, so
    // nothing left over from an earlier call needs clearing.
    cudaError_t e = csa2::launch_attend_umma(csa2::make_view(cache), heads, q, topk, scale, out, out_is_fp32, 0u,
                                             scratch, (cudaStream_t)stream);
    return e == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA;
}

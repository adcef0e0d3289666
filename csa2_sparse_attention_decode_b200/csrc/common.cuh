// Device-side helpers shared by the libcsa2 kernels: number formats, page
// addressing and the device error word.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>
#include <utility>

#include <nvtx3/nvToolsExt.h>

#include "../../include/csa2.h"

namespace csa2 {

// ---------------------------------------------------------------- tracing
// An NVTX range around each C-ABI call, named after the call, so a profiler's
// timeline shows which call enqueued which kernels (NVTX costs nothing when
// no tool is attached).
struct TraceRange {
    explicit TraceRange(const char *name) { nvtxRangePushA(name); }
    ~TraceRange() { nvtxRangePop(); }
    TraceRange(const TraceRange &) = delete;
    TraceRange &operator=(const TraceRange &) = delete;
};
#define CSA2_TRACE(name) ::csa2::TraceRange csa2_trace_range_(name)

// ---------------------------------------------------------------- diagnostics
// Defined in capi.cu: launch counting and optional event brackets.
void note_launch(int kernel, cudaStream_t st, bool before);

struct LaunchScope {
    int k;
    cudaStream_t st;
    LaunchScope(int kernel, cudaStream_t s) : k(kernel), st(s) { note_launch(k, st, true); }
    ~LaunchScope() { note_launch(k, st, false); }
};

// ---------------------------------------------------------------- one-time set-up
// Per-device set-up of a launcher (function attributes, occupancy queries)
// that host threads may reach concurrently: the first caller on a device runs
// init under a lock; values init stores for that device are visible to every
// caller that sees the flag set.
struct DeviceOnce {
    static constexpr int N = 64;
    std::atomic<bool> done[N] = {};
    std::mutex mu;
    template <class F>
    cudaError_t run(int dev, F &&init)
    {
        if (dev < 0 || dev >= N) return cudaErrorInvalidDevice;
        if (done[dev].load(std::memory_order_acquire)) return cudaSuccess;
        std::lock_guard<std::mutex> lk(mu);
        if (done[dev].load(std::memory_order_relaxed)) return cudaSuccess;
        const cudaError_t e = init();
        if (e == cudaSuccess) done[dev].store(true, std::memory_order_release);
        return e;
    }
};

// ---------------------------------------------------------------- launch order
// Programmatic dependent launch: every kernel lets the next one in the
// stream start its launch and set-up early, and waits for the previous one
// (completion and memory) before touching anything it may have written.
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void allow_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
// Cluster-wide barrier of every thread of every CTA of the cluster, in the
// warp-aligned form (each warp arrives as one); every thread of each warp
// must reach it together.  Release / acquire at cluster scope, as
// cooperative_groups' cluster sync.
__device__ __forceinline__ void cluster_sync_aligned()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// A hint that brings the 128-byte line holding p into L2; it reads nothing
// into the program, so it may run before griddepcontrol.wait: L2 is the
// point of coherence, and the loads after the wait still see the producer's
// writes.
__device__ __forceinline__ void prefetch_l2(const void *p) { asm volatile("prefetch.global.L2 [%0];" ::"l"(p)); }
// Lanes of one warp hint the lines of bytes [lo, hi) of buf, at most
// max_lines lines per lane.
__device__ __forceinline__ void prefetch_l2_range(const void *buf, size_t lo, size_t hi, int lane, int max_lines)
{
    const char *b = static_cast<const char *>(buf);
    lo &= ~(size_t)127;
    for (int k = 0; k < max_lines; ++k) {
        const size_t off = lo + ((size_t)k * 32 + lane) * 128;
        if (off >= hi) break;
        prefetch_l2(b + off);
    }
}

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// The same, for a kernel launched in thread-block clusters of cluster_x CTAs
// (sizes above 8 need cudaFuncAttributeNonPortableClusterSizeAllowed).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                      int cluster_x, Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = (unsigned)cluster_x;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// How many clusters of cluster_x CTAs of this shape `kernel` can have
// resident at once on the current device (0 if none fits, or on error).
template <typename... KArgs>
inline int max_active_clusters(void (*kernel)(KArgs...), dim3 block, size_t smem, int cluster_x)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(cluster_x, 1, 1);
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)cluster_x;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, (void *)kernel, &cfg) != cudaSuccess) {
        cudaGetLastError();
        return 0;
    }
    return n;
}

// ---------------------------------------------------------------- errors
__device__ __forceinline__ void set_error(int32_t *err, int32_t code)
{
    if (err) atomicCAS(err, 0, code);
}

// ---------------------------------------------------------------- formats
// e4m3 with round-to-nearest-even and saturation to +-448 (the fp8 KV /
// indexer-key format of the CSA2 config).
__device__ __forceinline__ uint8_t f32_to_e4m3(float x)
{
    return (uint8_t)__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3);
}

__device__ __forceinline__ float e4m3_to_f32(uint8_t c)
{
    __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)c, __NV_E4M3);
    return __half2float(__half(h));
}

// e2m1 magnitude code of a = |x| with round-to-nearest, ties to the even code
// (magnitudes 0, .5, 1, 1.5, 2, 3, 4, 6; saturating).  Ties sit at the
// midpoints .25 .75 1.25 1.75 2.5 3.5 5: a tie goes up exactly when the upper
// neighbour has the even code.
__device__ __forceinline__ uint32_t e2m1_mag_code(float a)
{
    return (uint32_t)(a > 0.25f) + (uint32_t)(a >= 0.75f) + (uint32_t)(a > 1.25f) +
           (uint32_t)(a >= 1.75f) + (uint32_t)(a > 2.5f) + (uint32_t)(a >= 3.5f) +
           (uint32_t)(a > 5.0f);
}

__device__ __forceinline__ uint32_t f32_to_e2m1(float x)
{
    uint32_t sign = (__float_as_uint(x) >> 31) << 3;
    return sign | e2m1_mag_code(fabsf(x));
}

// Smallest integer e with amax <= 448 * 2^e (amax > 0, finite).
__device__ __forceinline__ int swa_exponent(float amax)
{
    int ex;
    float f = frexpf(amax, &ex);          // amax = f * 2^ex, f in [0.5, 1)
    return (f > 0.875f) ? ex - 8 : ex - 9;
}

// ---------------------------------------------------------------- layout
struct CacheView {
    uint8_t *pool;
    uint8_t *codes, *scales, *keys, *summ;     // the four planes of the pool
    int32_t n_pages;
    const int32_t *page_table;
    int32_t max_pages;
    int32_t *n_tokens;
    const int32_t *m;
    uint8_t *swa;
    float *pending;
    int32_t *error;
    int32_t batch;
};

__host__ inline CacheView make_view(const csa2_cache *c)
{
    CacheView v;
    v.pool = (uint8_t *)c->pool;
    v.codes = v.pool + CSA2_PLANE_CODES(c->n_pages);
    v.scales = v.pool + CSA2_PLANE_SCALES(c->n_pages);
    v.keys = v.pool + CSA2_PLANE_KEYS(c->n_pages);
    v.summ = v.pool + CSA2_PLANE_SUMM(c->n_pages);
    v.n_pages = c->n_pages;
    v.page_table = c->page_table;
    v.max_pages = c->max_pages;
    v.n_tokens = c->n_tokens;
    v.m = c->m;
    v.swa = (uint8_t *)c->swa;
    v.pending = c->pending;
    v.error = c->error;
    v.batch = c->batch;
    return v;
}

// Page id of entry e (or of block e/8) of request b; -1 (and the error word
// set) when the page slot or the page id is out of range.
__device__ __forceinline__ int entry_pid(const CacheView &c, int b, int e)
{
    int pi = e >> 6;
    if (e < 0 || pi >= c.max_pages) {
        set_error(c.error, CSA2_DEV_CAPACITY);
        return -1;
    }
    int pid = __ldg(c.page_table + (size_t)b * c.max_pages + pi);
    if (pid < 0 || pid >= c.n_pages) {
        set_error(c.error, CSA2_DEV_BAD_PAGE);
        return -1;
    }
    return pid;
}

// Field rows of entry slot `slot` (0..63) / summary slot (0..7) of page pid.
__device__ __forceinline__ uint8_t *codes_row(const CacheView &c, int pid, int slot)
{
    return c.codes + (size_t)pid * CSA2_PAGE_CODES_BYTES + slot * CSA2_CODE_BYTES;
}
__device__ __forceinline__ uint8_t *scales_row(const CacheView &c, int pid, int slot)
{
    return c.scales + (size_t)pid * CSA2_PAGE_SCALES_BYTES + slot * CSA2_SCALE_BYTES;
}
__device__ __forceinline__ uint8_t *keys_row(const CacheView &c, int pid, int slot)
{
    return c.keys + (size_t)pid * CSA2_PAGE_KEYS_BYTES + slot * CSA2_KEY_DIM;
}
__device__ __forceinline__ uint8_t *summ_row(const CacheView &c, int pid, int sslot)
{
    return c.summ + (size_t)pid * CSA2_PAGE_SUMM_BYTES + sslot * CSA2_KEY_DIM;
}

__device__ __forceinline__ uint8_t *swa_base(const CacheView &c, int b)
{
    return c.swa + (size_t)b * CSA2_SWA_BYTES;
}

// Entries of request b, clamped to the pages it owns (a corrupt n_tokens
// can never push an index past the request's capacity).
__device__ __forceinline__ int n_entries_of(const CacheView &c, int b)
{
    int m = c.m[b];
    int n = c.n_tokens[b] / (m == 2 ? 2 : 1);
    return max(0, min(n, c.max_pages * CSA2_PAGE_ENTRIES));
}

}  // namespace csa2

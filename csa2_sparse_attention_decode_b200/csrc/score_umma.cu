// Indexer scoring on the 5th-generation tensor cores:
//   score(row) = sum_h w_h * ReLU(q_h . row)
// for rows = FP8 block summaries (FULL), every FP8 key (FLAT) or the pool's
// FP8 keys (FULL / REINDEX rescoring).  Source: 0539edu.com/news/5732216 §3
// (indexer: 32 query heads x 128 dims; hierarchical blocks of 8 positions).
//
// Design (one persistent CTA per SM, 6 warps):
//   warp 4      TMA producer: 128-row tiles (16 KB of FP8) into a 6-stage
//               shared-memory ring, 128-byte swizzled, one box per page run.
//   warps 0-3   thread = row: FP8 -> f16 (exact) straight into tensor memory
//               as the MMA's A operand; then the epilogue reads the 32 head
//               dot products of its row back from tensor memory and applies
//               ReLU and the head weights.
//   warp 5      allocates tensor memory and issues the MMAs:
//               D[128 x 32] (fp32) = A[128 x 128] (f16, TMEM) . Q^T (f16, smem).
// The query is converted once per request to f16 with an exact per-head
// power-of-two scale (so every bf16 query value stays exact), undone on the
// head weight: w_h * ReLU(dot) = (w_h * 2^-s) * ReLU(2^s dot).
// Tiles of all requests form one list split evenly over the CTAs.
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "index.cuh"
#include "umma.cuh"

namespace csa2 {
using namespace umma;

namespace {

constexpr int TILE = 128;
constexpr int STAGES = 6;
constexpr int STAGE_BYTES = TILE * CSA2_KEY_DIM;            // 16 KB
constexpr int QBYTES = CSA2_IDX_HEADS * CSA2_KEY_DIM * 2;   // 8 KB of f16
constexpr int THREADS = 192;
constexpr uint32_t TMEM_COLS = 256;
constexpr uint32_t A_COL0 = 0, D_COL0 = 128;                // A: 2 x 64 cols, D: 2 x 32 cols
constexpr size_t SMEM_BYTES = 1024 + (size_t)STAGES * STAGE_BYTES + 2 * QBYTES;
constexpr uint32_t IDESC = idesc_f16(128, 32, false, false, false);

struct Params {
    CacheView c;
    int src;
    const uint16_t *q_idx;
    const float *w;
    const int32_t *pool;
    const int32_t *pool_len;
    float *scores;
    int64_t stride;
};

__device__ __forceinline__ int rows_of_req(const Params &p, int b)
{
    int n = n_entries_of(p.c, b);
    if (p.src == ROWS_KEYS) return n;
    if (p.src == ROWS_SUMMARIES) return (n + CSA2_BLOCK - 1) / CSA2_BLOCK;
    return max(0, min(p.pool_len[b], CSA2_POOL));
}

// Walks this CTA's contiguous slice [i0, i1) of the global tile list.
struct TileIter {
    int b, t, rows, tiles, left;
    __device__ void init(const Params &p, long long i0, long long i1)
    {
        left = (int)(i1 - i0);
        b = 0;
        long long acc = 0;
        for (; b < p.c.batch; ++b) {
            rows = rows_of_req(p, b);
            tiles = (rows + TILE - 1) / TILE;
            if (i0 < acc + tiles) break;
            acc += tiles;
        }
        t = (int)(i0 - acc);
    }
    __device__ void next(const Params &p)
    {
        --left;
        if (left <= 0) return;
        ++t;
        while (t >= tiles) {
            ++b;
            t = 0;
            rows = rows_of_req(p, b);
            tiles = (rows + TILE - 1) / TILE;
        }
    }
};

__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, volatile int *abort, int32_t *err)
{
    for (uint32_t i = 0; i < (1u << 22); ++i) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((i & 1023) == 1023 && *abort) return false;
    }
    *abort = 1;
    set_error(err, CSA2_DEV_TIMEOUT);
    return false;
}

__device__ __forceinline__ void bar_workers() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__global__ void __launch_bounds__(THREADS, 1)
score_umma_kernel(const __grid_constant__ CUtensorMap map_summ, const __grid_constant__ CUtensorMap map_keys64,
                  const __grid_constant__ CUtensorMap map_keys8, Params p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t *qbuf = sm + STAGES * STAGE_BYTES;
    __shared__ __align__(8) uint64_t full[STAGES], empty[STAGES], a_full[2], d_full[2], d_empty[2];
    __shared__ float wq[2][CSA2_IDX_HEADS];
    __shared__ uint32_t tmem_base;
    __shared__ long long s_total;
    __shared__ volatile int s_abort;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (warp == 5) tmem_alloc(&tmem_base, TMEM_COLS);
    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 4);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&a_full[i], 4);
            mbar_init(&d_full[i], 1);
            mbar_init(&d_empty[i], 4);
        }
        s_abort = 0;
        mbar_fence_init();
    }
    if (warp == 0) {
        long long tot = 0;
        for (int b = lane; b < p.c.batch; b += 32) tot += (rows_of_req(p, b) + TILE - 1) / TILE;
#pragma unroll
        for (int o = 16; o; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
        if (lane == 0) s_total = tot;
    }
    __syncthreads();
    fence_after_sync();
    const uint32_t tb = tmem_base;
    const long long total = s_total;
    const long long i0 = total * blockIdx.x / gridDim.x, i1 = total * (blockIdx.x + 1) / gridDim.x;
    const int n_items = (int)(i1 - i0);
    volatile int *abort = &s_abort;

    if (warp == 4 && n_items > 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            tma_prefetch_map(&map_summ);
            tma_prefetch_map(&map_keys64);
            tma_prefetch_map(&map_keys8);
        }
        TileIter it;
        it.init(p, i0, i1);
        int issued = 0;
        for (int j = 0; j < n_items; ++j, it.next(p)) {
            const int s = j % STAGES;
            if (j >= STAGES && !wait_or_abort(&empty[s], ((j / STAGES) - 1) & 1, abort, p.c.error)) break;
            const int b = it.b, r0 = it.t * TILE;
            const int valid = min(TILE, it.rows - r0);
            // Lane l prepares chunk l of this tile (a page or an 8-row run).
            int chunk_rows = (p.src == ROWS_KEYS) ? 64 : 8;
            int n_chunks = (valid + chunk_rows - 1) / chunk_rows;
            int pid = -1, y = 0;
            if (lane < n_chunks) {
                int e;                                   // first entry of the chunk
                if (p.src == ROWS_SUMMARIES) e = (r0 + 8 * lane) * CSA2_BLOCK;
                else if (p.src == ROWS_KEYS) e = r0 + 64 * lane;
                else {
                    e = p.pool[(size_t)b * CSA2_POOL + r0 + 8 * lane];
                    if (e < 0 || e >= n_entries_of(p.c, b) || (e & 7)) {
                        set_error(p.c.error, CSA2_DEV_BAD_INDEX);
                        e = -1;
                    }
                }
                if (e >= 0) {
                    int pi = e >> 6;
                    if (pi < p.c.max_pages) {
                        int id = p.c.page_table[(size_t)b * p.c.max_pages + pi];
                        if (id >= 0 && id < p.c.n_pages) {
                            pid = id;
                            y = (p.src == ROWS_SUMMARIES) ? 0 : (e & 63);
                        } else {
                            set_error(p.c.error, CSA2_DEV_BAD_PAGE);
                        }
                    } else {
                        set_error(p.c.error, CSA2_DEV_CAPACITY);
                    }
                }
            }
            const uint32_t ok = __ballot_sync(0xffffffffu, pid >= 0);
            const uint32_t chunk_bytes = (p.src == ROWS_KEYS) ? 8192u : 1024u;
            if (lane == 0) mbar_arrive_expect_tx(&full[s], __popc(ok) * chunk_bytes);
            __syncwarp();
            if (pid >= 0) {
                uint8_t *dst = sm + s * STAGE_BYTES + lane * chunk_bytes;
                const CUtensorMap *m = (p.src == ROWS_SUMMARIES) ? &map_summ
                                     : (p.src == ROWS_KEYS)      ? &map_keys64
                                                                 : &map_keys8;
                tma_load_3d(dst, m, 0, y, pid, &full[s]);
            }
            issued = j + 1;
        }
        // Never leave with copies in flight: wait for the last stages to land.
        if (lane == 0)
            for (int j = max(0, issued - STAGES); j < issued; ++j) mbar_wait(&full[j % STAGES], (j / STAGES) & 1);
        __syncwarp();
    } else if (warp == 5 && n_items > 0) {
        // ------------------------------------------------------------ MMA issuer
        TileIter it;
        it.init(p, i0, i1);
        int cur_b = -1, sw = -1, issued = 0;
        for (int j = 0; j < n_items; ++j, it.next(p)) {
            if (it.b != cur_b) {
                cur_b = it.b;
                ++sw;
            }
            const int ab = j & 1, qb = sw & 1;
            if (!wait_or_abort(&a_full[ab], (j >> 1) & 1, abort, p.c.error)) break;
            if (j >= 2 && !wait_or_abort(&d_empty[ab], ((j >> 1) - 1) & 1, abort, p.c.error)) break;
            fence_after_sync();
            if (lane == 0) {
                const uint32_t qaddr = smem_addr(qbuf + qb * QBYTES);
#pragma unroll
                for (int kk = 0; kk < CSA2_KEY_DIM / 16; ++kk) {
                    uint64_t bd = smem_desc(qaddr + (kk >> 2) * 4096 + (kk & 3) * 32, 16, 1024);
                    mma_ts(tb + D_COL0 + 32 * ab, tb + A_COL0 + 64 * ab + 8 * kk, bd, IDESC, kk > 0 ? 1u : 0u);
                }
                mma_commit(&d_full[ab]);
            }
            __syncwarp();
            issued = j + 1;
        }
        if (lane == 0)
            for (int j = max(0, issued - 2); j < issued; ++j) mbar_wait(&d_full[j & 1], (j >> 1) & 1);
        __syncwarp();
    } else if (warp < 4 && n_items > 0) {
        // ------------------------------------------------------------ workers
        TileIter it;
        it.init(p, i0, i1);
        const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
        int cur_b = -1, sw = -1;
        int pb = 0, pt = 0, prow = 0, pqb = 0;       // previous item (for its epilogue)
        auto epilogue = [&](int i, int b, int t, int rows, int qb) {
            const int db = i & 1;
            bool ok = wait_or_abort(&d_full[db], (i >> 1) & 1, abort, p.c.error);
            fence_after_sync();
            uint32_t r[32];
            tmem_ld32(tb + lane_base + D_COL0 + 32 * db, r);
            tmem_ld_wait();
            fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&d_empty[db]);
            float sc = 0.0f;
#pragma unroll
            for (int h = 0; h < CSA2_IDX_HEADS; ++h) sc = fmaf(wq[qb][h], fmaxf(__uint_as_float(r[h]), 0.0f), sc);
            const int row = t * TILE + tid;
            if (ok && row < rows) p.scores[(size_t)b * p.stride + row] = sc;
        };
        for (int j = 0; j < n_items; ++j, it.next(p)) {
            if (it.b != cur_b) {
                // New request: convert its query into the free q buffer.
                cur_b = it.b;
                ++sw;
                const int qb = sw & 1;
                const int h = tid >> 2, qd = tid & 3;
                const uint4 *src = reinterpret_cast<const uint4 *>(p.q_idx + ((size_t)cur_b * CSA2_IDX_HEADS + h) *
                                                                                 CSA2_KEY_DIM + 32 * qd);
                uint4 raw[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) raw[i] = src[i];
                const uint32_t *rw = reinterpret_cast<const uint32_t *>(raw);
                float amax = 0.0f;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    amax = fmaxf(amax, fabsf(__uint_as_float(rw[i] << 16)));
                    amax = fmaxf(amax, fabsf(__uint_as_float(rw[i] & 0xffff0000u)));
                }
                amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
                amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
                int ex = 0;
                if (amax > 0.0f) frexpf(amax, &ex);
                const int sh = (amax > 0.0f) ? 15 - ex : 0;          // amax * 2^sh in [2^14, 2^15)
                uint8_t *qdst = qbuf + qb * QBYTES + (qd >> 1) * 4096 + h * 128;
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    uint32_t o[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        uint32_t v = rw[4 * cc + i];
                        __half lo = __float2half_rn(ldexpf(__uint_as_float(v << 16), sh));
                        __half hi = __float2half_rn(ldexpf(__uint_as_float(v & 0xffff0000u), sh));
                        o[i] = (uint32_t)__half_as_ushort(lo) | ((uint32_t)__half_as_ushort(hi) << 16);
                    }
                    const int chunk = 4 * (qd & 1) + cc;
                    *reinterpret_cast<uint4 *>(qdst + ((chunk ^ (h & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
                }
                if (qd == 0) wq[qb][h] = ldexpf(p.w[(size_t)cur_b * CSA2_IDX_HEADS + h], -sh);
                fence_proxy_async_smem();
                bar_workers();
            }
            const int s = j % STAGES, ab = j & 1;
            wait_or_abort(&full[s], (j / STAGES) & 1, abort, p.c.error);
            // Row tid of the tile: 8 swizzled 16-byte chunks -> 64 f16x2 columns.
            const uint8_t *row = sm + s * STAGE_BYTES + tid * 128;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t cols[32];
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    const int c = 4 * half + c4;
                    uint4 v = *reinterpret_cast<const uint4 *>(row + ((c ^ (tid & 7)) << 4));
                    uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(wv[i] & 0xffff), __NV_E4M3);
                        __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(wv[i] >> 16), __NV_E4M3);
                        cols[8 * c4 + 2 * i] = (uint32_t)lo.x | ((uint32_t)lo.y << 16);
                        cols[8 * c4 + 2 * i + 1] = (uint32_t)hi.x | ((uint32_t)hi.y << 16);
                    }
                }
                tmem_st32(tb + lane_base + A_COL0 + 64 * ab + 32 * half, cols);
            }
            tmem_st_wait();
            fence_before_sync();
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&a_full[ab]);
                mbar_arrive(&empty[s]);
            }
            if (j > 0) epilogue(j - 1, pb, pt, prow, pqb);
            pb = it.b;
            pt = it.t;
            prow = it.rows;
            pqb = sw & 1;
        }
        epilogue(n_items - 1, pb, pt, prow, pqb);
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 5) {
        fence_after_sync();
        tmem_dealloc(tb, TMEM_COLS);
    }
}

// ---------------------------------------------------------------- host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (PFN_cuTensorMapEncodeTiled_v12000)ptr;
    }
    return fn;
}

// 3-D byte tensor over one page field: (128 bytes, slots, pages).
bool make_page_map(CUtensorMap *m, void *base, int slots, int box_slots, int n_pages)
{
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {128, (cuuint64_t)slots, (cuuint64_t)n_pages};
    cuuint64_t strides[2] = {128, CSA2_PAGE_BYTES};
    cuuint32_t box[3] = {128, (cuuint32_t)box_slots, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int sm_count()
{
    static int n[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) dev = 0;
    if (!n[dev]) {
        int v = 0;
        cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
        n[dev] = v > 0 ? v : 148;
    }
    return n[dev];
}

}  // namespace

cudaError_t launch_score(const CacheView &c, int src, const uint16_t *q_idx, const float *w, const int32_t *pool,
                         const int32_t *pool_len, float *scores, int64_t stride, int max_rows, cudaStream_t st)
{
    (void)max_rows;
    static bool attr_done[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 64 || !attr_done[dev]) {
        e = cudaFuncSetAttribute(score_umma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
        if (e != cudaSuccess) return e;
        if (dev < 64) attr_done[dev] = true;
    }
    CUtensorMap m_summ, m_keys64, m_keys8;
    if (!make_page_map(&m_summ, c.pool + CSA2_PAGE_SUMM_OFF, 8, 8, c.n_pages) ||
        !make_page_map(&m_keys64, c.pool + CSA2_PAGE_KEYS_OFF, 64, 64, c.n_pages) ||
        !make_page_map(&m_keys8, c.pool + CSA2_PAGE_KEYS_OFF, 64, 8, c.n_pages))
        return cudaErrorInvalidValue;
    Params p{c, src, q_idx, w, pool, pool_len, scores, stride};
    int kid = src == ROWS_KEYS ? CSA2_KERNEL_FLAT_SCORE : src == ROWS_SUMMARIES ? CSA2_KERNEL_BLOCK_SCORE
                                                                                : CSA2_KERNEL_POOL_SCORE;
    LaunchScope scope(kid, st);
    score_umma_kernel<<<sm_count(), THREADS, SMEM_BYTES, st>>>(m_summ, m_keys64, m_keys8, p);
    return cudaGetLastError();
}

}  // namespace csa2

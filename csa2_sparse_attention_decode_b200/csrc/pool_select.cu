// Exact rescoring of the hierarchical candidate pool fused with its top-512
// selection:
//   score(e) = sum_h w_h * ReLU(q_h . k_e)   for every entry e of the pool,
//   topk     = the 512 best pool entries (score desc, ties to the lower pool
//              position), ascending, -1 padded.
// Source: 0539edu.com/news/5732216 §3 (indexer 32 heads x 128; hierarchical
// 2048 blocks x 8 positions = 16384 candidates; top_k 512; Full builds the
// pool, Reindex searches inside it with its own query).
//
// One 8-CTA cluster per request.  CTA r scores pool rows [r*chunk,
// r*chunk + chunk) (chunk a multiple of 128, at most 2048) and keeps the
// order-preserving keys of its scores in shared memory; the cluster then runs
// the selection of select.cuh over them and writes the selected pool ids.
// Scoring roles (256 threads):
//   warp 4      looks up the page of every 8-row run of the CTA's rows, then
//               copies the runs (8 rows x 128 B of FP8 keys) by TMA into an
//               8-stage ring of 128-row tiles, 128-byte swizzled;
//   warp 5      issues the MMAs: D[128 x 32] (fp32, tensor memory) =
//               sum_p K[128 x 128] (e4m3) . Qp^T (kind::f8f6f4), Q1 + Q2 + Q3
//               the query split exactly into e5m2 parts (idx_query.cuh), into
//               four rotating accumulators;
//   warps 0-3   split the query, then one thread per row: score =
//               sum_h w'_h ReLU(D[h]);
//   warps 6-7   join for the selection.
#include <cudaTypedefs.h>

#include <cooperative_groups.h>

#include "common.cuh"
#include "idx_query.cuh"
#include "index.cuh"
#include "select.cuh"
#include "umma.cuh"

namespace cg = cooperative_groups;

namespace csa2 {
using namespace umma;

namespace {

constexpr int NC = 8;                                    // CTAs per request
constexpr int NT = 256;
constexpr int TILE = 128;
constexpr int STAGES = 8;
constexpr int CHUNK_MAX = CSA2_POOL / NC;                // 2048 rows per CTA
constexpr int RUNS = CHUNK_MAX / CSA2_BLOCK;             // 256 runs of 8 rows
constexpr int STAGE_BYTES = TILE * CSA2_KEY_DIM;         // 16 KB
constexpr int RUN_BYTES = CSA2_BLOCK * CSA2_KEY_DIM;     // 1 KB
constexpr int BITS_WORDS = CHUNK_MAX / 32;
constexpr size_t OFF_Q = (size_t)STAGES * STAGE_BYTES;
constexpr size_t OFF_KEYS = OFF_Q + IQ_BYTES;
constexpr size_t OFF_CAND = OFF_KEYS + CHUNK_MAX * 4;
constexpr size_t OFF_ALL = OFF_CAND + 2 * sel::CAND * 4;
constexpr size_t OFF_BITS = OFF_ALL + 2 * sel::RANK_MAX * 4;
constexpr size_t OFF_RUNS = OFF_BITS + BITS_WORDS * 4;
constexpr size_t SMEM_BYTES = 1024 + OFF_RUNS + RUNS * 4;
constexpr int ACC = 4;                                   // accumulators in tensor memory
constexpr int ACC_COLS = CSA2_IDX_HEADS;                 // 32 columns each
constexpr int QPART_BYTES = CSA2_IDX_HEADS * CSA2_KEY_DIM;
constexpr uint32_t TMEM_COLS = ACC * ACC_COLS;           // 128
// kind::f8f6f4: D f32, A e4m3 (0), B e5m2 (1), both K-major, N = 32, M = 128.
constexpr uint32_t IDESC = (1u << 4) | (0u << 7) | (1u << 10) | ((uint32_t)(ACC_COLS >> 3) << 17) | (8u << 24);

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

__device__ __forceinline__ void mma_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc, uint32_t acc)
{
    asm volatile("{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
                 "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
                 "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(acc)
                 : "memory");
}

__device__ __forceinline__ void bar_workers() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__global__ void __cluster_dims__(NC, 1, 1) __launch_bounds__(NT, 1)
pool_select_kernel(const __grid_constant__ CUtensorMap keys8, CacheView c, const uint16_t *q_idx, const float *w,
                   const int32_t *pool, const int32_t *pool_len, int32_t *topk)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t *ring = sm, *qbuf = sm + OFF_Q;
    uint32_t *keys = reinterpret_cast<uint32_t *>(sm + OFF_KEYS);
    int32_t *runs = reinterpret_cast<int32_t *>(sm + OFF_RUNS);
    __shared__ __align__(8) uint64_t full[STAGES], empty[STAGES], d_full[ACC], d_empty[ACC], q_full;
    __shared__ float wq[CSA2_IDX_HEADS];
    __shared__ uint32_t tmem_base;
    __shared__ volatile int s_abort;
    cg::cluster_group cluster = cg::this_cluster();

    const int rank = (int)cluster.block_rank(), b = blockIdx.y;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (warp == 5) {
        tmem_alloc(&tmem_base, TMEM_COLS);
        fence_before_sync();
    }
    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < ACC; ++i) {
            mbar_init(&d_full[i], 1);
            mbar_init(&d_empty[i], 4);
        }
        mbar_init(&q_full, 1);
        s_abort = 0;
        mbar_fence_init();
    }
    if (tid == 32 * 4) tma_prefetch_map(&keys8);
    grid_dependency_wait();                      // the pool may come from the previous kernel
    allow_dependents();
    const int n_entries = n_entries_of(c, b);
    const int n = max(0, min(pool_len[b], CSA2_POOL));
    const int chunk = ((n + NC * TILE - 1) / (NC * TILE)) * TILE;
    const int lo = rank * chunk;
    const int cnt = max(0, min(n, lo + chunk) - lo);
    const int n_tiles = (cnt + TILE - 1) / TILE;
    __syncthreads();
    fence_after_sync();
    const uint32_t tb = tmem_base;
    volatile int *abort = &s_abort;
    uint32_t kmin = 0xffffffffu, kmax = 0u;

    if (warp == 4 && n_tiles > 0) {
        // ------------------------------------------------------------ producer
        // Plane row of every run: pool id, then page table, 8 runs per lane
        // with all loads of a round in flight together.
        const int n_runs = (cnt + CSA2_BLOCK - 1) / CSA2_BLOCK;
        int e_[8], pg_[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int j = lane + 32 * u;
            e_[u] = j < n_runs ? pool[(size_t)b * CSA2_POOL + lo + CSA2_BLOCK * j] : -1;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int e = e_[u];
            pg_[u] = (e >= 0 && e < n_entries && (e >> 6) < c.max_pages)
                         ? c.page_table[(size_t)b * c.max_pages + (e >> 6)] : -1;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            const int j = lane + 32 * u;
            if (j >= n_runs) continue;
            const int e = e_[u], pg = pg_[u];
            int pid = -1;
            if (e < 0 || e >= n_entries || (e & (CSA2_BLOCK - 1))) set_error(c.error, CSA2_DEV_BAD_INDEX);
            else if ((e >> 6) >= c.max_pages) set_error(c.error, CSA2_DEV_CAPACITY);
            else if (pg < 0 || pg >= c.n_pages) set_error(c.error, CSA2_DEV_BAD_PAGE);
            else pid = pg * CSA2_PAGE_ENTRIES + (e & (CSA2_PAGE_ENTRIES - 1));
            runs[j] = pid;
        }
        __syncwarp();
        int issued = 0;
        for (int t = 0; t < n_tiles; ++t) {
            const int s = t % STAGES;
            bool okw = true;
            if (lane == 0 && t >= STAGES) okw = wait_or_abort(&empty[s], ((t / STAGES) - 1) & 1, abort, c.error);
            if (!__shfl_sync(0xffffffffu, okw, 0)) break;          // warp-uniform decision
            const int j = 16 * t + lane;
            const int row = (lane < 16 && j < n_runs) ? runs[j] : -1;
            const uint32_t ok = __ballot_sync(0xffffffffu, row >= 0);
            if (lane == 0) mbar_arrive_expect_tx(&full[s], (uint32_t)__popc(ok) * RUN_BYTES);
            __syncwarp();
            if (row >= 0) tma_load_2d(ring + s * STAGE_BYTES + lane * RUN_BYTES, &keys8, 0, row, &full[s]);
            __syncwarp();
            issued = t + 1;
        }
        // Never leave with copies in flight: wait for the last stages to land.
        if (lane == 0)
            for (int j = max(0, issued - STAGES); j < issued; ++j) mbar_wait(&full[j % STAGES], (j / STAGES) & 1);
        __syncwarp();
    } else if (warp == 5 && n_tiles > 0) {
        // ------------------------------------------------------------ MMA issuer
        const uint32_t qaddr = smem_addr(qbuf);
        int issued = 0;
        for (int t = 0; t < n_tiles; ++t) {
            const int ab = t % ACC, s = t % STAGES;
            bool okw = true;
            if (lane == 0) {
                if (t == 0) okw = wait_or_abort(&q_full, 0, abort, c.error);
                if (okw) okw = wait_or_abort(&full[s], (t / STAGES) & 1, abort, c.error);
                if (okw && t >= ACC) okw = wait_or_abort(&d_empty[ab], ((t / ACC) - 1) & 1, abort, c.error);
            }
            if (!__shfl_sync(0xffffffffu, okw, 0)) break;          // warp-uniform decision
            fence_after_sync();
            if (lane == 0) {
                const uint32_t aaddr = smem_addr(ring + s * STAGE_BYTES);
#pragma unroll
                for (int kk = 0; kk < CSA2_KEY_DIM / 32; ++kk)
#pragma unroll
                    for (int pp = 0; pp < IQ_PARTS; ++pp)
                        mma_f8(tb + ACC_COLS * ab, smem_desc(aaddr + kk * 32, 16, 1024),
                               smem_desc(qaddr + pp * QPART_BYTES + kk * 32, 16, 1024), IDESC, (kk | pp) ? 1u : 0u);
                mma_commit(&d_full[ab]);
                mma_commit(&empty[s]);                              // stage free once the MMAs have read it
            }
            __syncwarp();
            issued = t + 1;
        }
        if (lane == 0)
            for (int j = max(0, issued - ACC); j < issued; ++j) mbar_wait(&d_full[j % ACC], (j / ACC) & 1);
        __syncwarp();
    } else if (warp < 4 && n_tiles > 0) {
        // ------------------------------------------------------------ workers
        iq_split(tid, q_idx, w, b, qbuf, wq);
        fence_proxy_async_smem();
        bar_workers();
        if (tid == 0) mbar_arrive(&q_full);
        float wr[CSA2_IDX_HEADS];
#pragma unroll
        for (int hh = 0; hh < CSA2_IDX_HEADS; ++hh) wr[hh] = wq[hh];
        const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
        for (int t = 0; t < n_tiles; ++t) {
            const int db = t % ACC;
            const bool ok = wait_or_abort(&d_full[db], (t / ACC) & 1, abort, c.error);
            fence_after_sync();
            uint32_t r0[32];
            tmem_ld32(tb + lane_base + ACC_COLS * db, r0);
            tmem_ld_wait();
            fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&d_empty[db]);
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int hh = 0; hh < CSA2_IDX_HEADS; ++hh)
                acc[hh & 3] = fmaf(wr[hh], fmaxf(__uint_as_float(r0[hh]), 0.0f), acc[hh & 3]);
            const float sc = (acc[0] + acc[1]) + (acc[2] + acc[3]);
            const int e = t * TILE + tid;
            if (e < cnt) {
                const uint32_t key = sel::ord_key(ok ? sc : 0.0f);
                keys[e] = key;
                kmin = min(kmin, key);
                kmax = max(kmax, key);
            }
        }
    }
    fence_before_sync();
    __syncthreads();

    // ---------------------------------------------------------------- selection
    sel::Bufs bf;
    bf.keys = keys;
    bf.scores = nullptr;
    bf.cand_key = reinterpret_cast<uint32_t *>(sm + OFF_CAND);
    bf.cand_idx = bf.cand_key + sel::CAND;
    bf.all_key = reinterpret_cast<uint32_t *>(sm + OFF_ALL);
    bf.all_idx = bf.all_key + sel::RANK_MAX;
    bf.bits = reinterpret_cast<uint32_t *>(sm + OFF_BITS);
    bf.bits_words = BITS_WORDS;
    sel::Out o;
    o.out = topk;
    o.out_stride = CSA2_TOPK;
    o.ids = pool;
    o.expand = 0;
    o.pool = nullptr;
    o.pool_len = nullptr;
    o.n_entries = n_entries;
    sel::select_core<NC, NT>(bf, b, n, chunk, lo, cnt, CSA2_TOPK, kmin, kmax, o);

    fence_before_sync();
    __syncthreads();
    if (warp == 5) {
        fence_after_sync();
        tmem_dealloc(tb, TMEM_COLS);
    }
}

// 2-D byte tensor over the key plane: rows of 128 bytes, boxes of 8 rows,
// 128-byte swizzled.
bool make_keys8_map(CUtensorMap *m, void *base, long long rows)
{
    auto fn = tensor_map_encoder();
    if (!fn) return false;
    cuuint64_t dims[2] = {128, (cuuint64_t)rows};
    cuuint64_t strides[1] = {128};
    cuuint32_t box[2] = {128, (cuuint32_t)CSA2_BLOCK};
    cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_pool_select(const CacheView &c, const uint16_t *q_idx, const float *w, const int32_t *pool,
                               const int32_t *pool_len, int32_t *topk, cudaStream_t st)
{
    static bool attr_done[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 64 || !attr_done[dev]) {
        e = cudaFuncSetAttribute(pool_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
        if (e != cudaSuccess) return e;
        if (dev < 64) attr_done[dev] = true;
    }
    CUtensorMap keys8;
    if (!make_keys8_map(&keys8, c.keys, (long long)c.n_pages * CSA2_PAGE_ENTRIES)) return cudaErrorInvalidValue;
    LaunchScope scope(CSA2_KERNEL_POOL_SCORE, st);
    return launch_pdl(pool_select_kernel, dim3(NC, c.batch), dim3(NT), SMEM_BYTES, st, keys8, c, q_idx, w, pool,
                      pool_len, topk);
}

}  // namespace csa2

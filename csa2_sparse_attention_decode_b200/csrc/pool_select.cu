// Exact rescoring of the hierarchical candidate pool fused with its top-512
// selection:
//   score(e) = sum_h w_h * ReLU(q_h . k_e)   for every entry e of the pool,
//   topk     = the 512 best pool entries (score desc, ties to the lower pool
//              position), ascending, -1 padded.
// Source: 0539edu.com/news/5732216 §3 (indexer 32 heads x 128; hierarchical
// 2048 blocks x 8 positions = 16384 candidates; top_k 512; Full builds the
// pool, Reindex searches inside it with its own query).
//
// One cluster of NC = 16, 8, 4 or 2 CTAs per request, chosen per launch
// from the batch and how many clusters of each size can be resident at once.
// CTA r scores pool rows [r*chunk, r*chunk + chunk) (chunk a multiple of
// 128, at most 16384 / NC) and keeps the
// order-preserving keys of its scores in shared memory; the cluster then runs
// the selection of select.cuh over them and writes the selected pool ids.
// Scoring roles (384 threads):
//   warps 5-11  look up the page of every 8-row run of the CTA's rows; warp
//               5 then copies the runs (8 rows x 128 B of FP8 keys, 1 KB)
//               with one TMA box each into an 8-stage ring of 128-row tiles,
//               128-byte swizzled;
//   warp 4      issues the MMAs: D[128 x 32] (fp32, tensor memory) =
//               sum_p K[128 x 128] (e4m3) . Qp^T (kind::f8f6f4), Q1 + Q2 + Q3
//               the query split exactly into e5m2 parts (idx_query.cuh), into
//               four rotating accumulators;
//   warps 0-3   split the query, then one thread per row: score =
//               sum_h w'_h ReLU(D[h]);
//   all warps then run the selection.
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

constexpr int NT = 384;
constexpr int TILE = 128;
constexpr int STAGES = 8;
constexpr int NPROD = NT - 5 * 32;                       // producer threads (warps 5-11): more copies in flight
constexpr int STAGE_BYTES = TILE * CSA2_KEY_DIM;         // 16 KB
// Shared-memory layout for NC CTAs per request (rows per CTA at most POOL/NC).
template <int NC>
struct Layout {
    static constexpr int CHUNK_MAX = CSA2_POOL / NC;     // 8192 ... 1024 rows (NC = 2 ... 16)
    static constexpr int RUNS = CHUNK_MAX / CSA2_BLOCK;  // runs of 8 rows
    static constexpr int BITS_WORDS = CHUNK_MAX / 32;
    static constexpr size_t OFF_Q = (size_t)STAGES * STAGE_BYTES;
    static constexpr size_t OFF_KEYS = OFF_Q + IQ_BYTES;
    static constexpr size_t OFF_CAND = OFF_KEYS + CHUNK_MAX * 4;
    static constexpr size_t OFF_ALL = OFF_CAND + 2 * sel::CAND * 4;
    static constexpr size_t OFF_BITS = OFF_ALL + 2 * sel::RANK_MAX * 4;
    static constexpr size_t OFF_RUNS = OFF_BITS + BITS_WORDS * 4;
    static constexpr size_t SMEM_BYTES = 1024 + OFF_RUNS + RUNS * 4;
};
constexpr int ACC = 2;                                   // accumulators in tensor memory
constexpr int ACC_COLS = IQ_ROWS;                        // 96 columns each: 3 query parts x 32 heads
constexpr uint32_t TMEM_COLS = 256;                      // >= ACC * ACC_COLS, a power of two
static_assert(ACC * ACC_COLS <= (int)TMEM_COLS, "tensor memory budget");
// kind::f8f6f4: D f32, A e4m3 (0), B e5m2 (1), both K-major, M = 128, N = 96:
// the three query parts sit side by side as 96 B rows, so one MMA per
// 32-dim K step scores a tile against all of them.
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
__device__ __forceinline__ void bar_producers() { asm volatile("bar.sync 2, %0;" ::"n"(NPROD) : "memory"); }

template <int NC>
__global__ void __launch_bounds__(NT, 1)
pool_select_kernel(const __grid_constant__ CUtensorMap map_keys8, CacheView c, const uint16_t *q_idx, const float *w,
                   const int32_t *pool, const int32_t *pool_len, int32_t *topk, float *topk_scores,
                   const int32_t *id_off)
{
    using Lay = Layout<NC>;
    constexpr int RUNS = Lay::RUNS;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t *ring = sm, *qbuf = sm + Lay::OFF_Q;
    uint32_t *keys = reinterpret_cast<uint32_t *>(sm + Lay::OFF_KEYS);
    int32_t *runs = reinterpret_cast<int32_t *>(sm + Lay::OFF_RUNS);
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
    if (warp == 6) {
        // L2 hints while the previous kernel finishes (nothing is read before
        // the wait): this CTA's share of request b's page table and of its
        // indexer query, and the request's length.
        const size_t pt = (size_t)c.max_pages * 4, qb = (size_t)CSA2_IDX_HEADS * CSA2_KEY_DIM * 2;
        prefetch_l2_range(c.page_table + (size_t)b * c.max_pages, pt * rank / NC, pt * (rank + 1) / NC, lane, 16);
        prefetch_l2_range(q_idx + (size_t)b * CSA2_IDX_HEADS * CSA2_KEY_DIM, qb * rank / NC, qb * (rank + 1) / NC,
                          lane, 1);
        if (rank == 0 && lane == 0) {
            prefetch_l2(c.n_tokens + b);
            prefetch_l2(c.m + b);
            prefetch_l2(w + (size_t)b * CSA2_IDX_HEADS);
        }
    }
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

    if (warp >= 5 && n_tiles > 0) {
        // ------------------------------------------------------------ producers
        // Plane row of every run (pool id, then page table, each round's
        // loads in flight together); then warp 5 copies each tile's 16 runs
        // (8 rows x 128 B of one page, 1 KB) with one TMA box each, lanes
        // 0-15 issuing together, 128-byte swizzled as the MMA reads them.
        const int ptid = tid - 5 * 32;
        const int n_runs = (cnt + CSA2_BLOCK - 1) / CSA2_BLOCK;
        constexpr int RPT = (RUNS + NPROD - 1) / NPROD;          // runs per producer thread
        int e_[RPT], pg_[RPT];
#pragma unroll
        for (int u = 0; u < RPT; ++u) {
            const int j = ptid + NPROD * u;
            e_[u] = j < n_runs ? pool[(size_t)b * CSA2_POOL + lo + CSA2_BLOCK * j] : -1;
        }
#pragma unroll
        for (int u = 0; u < RPT; ++u) {
            const int e = e_[u];
            pg_[u] = (e >= 0 && e < n_entries && (e >> 6) < c.max_pages)
                         ? c.page_table[(size_t)b * c.max_pages + (e >> 6)] : -1;
        }
#pragma unroll
        for (int u = 0; u < RPT; ++u) {
            const int j = ptid + NPROD * u;
            if (j >= n_runs) continue;
            const int e = e_[u], pg = pg_[u];
            int pid = -1;
            if (e < 0 || e >= n_entries || (e & (CSA2_BLOCK - 1))) set_error(c.error, CSA2_DEV_BAD_INDEX);
            else if ((e >> 6) >= c.max_pages) set_error(c.error, CSA2_DEV_CAPACITY);
            else if (pg < 0 || pg >= c.n_pages) set_error(c.error, CSA2_DEV_BAD_PAGE);
            else pid = pg * CSA2_PAGE_ENTRIES + (e & (CSA2_PAGE_ENTRIES - 1));
            runs[j] = pid;
        }
        bar_producers();
        if (warp == 5) {
            if (lane == 0) tma_prefetch_map(&map_keys8);
            int issued = 0;
            for (int t = 0; t < n_tiles; ++t) {
                const int s = t % STAGES;
                bool okw = true;
                if (lane == 0 && t >= STAGES) okw = wait_or_abort(&empty[s], ((t / STAGES) - 1) & 1, abort, c.error);
                if (!__shfl_sync(0xffffffffu, okw, 0)) break;      // warp-uniform decision
                uint8_t *stage = ring + s * STAGE_BYTES;
                const int run = 16 * t + lane;
                const int pid = (lane < 16 && run < n_runs) ? runs[run] : -1;
                const uint32_t ok = __ballot_sync(0xffffffffu, pid >= 0);
                if (lane == 0) mbar_arrive_expect_tx(&full[s], (uint32_t)__popc(ok) * CSA2_BLOCK * CSA2_KEY_DIM);
                __syncwarp();
                if (pid >= 0) tma_load_2d(stage + lane * CSA2_BLOCK * CSA2_KEY_DIM, &map_keys8, 0, pid, &full[s]);
                issued = t + 1;
            }
            // Never leave with copies in flight: wait for the last stages to land.
            if (lane == 0)
                for (int j = max(0, issued - STAGES); j < issued; ++j) mbar_wait(&full[j % STAGES], (j / STAGES) & 1);
            __syncwarp();
        }
    } else if (warp == 4 && n_tiles > 0) {
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
                    mma_f8(tb + ACC_COLS * ab, smem_desc(aaddr + kk * 32, 16, 1024),
                           smem_desc(qaddr + kk * 32, 16, 1024), IDESC, kk > 0 ? 1u : 0u);
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
            uint32_t r0[32], r1[32], r2[32];                       // the three query parts' products
            tmem_ld32(tb + lane_base + ACC_COLS * db, r0);
            tmem_ld32(tb + lane_base + ACC_COLS * db + 32, r1);
            tmem_ld32(tb + lane_base + ACC_COLS * db + 64, r2);
            tmem_ld_wait();
            fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&d_empty[db]);
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int hh = 0; hh < CSA2_IDX_HEADS; ++hh)
                acc[hh & 3] = fmaf(wr[hh],
                                   fmaxf((__uint_as_float(r0[hh]) + __uint_as_float(r1[hh])) + __uint_as_float(r2[hh]),
                                         0.0f),
                                   acc[hh & 3]);
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
    bf.cand_key = reinterpret_cast<uint32_t *>(sm + Lay::OFF_CAND);
    bf.cand_idx = bf.cand_key + sel::CAND;
    bf.all_key = reinterpret_cast<uint32_t *>(sm + Lay::OFF_ALL);
    bf.all_idx = bf.all_key + sel::RANK_MAX;
    bf.bits = reinterpret_cast<uint32_t *>(sm + Lay::OFF_BITS);
    bf.bits_words = Lay::BITS_WORDS;
    sel::Out o;
    o.out = topk;
    o.out_stride = CSA2_TOPK;
    o.ids = pool;
    o.expand = 0;
    o.pool = nullptr;
    o.pool_len = nullptr;
    o.n_entries = n_entries;
    o.vals = topk_scores;
    o.id_off = id_off;
    o.id_shift = 0;
    o.run_rows = runs;                           // the attention gathers the winners' latents next
    o.codes = c.codes;
    o.scales = c.scales;
    sel::select_core<NC, NT>(bf, b, n, chunk, lo, cnt, CSA2_TOPK, kmin, kmax, o);

    fence_before_sync();
    __syncthreads();
    if (warp == 5) {
        fence_after_sync();
        tmem_dealloc(tb, TMEM_COLS);
    }
}

}  // namespace

cudaError_t launch_pool_select(const CacheView &c, const uint16_t *q_idx, const float *w, const int32_t *pool,
                               const int32_t *pool_len, int32_t *topk, cudaStream_t st, float *topk_scores,
                               const int32_t *id_off)
{
    // Clusters of 16, 8, 4 or 2 CTAs per request, whichever minimises
    // resident waves x a cluster's time (the selection's fixed ~12 us +
    // ~0.74 us per gathered 128-row tile of a CTA, up to 16384 / NC rows).
    static DeviceOnce once;
    static int active[DeviceOnce::N][4] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess)
        e = once.run(dev, [&] {
            // Clusters of 2 need nearly all of a CTA's shared memory: left out
            // where the device does not grant it.
            const bool two = cudaFuncSetAttribute(pool_select_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                  (int)Layout<2>::SMEM_BYTES) == cudaSuccess;
            if (!two) cudaGetLastError();
            cudaError_t r = cudaFuncSetAttribute(pool_select_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)Layout<4>::SMEM_BYTES);
            if (r == cudaSuccess)
                r = cudaFuncSetAttribute(pool_select_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Layout<8>::SMEM_BYTES);
            if (r == cudaSuccess)
                r = cudaFuncSetAttribute(pool_select_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Layout<16>::SMEM_BYTES);
            if (r == cudaSuccess)
                r = cudaFuncSetAttribute(pool_select_kernel<16>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
            if (r == cudaSuccess) {
                active[dev][0] = two ? max_active_clusters(pool_select_kernel<2>, dim3(NT), Layout<2>::SMEM_BYTES, 2) : 0;
                active[dev][1] = max_active_clusters(pool_select_kernel<4>, dim3(NT), Layout<4>::SMEM_BYTES, 4);
                active[dev][2] = max_active_clusters(pool_select_kernel<8>, dim3(NT), Layout<8>::SMEM_BYTES, 8);
                active[dev][3] = max_active_clusters(pool_select_kernel<16>, dim3(NT), Layout<16>::SMEM_BYTES, 16);
            }
            return r;
        });
    if (e != cudaSuccess) return e;
    int nc = 8;
    double best = 1e30;
    for (int i = 3; i >= 0; --i) {                  // 16 first: it wins ties
        const int size = 2 << i, act = active[dev][i];
        if (act < 1) continue;
        const double us = (double)((c.batch + act - 1) / act) * (12.0 + 0.74 * (CSA2_POOL / size / TILE));
        if (us < best) {
            best = us;
            nc = size;
        }
    }
    CUtensorMap map_keys8;
    if (!make_plane_map(&map_keys8, c.keys, (long long)c.n_pages * CSA2_PAGE_ENTRIES, CSA2_BLOCK))
        return cudaErrorInvalidValue;
    LaunchScope scope(CSA2_KERNEL_POOL_SCORE, st);
    if (nc == 16)
        return launch_pdl_cluster(pool_select_kernel<16>, dim3(16, c.batch), dim3(NT), Layout<16>::SMEM_BYTES, st, 16,
                                  map_keys8, c, q_idx, w, pool, pool_len, topk, topk_scores, id_off);
    if (nc == 2)
        return launch_pdl_cluster(pool_select_kernel<2>, dim3(2, c.batch), dim3(NT), Layout<2>::SMEM_BYTES, st, 2,
                                  map_keys8, c, q_idx, w, pool, pool_len, topk, topk_scores, id_off);
    if (nc == 4)
        return launch_pdl_cluster(pool_select_kernel<4>, dim3(4, c.batch), dim3(NT), Layout<4>::SMEM_BYTES, st, 4,
                                  map_keys8, c, q_idx, w, pool, pool_len, topk, topk_scores, id_off);
    return launch_pdl_cluster(pool_select_kernel<8>, dim3(8, c.batch), dim3(NT), Layout<8>::SMEM_BYTES, st, 8,
                              map_keys8, c, q_idx, w, pool, pool_len, topk, topk_scores, id_off);
}

}  // namespace csa2

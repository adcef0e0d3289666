// Indexer scoring on the 5th-generation tensor cores:
//   score(row) = sum_h w_h * ReLU(q_h . row)
// for rows = FP8 block summaries (FULL), every FP8 key (FLAT) or the pool's
// FP8 keys (FULL / REINDEX rescoring).  Source: 0539edu.com/news/5732216 §3
// (indexer: 32 query heads x 128 dims; hierarchical blocks of 8 positions).
//
// Design (two persistent CTAs per SM, 6 warps each):
//   warp 4      TMA producer: 128-row tiles (16 KB of FP8) into a 5-stage
//               shared-memory ring, 128-byte swizzled, one box per page run.
//   warp 5      allocates tensor memory and issues the MMAs straight on the
//               FP8 tile: D[128 x 32] (fp32) = sum_p K[128 x 128] (e4m3) .
//               Qp^T, kind::f8f6f4, where Q1 + Q2 + Q3 is the query split
//               exactly into three e5m2 parts (idx_query.cuh); the tensor
//               cores add the three products into one accumulator.  Four
//               accumulators of 32 columns let the MMAs run ahead of the
//               epilogue.
//   warps 0-3   convert the query once per request; thread = row epilogue:
//               score = sum_h w'_h ReLU(D[h]).
// The tensor cores accumulate these products at fp32 precision (checked on
// hardware against exact sums), so the scores are fp32-accumulated
// sum_h w_h ReLU(q_h . k) as the method defines them.
// Tiles of all requests form one list split evenly over the CTAs.
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "idx_query.cuh"
#include "index.cuh"
#include "select.cuh"
#include "umma.cuh"

namespace csa2 {
using namespace umma;

namespace {

constexpr int TILE = 128;
constexpr int STAGES = 4;
constexpr int CTAS_PER_SM = 2;                              // two independent pipelines per SM
constexpr int PW = 16;                                      // producer look-up window (tiles)
constexpr int STAGE_BYTES = TILE * CSA2_KEY_DIM;            // 16 KB
constexpr int QBYTES = IQ_BYTES;                            // 3 parts x 32 heads x 128 dims of e5m2
constexpr int ACC = 2;                                      // accumulators in tensor memory
constexpr int ACC_COLS = IQ_ROWS;                           // 96 columns each: 3 query parts x 32 heads
constexpr int THREADS = 192;
constexpr uint32_t TMEM_COLS = 256;                         // >= ACC * ACC_COLS, a power of two
static_assert(ACC * ACC_COLS <= (int)TMEM_COLS && CTAS_PER_SM * TMEM_COLS <= 512, "tensor memory budget");
constexpr size_t SMEM_BYTES = 1024 + (size_t)STAGES * STAGE_BYTES + QBYTES;   // + 8 * (batch + 1)
constexpr int MAX_BATCH = 1024;
// kind::f8f6f4: D f32, A e4m3 (0), B e5m2 (1), both K-major, M = 128, N = 96:
// the three query parts sit side by side as 96 B rows, so one MMA per
// 32-dim K step scores a tile against all of them.
constexpr uint32_t IDESC = (1u << 4) | (0u << 7) | (1u << 10) | ((uint32_t)(ACC_COLS >> 3) << 17) | (8u << 24);

// 2-D views (rows of 128 bytes) of the summary plane (boxes of one page's
// 8 rows and of a whole 128-row tile) and of the key plane (boxes of one
// 64-row page and of a whole tile).
struct PlaneMaps {
    CUtensorMap summ8, summ128, keys64, keys128;
};

struct Params {
    CacheView c;
    int src;
    const uint16_t *q_idx;
    const float *w;
    float *scores;
    int64_t stride;
    uint4 *range;       // optional: per request and slot {max key, min key, min of the 32-row groups' maxima, -}
};

__device__ __forceinline__ int rows_of_req(const Params &p, int b)
{
    const int n = n_entries_of(p.c, b);
    return (p.src == ROWS_KEYS) ? n : (n + CSA2_BLOCK - 1) / CSA2_BLOCK;
}

// Walks this CTA's contiguous slice [i0, i1) of the global tile list, using
// the per-request row counts and tile prefix sums kept in shared memory.
struct TileIter {
    int b, t, rows, tiles, left;
    const int *s_rows, *s_pre;   // s_pre[b] = tiles of requests < b; s_pre[batch] = total
    int batch;
    __device__ void init(const int *rows_, const int *pre_, int batch_, long long i0, long long i1)
    {
        s_rows = rows_;
        s_pre = pre_;
        batch = batch_;
        left = (int)(i1 - i0);
        int lo = 0, hi = batch;                      // last b with s_pre[b] <= i0 and tiles > 0
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (s_pre[mid] <= i0) lo = mid; else hi = mid;
        }
        b = lo;
        while (b < batch - 1 && s_pre[b + 1] <= i0) ++b;
        rows = s_rows[b];
        tiles = s_pre[b + 1] - s_pre[b];
        t = (int)(i0 - s_pre[b]);
    }
    __device__ void next()
    {
        --left;
        if (left <= 0) return;
        ++t;
        while (t >= tiles) {
            ++b;
            t = 0;
            rows = s_rows[b];
            tiles = s_pre[b + 1] - s_pre[b];
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

__device__ __forceinline__ void mma_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc, uint32_t acc)
{
    asm volatile("{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
                 "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
                 "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(acc)
                 : "memory");
}


__global__ void __launch_bounds__(THREADS, CTAS_PER_SM)
score_umma_kernel(const __grid_constant__ PlaneMaps maps, Params p)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t *qbuf = sm + STAGES * STAGE_BYTES;
    __shared__ __align__(8) uint64_t full[STAGES], empty[STAGES], d_full[ACC], d_empty[ACC], q_full;
    __shared__ float wq[CSA2_IDX_HEADS];
    __shared__ uint32_t tmem_base;
    __shared__ long long s_total;
    __shared__ volatile int s_abort;
    __shared__ int win_b[2][PW], win_r0[2][PW], win_n[2][PW], win_pid[2][PW][16];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (warp == 5) tmem_alloc(&tmem_base, TMEM_COLS);
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
    int *s_rows = reinterpret_cast<int *>(qbuf + QBYTES), *s_pre = s_rows + p.c.batch;
    if (warp == 4) {
        // L2 hints while the previous kernel finishes: the request lengths,
        // and this CTA's share of the page table and of the queries (all of
        // them are hinted by the grid as a whole).
        const size_t nb = (size_t)p.c.batch * 4;
        prefetch_l2_range(p.c.n_tokens, 0, nb, lane, 8);
        prefetch_l2_range(p.c.m, 0, nb, lane, 8);
        const size_t pt = (size_t)p.c.batch * p.c.max_pages * 4, G = gridDim.x;
        prefetch_l2_range(p.c.page_table, pt * blockIdx.x / G, pt * (blockIdx.x + 1) / G, lane, 16);
        const size_t qb = (size_t)p.c.batch * CSA2_IDX_HEADS * CSA2_KEY_DIM * 2;
        prefetch_l2_range(p.q_idx, qb * blockIdx.x / G, qb * (blockIdx.x + 1) / G, lane, 4);
        if (blockIdx.x == 0) prefetch_l2_range(p.w, 0, (size_t)p.c.batch * CSA2_IDX_HEADS * 4, lane, 4);
    }
    grid_dependency_wait();                      // inputs may come from the previous kernel
    allow_dependents();
    if (warp == 0) {
        // rows and tile prefix sums of every request, 32 requests per round
        int carry = 0;
        for (int b0 = 0; b0 < p.c.batch; b0 += 32) {
            const int b = b0 + lane;
            const int rows = b < p.c.batch ? rows_of_req(p, b) : 0;
            const int tiles = (rows + TILE - 1) / TILE;
            int incl = tiles;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += v;
            }
            if (b < p.c.batch) {
                s_rows[b] = rows;
                s_pre[b] = carry + incl - tiles;
            }
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) {
            s_pre[p.c.batch] = carry;
            s_total = carry;
        }
    }
    __syncthreads();
    fence_after_sync();
    const uint32_t tb = tmem_base;
    const long long total = s_total;
    // [i0, i1) = [total * x / G, total * (x + 1) / G) with one 64-bit
    // division: total = tq G + tr, tr < G, so the rest is 32-bit.
    const uint32_t G = gridDim.x, x = blockIdx.x;
    const long long tq = total / G;
    const uint32_t tr = (uint32_t)(total - tq * G);
    const long long i0 = tq * x + tr * x / G, i1 = tq * (x + 1) + tr * (x + 1) / G;
    const int n_items = (int)(i1 - i0);
    volatile int *abort = &s_abort;

    if (warp == 4 && n_items > 0) {
        // ------------------------------------------------------------ producer
        // Page ids are looked up a window of PW tiles at a time, all lanes in
        // parallel, so the issue loop never waits on a dependent global load.
        const int chunk_rows = (p.src == ROWS_KEYS) ? 64 : 8;
        const int full_chunks = TILE / chunk_rows;                  // chunks of a complete tile
        const uint32_t chunk_bytes = (uint32_t)chunk_rows * CSA2_KEY_DIM;
        const int rows_per_page = (p.src == ROWS_SUMMARIES) ? 8 : 64;
        const CUtensorMap *m_chunk = (p.src == ROWS_SUMMARIES) ? &maps.summ8 : &maps.keys64;
        const CUtensorMap *m_tile = (p.src == ROWS_SUMMARIES) ? &maps.summ128 : &maps.keys128;
        if (lane == 0) {
            tma_prefetch_map(m_chunk);
            tma_prefetch_map(m_tile);
        }
        int issued = 0;
        bool stop = false;
        const int n_win = (n_items + PW - 1) / PW;
        // Window w's look-ups go to buffer w & 1.  The page-table loads of
        // window w + 1 are issued before window w's copies and consumed after
        // them, so their latency hides behind the copies.
        int e_[8], pg_[8];
        auto meta = [&](int w) {                    // lane i: tile i of window w
            const int wb = w & 1, nw = min(PW, n_items - w * PW);
            if (lane < nw) {
                const long long g = i0 + (long long)w * PW + lane;
                int lo = 0, hi = p.c.batch;         // the last request with s_pre[b] <= g owns tile g
                while (hi - lo > 1) {
                    const int mid = (lo + hi) >> 1;
                    if (s_pre[mid] <= g) lo = mid; else hi = mid;
                }
                const int t = (int)(g - s_pre[lo]);
                win_b[wb][lane] = lo;
                win_r0[wb][lane] = t * TILE;
                win_n[wb][lane] = (min(TILE, s_rows[lo] - t * TILE) + chunk_rows - 1) / chunk_rows;
            }
            __syncwarp();
        };
        auto issue_loads = [&](int w) {             // non-blocking: loads in flight
            // Every lane loads for every u with no branch around the load: with
            // each load under a lane-divergent branch the eight look-ups of a
            // lane were measured to complete one after another (eight memory
            // latencies); unconditional loads from clamped addresses are in
            // flight together.  A dead or out-of-range chunk reads entry 0,
            // which always exists.
            const int wb = w & 1, nw = min(PW, n_items - w * PW);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int k = lane + 32 * u, i = k >> 4, ch = k & 15;
                const bool live = i < nw && ch < win_n[wb][i];
                const int b = live ? win_b[wb][i] : 0, r0 = live ? win_r0[wb][i] : 0;
                const int e = (p.src == ROWS_SUMMARIES) ? (r0 + 8 * ch) * CSA2_BLOCK : r0 + 64 * ch;
                const bool in_pt = live && (e >> 6) < p.c.max_pages;
                e_[u] = live ? e : -1;
                pg_[u] = p.c.page_table[in_pt ? (size_t)b * p.c.max_pages + (e >> 6) : 0];
            }
        };
        auto finish = [&](int w) {                  // blocking: checks, then shared memory
            const int wb = w & 1, nw = min(PW, n_items - w * PW);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int k = lane + 32 * u, i = k >> 4, ch = k & 15;
                const int e = e_[u], pg = pg_[u];
                int pid = -1;
                if (e >= 0) {
                    if ((e >> 6) >= p.c.max_pages) {
                        set_error(p.c.error, CSA2_DEV_CAPACITY);
                    } else if (pg < 0 || pg >= p.c.n_pages) {
                        set_error(p.c.error, CSA2_DEV_BAD_PAGE);
                    } else {
                        pid = pg * rows_per_page + ((p.src == ROWS_SUMMARIES) ? 0 : (e & 63));   // plane row
                    }
                }
                if (i < nw) win_pid[wb][i][ch] = pid;
            }
            __syncwarp();
        };
        meta(0);
        issue_loads(0);
        finish(0);
        for (int w = 0; w < n_win && !stop; ++w) {
            const int wb = w & 1, nw = min(PW, n_items - w * PW);
            if (w + 1 < n_win) {
                meta(w + 1);
                issue_loads(w + 1);
            }
            for (int i = 0; i < nw; ++i) {
                const int j = w * PW + i, s = j % STAGES;
                bool okw = true;
                if (lane == 0 && j >= STAGES) okw = wait_or_abort(&empty[s], ((j / STAGES) - 1) & 1, abort, p.c.error);
                if (!__shfl_sync(0xffffffffu, okw, 0)) {          // warp-uniform decision
                    stop = true;
                    break;
                }
                const int row = lane < 16 ? win_pid[wb][i][lane] : -1;       // first plane row of the chunk
                const uint32_t ok = __ballot_sync(0xffffffffu, row >= 0);
                const int row0 = __shfl_sync(0xffffffffu, row, 0);
                const bool contig = __popc(ok) == full_chunks &&
                                    __all_sync(0xffffffffu, lane >= full_chunks || row == row0 + lane * chunk_rows);
                uint8_t *dst = sm + s * STAGE_BYTES;
                if (contig) {
                    // the whole tile is one run of plane rows: a single 16 KB copy
                    if (lane == 0) {
                        mbar_arrive_expect_tx(&full[s], STAGE_BYTES);
                        tma_load_2d(dst, m_tile, 0, row0, &full[s]);
                    }
                } else {
                    if (lane == 0) mbar_arrive_expect_tx(&full[s], __popc(ok) * chunk_bytes);
                    __syncwarp();
                    if (row >= 0) tma_load_2d(dst + lane * chunk_bytes, m_chunk, 0, row, &full[s]);
                }
                __syncwarp();
                issued = j + 1;
            }
            if (!stop && w + 1 < n_win) finish(w + 1);
        }
        // Never leave with copies in flight: wait for the last stages to land.
        if (lane == 0)
            for (int j = max(0, issued - STAGES); j < issued; ++j) mbar_wait(&full[j % STAGES], (j / STAGES) & 1);
        __syncwarp();
    } else if (warp == 5 && n_items > 0) {
        // ------------------------------------------------------------ MMA issuer
        TileIter it;
        it.init(s_rows, s_pre, p.c.batch, i0, i1);
        int cur_b = -1, sw = -1, issued = 0;
        const uint32_t qaddr = smem_addr(qbuf);
        for (int j = 0; j < n_items; ++j, it.next()) {
            const int ab = j % ACC, s = j % STAGES;
            bool okw = true;
            if (lane == 0) {
                if (it.b != cur_b) okw = wait_or_abort(&q_full, (sw + 1) & 1, abort, p.c.error);
                if (okw) okw = wait_or_abort(&full[s], (j / STAGES) & 1, abort, p.c.error);
                if (okw && j >= ACC) okw = wait_or_abort(&d_empty[ab], ((j / ACC) - 1) & 1, abort, p.c.error);
            }
            if (it.b != cur_b) {
                cur_b = it.b;
                ++sw;
            }
            if (!__shfl_sync(0xffffffffu, okw, 0)) break;          // warp-uniform decision
            fence_after_sync();
            if (lane == 0) {
                const uint32_t aaddr = smem_addr(sm + s * STAGE_BYTES);
#pragma unroll
                for (int kk = 0; kk < CSA2_KEY_DIM / 32; ++kk)
                    mma_f8(tb + ACC_COLS * ab, smem_desc(aaddr + kk * 32, 16, 1024),
                           smem_desc(qaddr + kk * 32, 16, 1024), IDESC, kk > 0 ? 1u : 0u);
                mma_commit(&d_full[ab]);
                mma_commit(&empty[s]);                              // stage free once the MMAs have read it
            }
            __syncwarp();
            issued = j + 1;
        }
        if (lane == 0)
            for (int j = max(0, issued - ACC); j < issued; ++j) mbar_wait(&d_full[j % ACC], (j / ACC) & 1);
        __syncwarp();
    } else if (warp < 4 && n_items > 0) {
        // ------------------------------------------------------------ workers
        TileIter it;
        it.init(s_rows, s_pre, p.c.batch, i0, i1);
        const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
        int cur_b = -1;
        float wr[CSA2_IDX_HEADS];                                  // this request's w'
        // The request's range over this warp's rows, folded into one of its
        // slots once per request and warp (the slots spread the atomics: a
        // few dozen per word).
        uint32_t r_mx = 0u, r_mn = 0xffffffffu, r_lb = 0xffffffffu;
        auto fold_range = [&](int b) {
            if (p.range && b >= 0 && lane == 0 && r_mx >= r_mn) {
                uint4 *r = p.range + (size_t)b * RANGE_SLOTS + ((blockIdx.x * 4 + warp) % RANGE_SLOTS);
                atomicMax(&r->x, r_mx);
                atomicMin(&r->y, r_mn);
                atomicMin(&r->z, r_lb);
            }
            r_mx = 0u;
            r_mn = r_lb = 0xffffffffu;
        };
        for (int j = 0; j < n_items; ++j, it.next()) {
            if (it.b != cur_b) {
                // New request.  Every MMA issued so far has completed (the
                // previous epilogue waited for it), so the q buffer is free.
                fold_range(cur_b);
                cur_b = it.b;
                iq_split(tid, p.q_idx, p.w, cur_b, qbuf, wq);
                fence_proxy_async_smem();
                bar_workers();
                if (tid == 0) mbar_arrive(&q_full);
#pragma unroll
                for (int hh = 0; hh < CSA2_IDX_HEADS; ++hh) wr[hh] = wq[hh];
            }
            // ---- epilogue of tile j
            const int db = j % ACC;
            const bool ok = wait_or_abort(&d_full[db], (j / ACC) & 1, abort, p.c.error);
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
            const int row = it.t * TILE + tid;
            const bool valid = ok && row < it.rows;
            if (valid) p.scores[(size_t)it.b * p.stride + row] = sc;
            if (p.range) {
                // this warp's 32 rows: their largest and smallest key, and
                // the smallest maximum of their groups of g rows that hold a
                // key (g the same for the whole request)
                const uint32_t key = valid ? sel::ord_key(sc) : 0u;
                const uint32_t mx = __reduce_max_sync(0xffffffffu, key);
                const uint32_t mn = __reduce_min_sync(0xffffffffu, valid ? key : 0xffffffffu);
                const int g = range_group(it.rows);           // the same in every lane
                uint32_t lb = mx;                             // g = 32: the warp is the group
                if (g < 32) {
                    uint32_t gm = key;
                    for (int o = g >> 1; o; o >>= 1) gm = max(gm, __shfl_xor_sync(0xffffffffu, gm, o));
                    const bool lead = (lane & (g - 1)) == 0 && row < it.rows && ok;
                    lb = __reduce_min_sync(0xffffffffu, lead ? gm : 0xffffffffu);
                }
                if (mx >= mn) {
                    r_mx = max(r_mx, mx);
                    r_mn = min(r_mn, mn);
                    r_lb = min(r_lb, lb);
                }
            }
        }
        fold_range(cur_b);
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 5) {
        fence_after_sync();
        tmem_dealloc(tb, TMEM_COLS);
    }
}

}  // namespace

// ---------------------------------------------------------------- host side
// 2-D byte tensor over a plane: rows of 128 bytes, boxes of box_rows rows,
// 128-byte swizzled.
bool make_plane_map(CUtensorMap *m, void *base, long long rows, int box_rows)
{
    auto fn = tensor_map_encoder();
    if (!fn) return false;
    cuuint64_t dims[2] = {128, (cuuint64_t)rows};
    cuuint64_t strides[1] = {128};
    cuuint32_t box[2] = {128, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

cudaError_t launch_score(const CacheView &c, int src, const uint16_t *q_idx, const float *w, float *scores,
                         int64_t stride, cudaStream_t st, uint4 *range)
{
    if (c.batch > MAX_BATCH || (src != ROWS_KEYS && src != ROWS_SUMMARIES)) return cudaErrorInvalidValue;
    static DeviceOnce once;
    static int n_sm[DeviceOnce::N] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess)
        e = once.run(dev, [&] {
            int v = 0;
            cudaError_t r = cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
            if (r == cudaSuccess)
                r = cudaFuncSetAttribute(score_umma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)(SMEM_BYTES + 8 * (MAX_BATCH + 1)));
            n_sm[dev] = v > 0 ? v : 148;
            return r;
        });
    if (e != cudaSuccess) return e;
    PlaneMaps maps;
    const long long np = c.n_pages;
    if (!make_plane_map(&maps.summ8, c.summ, np * 8, 8) || !make_plane_map(&maps.summ128, c.summ, np * 8, 128) ||
        !make_plane_map(&maps.keys64, c.keys, np * 64, 64) || !make_plane_map(&maps.keys128, c.keys, np * 64, 128))
        return cudaErrorInvalidValue;
    Params p{c, src, q_idx, w, scores, stride, range};
    const int kid = src == ROWS_KEYS ? CSA2_KERNEL_FLAT_SCORE : CSA2_KERNEL_BLOCK_SCORE;
    const size_t smem = SMEM_BYTES + 8 * ((size_t)c.batch + 1);
    LaunchScope scope(kid, st);
    return launch_pdl(score_umma_kernel, dim3(CTAS_PER_SM * n_sm[dev]), dim3(THREADS), smem, st, maps, p);
}

}  // namespace csa2

// Indexer selection: an exact radix top-k (score descending, ties to the
// lower index) whose output is the selected ids in ascending order.  The
// scores come from score_umma.cu.
//
// Sources: 0539edu.com/news/5732216 §3 (indexer 32 heads x 128, top_k 512,
// hierarchical 2048 blocks x 8 positions -> 16384 candidates; Full builds the
// pool, Reindex searches inside it).
#include <cooperative_groups.h>

#include "common.cuh"
#include "index.cuh"
#include "select.cuh"

namespace cg = cooperative_groups;

namespace csa2 {

// ------------------------------------------------------------------ top-k
// Each row runs on one CTA or on a cluster of 4, 8 or 16, chosen per launch
// by a cost model: resident waves x (the exchange rounds' fixed cost + the
// per-CTA key passes).
constexpr int SEL_THREADS = 1024;
constexpr int SEL_CAP = 32768;         // keys a CTA keeps in shared memory (128 KB)
constexpr double SELECT_ROUNDS_US[4] = {2.0, 8.0, 9.0, 10.0};   // fixed cost for 1, 4, 8, 16 CTAs
constexpr double SELECT_KEY_NS = 1.5;                            // per key a CTA holds
constexpr int SEL_BITS = SEL_CAP / 32;
constexpr size_t SEL_SMEM = (size_t)(SEL_CAP + 2 * sel::CAND + 2 * sel::RANK_MAX + SEL_BITS) * sizeof(uint32_t);

// One cluster of NC CTAs per row (grid = NC x batch; NC = 1 is a plain
// CTA and uses no cluster barriers).  Selects the top min(k, n) of
// scores[b][0..n) -- score descending, ties to the lower index -- and writes
// the selected ids in ascending order to out[b][0..k) (-1 padded).  The id of
// element i is i, or ids[b][i] when ids != nullptr.  With expand the selected
// ids are block numbers: the pool of their entries (< n_entries) is written
// to pool[b][0..16384) in ascending order and its length to pool_len[b].
// Optionally the selected scores go to vals[b][0..k) (-inf padded) and
// (id_off[b] >> id_shift) is added to every written id.
// CTA r owns the contiguous index range [r*chunk, (r+1)*chunk) and stages
// its keys in shared memory (or re-reads global memory when chunk > SEL_CAP).
template <int NC>
__device__ __forceinline__ void select_body(CacheView c, int src, const float *scores, int64_t score_stride, const int32_t *pool_len_in,
                      const int32_t *ids, int k, int32_t *out, int out_stride, int expand, int32_t *pool,
                      int32_t *pool_len, float *vals, const int32_t *id_off, int id_shift, uint4 *range)
{
    extern __shared__ uint32_t dsm[];
    const int rank = (NC > 1) ? (int)cg::this_cluster().block_rank() : 0;
    const int b = blockIdx.y;
    const int tid = threadIdx.x;
    grid_dependency_wait();                      // scores come from the previous kernel
    allow_dependents();
    // ROWS_GIVEN: a bare score matrix, row lengths in pool_len_in, no cache.
    const int n_entries = (src == ROWS_GIVEN) ? 0 : n_entries_of(c, b);
    const int n = (src == ROWS_KEYS) ? n_entries
                : (src == ROWS_SUMMARIES) ? (n_entries + CSA2_BLOCK - 1) / CSA2_BLOCK
                                          : (int)max((int64_t)0, min((int64_t)pool_len_in[b], score_stride));
    const int chunk = (n + NC - 1) / NC;
    const int lo = rank * chunk;
    const int cnt = max(0, min(n, lo + chunk) - lo);
    const bool in_smem = chunk <= SEL_CAP;
    const float *s = scores + (size_t)b * score_stride + lo;

    uint32_t *keys = dsm;
    sel::Bufs bf;
    bf.keys = in_smem ? keys : nullptr;
    bf.scores = s;
    bf.cand_key = dsm + SEL_CAP;
    bf.cand_idx = bf.cand_key + sel::CAND;
    bf.all_key = bf.cand_idx + sel::CAND;
    bf.all_idx = bf.all_key + sel::RANK_MAX;
    bf.bits = bf.all_idx + sel::RANK_MAX;
    bf.bits_words = SEL_BITS;
    uint32_t kmin = 0xffffffffu, kmax = 0u;
    // The scan's range of the request's keys, when it kept one: then the
    // selection needs no exchange between its CTAs to find it.  Slots that a
    // selection has reset carry RANGE_TAG in their last word (the scan's
    // atomics leave it alone); until every slot does (a fresh workspace),
    // the exchange runs instead.  Every CTA of the cluster reads the same
    // words and takes the same decision.
    __shared__ uint32_t s_range[4];
    __shared__ int s_use_range;
    static_assert(RANGE_SLOTS == 32, "one slot per lane");
    if (tid < 32) {
        bool ok = range != nullptr && n > k;
        uint4 r = make_uint4(0u, 0xffffffffu, 0xffffffffu, 0u);
        if (ok) r = range[(size_t)b * RANGE_SLOTS + tid];
        ok = __all_sync(0xffffffffu, ok && r.w == RANGE_TAG);
        const uint32_t mx = __reduce_max_sync(0xffffffffu, r.x), mn = __reduce_min_sync(0xffffffffu, r.y);
        const uint32_t lb = __reduce_min_sync(0xffffffffu, r.z);
        if (tid == 0) {
            s_use_range = ok;
            s_range[0] = mn;                       // smallest key
            s_range[1] = mx;                       // largest key
            const int g = range_group(n);
            s_range[2] = lb;                       // smallest maximum of a group of g rows
            s_range[3] = (uint32_t)((n + g - 1) / g);  // groups of g rows, each with at least one key
        }
    }
    if (in_smem) {
        // 8 independent loads in flight per thread per round.
        for (int e0 = 0; e0 < cnt; e0 += 8 * SEL_THREADS) {
            float v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int e = e0 + u * SEL_THREADS + tid;
                v[u] = e < cnt ? s[e] : 0.0f;
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int e = e0 + u * SEL_THREADS + tid;
                if (e < cnt) {
                    const uint32_t key = sel::ord_key(v[u]);
                    keys[e] = key;
                    kmin = min(kmin, key);
                    kmax = max(kmax, key);
                }
            }
        }
    } else {
        for (int e = tid; e < cnt; e += SEL_THREADS) {
            const uint32_t key = sel::ord_key(s[e]);
            kmin = min(kmin, key);
            kmax = max(kmax, key);
        }
    }
    __syncthreads();
    sel::Out o;
    o.out = out;
    o.out_stride = out_stride;
    o.ids = ids;
    o.expand = expand;
    o.pool = pool;
    o.pool_len = pool_len;
    o.n_entries = n_entries;
    o.vals = vals;
    o.id_off = id_off;
    o.id_shift = id_shift;
    sel::select_core<NC, SEL_THREADS>(bf, b, n, chunk, lo, cnt, k, kmin, kmax, o, s_use_range ? s_range : nullptr);
    // Every CTA of the cluster read the range before the last cluster
    // barrier: start the next scan's reduction from the empty range.
    if (range != nullptr && rank == 0 && tid < RANGE_SLOTS)
        range[(size_t)b * RANGE_SLOTS + tid] = make_uint4(0u, 0xffffffffu, 0xffffffffu, RANGE_TAG);
}

#define CSA2_SELECT_ARGS                                                                                      \
    CacheView c, int src, const float *scores, int64_t score_stride, const int32_t *pool_len_in,               \
        const int32_t *ids, int k, int32_t *out, int out_stride, int expand, int32_t *pool, int32_t *pool_len,    \
        float *vals, const int32_t *id_off, int id_shift, uint4 *range
#define CSA2_SELECT_PASS \
    c, src, scores, score_stride, pool_len_in, ids, k, out, out_stride, expand, pool, pool_len, vals, id_off, id_shift, \
        range

template <int NC>
__global__ void __launch_bounds__(SEL_THREADS, 1) select_cluster_kernel(CSA2_SELECT_ARGS)
{
    select_body<NC>(CSA2_SELECT_PASS);
}

__global__ void __launch_bounds__(SEL_THREADS, 1) select_cta_kernel(CSA2_SELECT_ARGS)
{
    select_body<1>(CSA2_SELECT_PASS);
}

// ------------------------------------------------------------------ launchers
namespace {

// CTAs per request for a selection over at most max_n rows: a cluster of
// 16, 8 or 4 CTAs, or one CTA (no cluster barriers).  act[i]: how many
// selections of 1, 4, 8 and 16 CTAs can be resident at once.  Rows longer
// than any size keeps in shared memory take the largest cluster the device
// can run (its CTAs then re-read the scores from global memory).
int select_ctas(int batch, int max_n, const int act[4])
{
    static const int sizes[4] = {1, 4, 8, 16};
    int best = act[3] >= 1 ? 16 : act[2] >= 1 ? 8 : 4;
    double best_us = 1e30;
    for (int i = 0; i < 4; ++i) {
        const int nc = sizes[i];
        const long long chunk = ((long long)max_n + nc - 1) / nc;
        if (chunk > SEL_CAP || act[i] < 1) continue;
        const long long waves = (batch + act[i] - 1) / act[i];
        const double us = (double)waves * (SELECT_ROUNDS_US[i] + SELECT_KEY_NS * 1e-3 * (double)chunk);
        if (us < best_us) {
            best_us = us;
            best = nc;
        }
    }
    return best;
}

}  // namespace

cudaError_t launch_select(const CacheView &c, int src, const float *scores, int64_t stride, const int32_t *pool_len_in,
                          const int32_t *ids, int k, int32_t *out, int out_stride, int expand, int32_t *pool,
                          int32_t *pool_len, int max_n, cudaStream_t st, float *vals, const int32_t *id_off,
                          int id_shift, uint4 *range)
{
    static DeviceOnce once;
    static int active[DeviceOnce::N][4] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    const int smem = (int)SEL_SMEM;
    if (e == cudaSuccess)
        e = once.run(dev, [&] {
            cudaError_t r = cudaFuncSetAttribute(select_cta_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
            if (r == cudaSuccess)
                r = cudaFuncSetAttribute(select_cluster_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
            if (r == cudaSuccess)
                r = cudaFuncSetAttribute(select_cluster_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
            if (r == cudaSuccess)
                r = cudaFuncSetAttribute(select_cluster_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
            if (r == cudaSuccess)
                r = cudaFuncSetAttribute(select_cluster_kernel<16>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
            if (r != cudaSuccess) return r;
            int per_sm = 0, sms = 0;
            if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, select_cta_kernel, SEL_THREADS, smem) !=
                    cudaSuccess ||
                cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
                cudaGetLastError();
                per_sm = sms = 0;
            }
            active[dev][0] = per_sm * sms;
            active[dev][1] = max_active_clusters(select_cluster_kernel<4>, dim3(SEL_THREADS), smem, 4);
            active[dev][2] = max_active_clusters(select_cluster_kernel<8>, dim3(SEL_THREADS), smem, 8);
            active[dev][3] = max_active_clusters(select_cluster_kernel<16>, dim3(SEL_THREADS), smem, 16);
            return cudaSuccess;
        });
    if (e != cudaSuccess) return e;
    const int nc = select_ctas(c.batch, max_n, active[dev]);
    LaunchScope scope(CSA2_KERNEL_SELECT, st);
    if (nc == 1)
        return launch_pdl(select_cta_kernel, dim3(1, c.batch), dim3(SEL_THREADS), smem, st, c, src, scores, stride,
                          pool_len_in, ids, k, out, out_stride, expand, pool, pool_len, vals, id_off, id_shift,
                          range);
    if (nc == 4)
        return launch_pdl_cluster(select_cluster_kernel<4>, dim3(4, c.batch), dim3(SEL_THREADS), smem, st, 4, c, src,
                                  scores, stride, pool_len_in, ids, k, out, out_stride, expand, pool, pool_len, vals,
                                  id_off, id_shift, range);
    if (nc == 8)
        return launch_pdl_cluster(select_cluster_kernel<8>, dim3(8, c.batch), dim3(SEL_THREADS), smem, st, 8, c, src,
                                  scores, stride, pool_len_in, ids, k, out, out_stride, expand, pool, pool_len, vals,
                                  id_off, id_shift, range);
    return launch_pdl_cluster(select_cluster_kernel<16>, dim3(16, c.batch), dim3(SEL_THREADS), smem, st, 16, c, src,
                              scores, stride, pool_len_in, ids, k, out, out_stride, expand, pool, pool_len, vals,
                              id_off, id_shift, range);
}

}  // namespace csa2

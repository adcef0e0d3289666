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

namespace cg = cooperative_groups;

namespace csa2 {

// ------------------------------------------------------------------ top-k
// Order-preserving 32-bit key of an fp32 score (-0 folded onto +0).
__device__ __forceinline__ uint32_t ord_key(float x)
{
    uint32_t u = __float_as_uint(x);
    if (u == 0x80000000u) u = 0;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

constexpr int SEL_CLUSTER = 8;         // CTAs per request (one thread-block cluster)
constexpr int SEL_THREADS = 1024;
constexpr int SEL_CAP = 32768;         // keys a CTA keeps in shared memory (128 KB)
constexpr int SEL_CAND = 2048;         // candidate keys kept after the first radix pass

// Inclusive scan over threads 0..255 (warps 0..7); every thread of the CTA
// must call it.  Returns the prefix for threads < 256.
__device__ __forceinline__ uint32_t scan256(uint32_t v, uint32_t *scratch)
{
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        uint32_t t = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += t;
    }
    if (wid < 8 && lane == 31) scratch[wid] = v;
    __syncthreads();
    uint32_t add = 0;
    if (wid < 8)
        for (int i = 0; i < wid; ++i) add += scratch[i];
    __syncthreads();
    return v + add;
}

// One cluster of NC CTAs per request (grid = NC x batch; NC = 1 is a plain
// CTA and uses no cluster barriers).  Selects the top
// min(k, n) of scores[b][0..n) -- score descending, ties to the lower index --
// and writes the selected ids in ascending order to out[b][0..k) (-1 padded).
// The id of element i is i, or ids[b][i] when ids != nullptr.  With expand the
// selected ids are block numbers: the pool of their entries (< n_entries) is
// written to pool[b][0..16384) in ascending order and its length to
// pool_len[b].
// CTA r owns the contiguous index range [r*chunk, (r+1)*chunk) and keeps its
// order-preserving keys in shared memory (falls back to re-reading global
// memory when chunk > SEL_CAP).  Four 8-bit radix passes find the exact
// threshold key T and how many ties at T to keep; the per-CTA histograms and
// the final per-CTA counts are exchanged through distributed shared memory.
template <int NC>
__device__ __forceinline__ void select_body(CacheView c, int src, const float *scores, int64_t score_stride, const int32_t *pool_len_in,
                      const int32_t *ids, int k, int32_t *out, int out_stride, int expand, int32_t *pool,
                      int32_t *pool_len)
{
    extern __shared__ uint32_t keys[];
    __shared__ uint32_t hist[2][256];
    __shared__ uint32_t whist[32][256];
    __shared__ uint32_t scratch[32];
    __shared__ uint32_t wsum[32][2];
    __shared__ uint32_t s_cnt[2];
    __shared__ uint32_t s_digit, s_above;
    const int rank = (NC > 1) ? (int)cg::this_cluster().block_rank() : 0;
    auto csync = [&]() {
        if constexpr (NC > 1) cg::this_cluster().sync();
        else __syncthreads();
    };
    auto remote = [&](uint32_t *ptr, int r) -> uint32_t * {
        if constexpr (NC > 1) return cg::this_cluster().map_shared_rank(ptr, r);
        else return ptr;
    };
    const int b = blockIdx.y;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    grid_dependency_wait();                      // scores come from the previous kernel
    allow_dependents();
    const int n_entries = n_entries_of(c, b);
    const int n = (src == ROWS_KEYS) ? n_entries
                : (src == ROWS_SUMMARIES) ? (n_entries + CSA2_BLOCK - 1) / CSA2_BLOCK
                                          : max(0, min(pool_len_in[b], CSA2_POOL));
    const int kk = min(k, n);
    const bool take_all = n <= k;
    const int chunk = (n + NC - 1) / NC;
    const int lo = rank * chunk;
    const int cnt = max(0, min(n, lo + chunk) - lo);
    const bool in_smem = chunk <= SEL_CAP;
    const int seg = ((cnt + 32 * 32 - 1) / (32 * 32)) * 32;     // elements per warp, multiple of 32
    const float *s = scores + (size_t)b * score_stride + lo;
    auto key_at = [&](int e) -> uint32_t { return in_smem ? keys[e] : ord_key(s[e]); };

    uint32_t *cand_key = keys + SEL_CAP, *cand_idx = cand_key + SEL_CAND;
    uint32_t kmin = 0xffffffffu, kmax = 0u;
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
                    const uint32_t key = ord_key(v[u]);
                    keys[e] = key;
                    kmin = min(kmin, key);
                    kmax = max(kmax, key);
                }
            }
        }
    } else {
        for (int e = tid; e < cnt; e += SEL_THREADS) {
            const uint32_t key = ord_key(s[e]);
            kmin = min(kmin, key);
            kmax = max(kmax, key);
        }
    }
    uint32_t prefix = 0, pmask = 0, krem = (uint32_t)kk;
    if (!take_all) {
        // Range of the keys across the cluster: their common leading bits
        // (sign, most of the exponent) need no radix pass.
#pragma unroll
        for (int o = 16; o; o >>= 1) {
            kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
            kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
        }
        if (lane == 0) {
            wsum[wid][0] = kmin;
            wsum[wid][1] = kmax;
        }
        __syncthreads();
        if (tid == 0) {
            uint32_t a = 0xffffffffu, z = 0u;
            for (int i = 0; i < 32; ++i) {
                a = min(a, wsum[i][0]);
                z = max(z, wsum[i][1]);
            }
            s_cnt[0] = a;
            s_cnt[1] = z;
        }
        csync();
        uint32_t gmin = 0xffffffffu, gmax = 0u;
        for (int r = 0; r < NC; ++r) {
            const uint32_t *rc = remote(&s_cnt[0], r);
            gmin = min(gmin, rc[0]);
            gmax = max(gmax, rc[1]);
        }
        int hi = 32 - __clz(gmin ^ gmax);                  // bits [hi-1 .. 0] vary
        pmask = hi >= 32 ? 0u : ~((1u << hi) - 1u);
        prefix = gmax & pmask;
        bool use_cand = false;                              // later passes scan only candidates
        int n_cand = 0;
        for (int pass = 0; hi > 0; ++pass) {
            const int wdt = min(8, hi), shift = hi - wdt, buf = pass & 1;
            const uint32_t dmask = (1u << wdt) - 1u;
            for (int i = tid; i < 32 * 256; i += SEL_THREADS) whist[i >> 8][i & 255] = 0;
            __syncthreads();
            if (use_cand) {
                for (int ci = tid; ci < n_cand; ci += SEL_THREADS) {
                    const uint32_t key = cand_key[ci];
                    if ((key & pmask) == prefix) atomicAdd(&whist[wid][(key >> shift) & dmask], 1u);
                }
            } else {
                for (int it = 0; it < seg; it += 32) {
                    const int e = wid * seg + it + lane;
                    if (e < cnt) {
                        const uint32_t key = key_at(e);
                        if ((key & pmask) == prefix) atomicAdd(&whist[wid][(key >> shift) & dmask], 1u);
                    }
                }
            }
            __syncthreads();
            if (tid < 256) {
                uint32_t t = 0;
#pragma unroll 8
                for (int w = 0; w < 32; ++w) t += whist[w][tid];
                hist[buf][tid] = t;
            }
            __syncthreads();
            csync();
            // Cluster-wide count of bin 255 - tid, then counts of bins >= it.
            uint32_t hv = 0;
            if (tid < 256) {
                uint32_t part[NC];
#pragma unroll
                for (int r = 0; r < NC; ++r) part[r] = remote(&hist[buf][0], r)[255 - tid];
#pragma unroll
                for (int r = 0; r < NC; ++r) hv += part[r];
            }
            const uint32_t incl = scan256(hv, scratch);
            if (tid < 256 && incl >= krem && incl - hv < krem) {
                s_digit = 255u - tid;
                s_above = incl - hv;
            }
            __syncthreads();
            prefix |= s_digit << shift;
            pmask |= dmask << shift;
            krem -= s_above;
            hi = shift;
            if (pass == 0 && hi > 0) {
                // Keep the keys that still match: usually a few hundred.
                if (tid == 0) s_cnt[0] = 0;
                __syncthreads();
                for (int it = 0; it < seg; it += 32) {
                    const int e = wid * seg + it + lane;
                    const uint32_t key = e < cnt ? key_at(e) : 0u;
                    const bool m = e < cnt && (key & pmask) == prefix;
                    const uint32_t mb = __ballot_sync(0xffffffffu, m);
                    uint32_t base = 0;
                    if (lane == 0 && mb) base = atomicAdd(&s_cnt[0], (uint32_t)__popc(mb));
                    base = __shfl_sync(0xffffffffu, base, 0);
                    const uint32_t pos = base + __popc(mb & ((1u << lane) - 1u));
                    if (m && pos < (uint32_t)SEL_CAND) {
                        cand_key[pos] = key;
                        cand_idx[pos] = (uint32_t)e;
                    }
                }
                __syncthreads();
                n_cand = (int)s_cnt[0];
                use_cand = n_cand <= SEL_CAND;
                __syncthreads();
            }
        }
    }
    const uint32_t T = prefix;
    // Per-warp counts of keys above T and equal to T, in index order.
    uint32_t ngt = 0, neq = 0;
    for (int it = 0; it < seg; it += 32) {
        const int e = wid * seg + it + lane;
        const bool valid = e < cnt;
        const uint32_t key = valid ? key_at(e) : 0u;
        ngt += __popc(__ballot_sync(0xffffffffu, valid && (take_all || key > T)));
        neq += __popc(__ballot_sync(0xffffffffu, valid && !take_all && key == T));
    }
    if (lane == 0) {
        wsum[wid][0] = ngt;
        wsum[wid][1] = neq;
    }
    __syncthreads();
    if (tid == 0) {
        uint32_t g = 0, q = 0;
        for (int i = 0; i < 32; ++i) {
            uint32_t a = wsum[i][0], bq = wsum[i][1];
            wsum[i][0] = g;
            wsum[i][1] = q;
            g += a;
            q += bq;
        }
        s_cnt[0] = g;
        s_cnt[1] = q;
    }
    __syncthreads();
    csync();
    uint32_t gt_b = 0, eq_b = 0;
    for (int r = 0; r < rank; ++r) {
        const uint32_t *rc = remote(&s_cnt[0], r);
        gt_b += rc[0];
        eq_b += rc[1];
    }
    gt_b += wsum[wid][0];
    eq_b += wsum[wid][1];
    const uint32_t lt_mask = (1u << lane) - 1u;
    for (int it = 0; it < seg; it += 32) {
        const int e = wid * seg + it + lane;
        const bool valid = e < cnt;
        const uint32_t key = valid ? key_at(e) : 0u;
        const bool g = valid && (take_all || key > T);
        const bool q = valid && !take_all && key == T;
        const uint32_t bg = __ballot_sync(0xffffffffu, g), bq = __ballot_sync(0xffffffffu, q);
        const uint32_t my_gt = gt_b + __popc(bg & lt_mask), my_eq = eq_b + __popc(bq & lt_mask);
        const int gi = lo + e;
        if (g || (q && my_eq < krem)) {
            const uint32_t pos = my_gt + min(my_eq, krem);
            if (expand) {
                for (int j = 0; j < CSA2_BLOCK; ++j) {
                    const int en = gi * CSA2_BLOCK + j;
                    pool[(size_t)b * CSA2_POOL + pos * CSA2_BLOCK + j] = en < n_entries ? en : -1;
                }
            } else {
                out[(size_t)b * out_stride + pos] = ids ? ids[(size_t)b * CSA2_POOL + gi] : gi;
            }
        }
        if (expand && valid && gi == n - 1) {
            const bool sel_last = g || (q && my_eq < krem);
            pool_len[b] = kk * CSA2_BLOCK - (sel_last ? n * CSA2_BLOCK - n_entries : 0);
        }
        gt_b += __popc(bg);
        eq_b += __popc(bq);
    }
    if (rank == 0) {
        if (expand) {
            for (int i = kk * CSA2_BLOCK + tid; i < CSA2_POOL; i += SEL_THREADS) pool[(size_t)b * CSA2_POOL + i] = -1;
            if (n == 0 && tid == 0) pool_len[b] = 0;
        } else {
            for (int i = kk + tid; i < k; i += SEL_THREADS) out[(size_t)b * out_stride + i] = -1;
        }
    }
    // No CTA may leave while another still reads its shared memory.
    csync();
}

#define CSA2_SELECT_ARGS                                                                                      \
    CacheView c, int src, const float *scores, int64_t score_stride, const int32_t *pool_len_in,               \
        const int32_t *ids, int k, int32_t *out, int out_stride, int expand, int32_t *pool, int32_t *pool_len
#define CSA2_SELECT_PASS c, src, scores, score_stride, pool_len_in, ids, k, out, out_stride, expand, pool, pool_len

__global__ void __cluster_dims__(SEL_CLUSTER, 1, 1) __launch_bounds__(SEL_THREADS, 1)
select_cluster_kernel(CSA2_SELECT_ARGS)
{
    select_body<SEL_CLUSTER>(CSA2_SELECT_PASS);
}

__global__ void __launch_bounds__(SEL_THREADS, 1) select_cta_kernel(CSA2_SELECT_ARGS)
{
    select_body<1>(CSA2_SELECT_PASS);
}

// ------------------------------------------------------------------ launchers
cudaError_t launch_select(const CacheView &c, int src, const float *scores, int64_t stride, const int32_t *pool_len_in,
                          const int32_t *ids, int k, int32_t *out, int out_stride, int expand, int32_t *pool,
                          int32_t *pool_len, int max_n, cudaStream_t st)
{
    static bool attr_done[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    const int smem = (SEL_CAP + 2 * SEL_CAND) * (int)sizeof(uint32_t);
    if (dev >= 64 || !attr_done[dev]) {
        e = cudaFuncSetAttribute(select_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(select_cta_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        if (dev < 64) attr_done[dev] = true;
    }
    LaunchScope scope(CSA2_KERNEL_SELECT, st);
    if (max_n <= SEL_CAP)   // fits one CTA's shared memory: no cluster barriers on the path
        return launch_pdl(select_cta_kernel, dim3(1, c.batch), dim3(SEL_THREADS), smem, st, c, src, scores, stride,
                          pool_len_in, ids, k, out, out_stride, expand, pool, pool_len);
    return launch_pdl(select_cluster_kernel, dim3(SEL_CLUSTER, c.batch), dim3(SEL_THREADS), smem, st, c, src, scores,
                      stride, pool_len_in, ids, k, out, out_stride, expand, pool, pool_len);
}

}  // namespace csa2

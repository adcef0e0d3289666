// Sequence-sharded decode: the merge steps between per-shard selections, and
// the log-sum-exp combine of per-shard attention results.
//
// The pages describe decode on one device (0539edu.com/news/5732216 §3: top
// 2048 blocks x 8 positions form a 16384-entry pool, rescored exactly for the
// top 512).  Split over shards, each shard's list holds its own top-k, and
// the global top-k of the union of those lists is the top-k of the whole:
// an element of the global top-k has fewer than k elements ahead of it
// anywhere, so fewer than k in its own shard.  Lists arrive in shard order
// and each is ascending by global id, so list position order is global id
// order and "ties to the lower index" carries over unchanged.
//
// shard_merge_kernel: one CTA per request.  Keys of all n_shards x k
// candidates are staged in shared memory, the exact selection of select.cuh
// picks the top k positions (ascending), and the positions whose id falls in
// this shard are compacted in order:
//   expand = 1: block ids -> this shard's pool of local entry ids;
//   expand = 0: entry ids -> this shard's local top-k ids.
// combine_kernel: one CTA per (request, head): out = sum_s w_s o_s with
// w_s = exp(lse_s - max) / sum_t exp(lse_t - max).
#include <cooperative_groups.h>

#include "common.cuh"
#include "index.cuh"
#include "select.cuh"

namespace csa2 {

namespace {

constexpr int MT = 512;                                  // merge threads
constexpr int MERGE_MAX = MAX_SHARDS * CSA2_MAX_BLOCKS;  // candidates at most (16384)
constexpr int MERGE_BITS = MERGE_MAX / 32;
constexpr size_t MERGE_SMEM =
    (size_t)(MERGE_MAX + CSA2_MAX_BLOCKS + 2 * sel::CAND + 2 * sel::RANK_MAX + MERGE_BITS) * sizeof(uint32_t);

__global__ void __launch_bounds__(MT, 1) shard_merge_kernel(CacheView c, const int32_t *entry_offset, int n_shards,
                                                             ShardLists l, int k, int expand, int32_t *out,
                                                             int32_t *pool_len)
{
    extern __shared__ uint32_t dsm[];
    uint32_t *keys = dsm;
    int32_t *picked = reinterpret_cast<int32_t *>(dsm + MERGE_MAX);     // [k] selected list positions
    __shared__ uint32_t wtot[MT / 32];
    __shared__ int s_partial_last;
    const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    grid_dependency_wait();                      // the lists come from earlier work
    allow_dependents();
    const int off = entry_offset[b];
    const bool ok = off >= 0 && (off & (CSA2_BLOCK - 1)) == 0;
    if (!ok && tid == 0) set_error(c.error, CSA2_DEV_BAD_REQUEST);
    const int n_entries = n_entries_of(c, b);
    const int n = n_shards * k;

    uint32_t kmin = 0xffffffffu, kmax = 0u;
    for (int i = tid; i < n; i += MT) {
        const int s = i / k, j = i - s * k;
        const uint32_t key = sel::ord_key(l.scores[s][(size_t)b * k + j]);
        keys[i] = key;
        kmin = min(kmin, key);
        kmax = max(kmax, key);
    }
    if (tid == 0) s_partial_last = 0;
    __syncthreads();
    sel::Bufs bf;
    bf.keys = keys;
    bf.scores = nullptr;
    bf.cand_key = dsm + MERGE_MAX + CSA2_MAX_BLOCKS;
    bf.cand_idx = bf.cand_key + sel::CAND;
    bf.all_key = bf.cand_idx + sel::CAND;
    bf.all_idx = bf.all_key + sel::RANK_MAX;
    bf.bits = bf.all_idx + sel::RANK_MAX;
    bf.bits_words = MERGE_BITS;
    sel::Out o;
    o.out = picked;                              // positions, ascending, -1 padded to k
    o.out_stride = 0;
    o.ids = nullptr;
    o.expand = 0;
    o.pool = nullptr;
    o.pool_len = nullptr;
    o.n_entries = 0;
    o.vals = nullptr;
    o.id_off = nullptr;
    o.id_shift = 0;
    sel::select_core<1, MT>(bf, b, n, n, 0, n, k, kmin, kmax, o);
    __syncthreads();

    // This shard's part, in order: thread t owns positions [t*per, t*per + per).
    const int lo_id = expand ? (off >> 3) : off;
    const int n_own = expand ? (n_entries + CSA2_BLOCK - 1) / CSA2_BLOCK : n_entries;
    const int per = (k + MT - 1) / MT;           // 4 (blocks) or 1 (entries)
    int loc[CSA2_MAX_BLOCKS / MT];
    uint32_t mine = 0;
#pragma unroll
    for (int u = 0; u < CSA2_MAX_BLOCKS / MT; ++u) {
        const int i = tid * per + u;
        int v = -1;
        if (ok && u < per && i < k) {
            const int p = picked[i];
            if (p >= 0) {
                const int s = p / k;
                const int id = l.ids[s][(size_t)b * k + (p - s * k)];
                if (id >= lo_id && id < lo_id + n_own) v = id - lo_id;
            }
        }
        loc[u] = v;
        mine += v >= 0;
    }
    // Exclusive scan of `mine` over the CTA.
    uint32_t incl = mine;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const uint32_t t = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += t;
    }
    if (lane == 31) wtot[wid] = incl;
    __syncthreads();
    uint32_t base = incl - mine, total = 0;
    for (int w = 0; w < MT / 32; ++w) {
        if (w < wid) base += wtot[w];
        total += wtot[w];
    }
    if (expand) {
        int32_t *pool = out + (size_t)b * CSA2_POOL;
#pragma unroll
        for (int u = 0; u < CSA2_MAX_BLOCKS / MT; ++u) {
            if (loc[u] < 0) continue;
            for (int t = 0; t < CSA2_BLOCK; ++t) {
                const int en = loc[u] * CSA2_BLOCK + t;
                pool[base * CSA2_BLOCK + t] = en < n_entries ? en : -1;
            }
            if ((loc[u] + 1) * CSA2_BLOCK > n_entries) s_partial_last = (loc[u] + 1) * CSA2_BLOCK - n_entries;
            ++base;
        }
        for (int i = (int)total * CSA2_BLOCK + tid; i < CSA2_POOL; i += MT) pool[i] = -1;
        __syncthreads();
        if (tid == 0) pool_len[b] = (int)total * CSA2_BLOCK - s_partial_last;
    } else {
        int32_t *tk = out + (size_t)b * CSA2_TOPK;
#pragma unroll
        for (int u = 0; u < CSA2_MAX_BLOCKS / MT; ++u)
            if (loc[u] >= 0) tk[base++] = loc[u];
        for (int i = (int)total + tid; i < CSA2_TOPK; i += MT) tk[i] = -1;
    }
}

__global__ void __launch_bounds__(128) combine_kernel(int n_parts, PartList p, int heads, void *out, int out_is_fp32)
{
    const size_t row = blockIdx.x;               // request * heads + head
    __shared__ float wgt[MAX_SHARDS];
    grid_dependency_wait();                      // the partials come from earlier work
    allow_dependents();
    if (threadIdx.x == 0) {
        float M = -INFINITY;
#pragma unroll
        for (int s = 0; s < MAX_SHARDS; ++s)
            if (s < n_parts) M = fmaxf(M, p.lse[s][row]);
        float W = 0.0f;
#pragma unroll
        for (int s = 0; s < MAX_SHARDS; ++s) {
            float e = 0.0f;
            if (s < n_parts && M != -INFINITY) {
                const float x = p.lse[s][row];
                e = x == -INFINITY ? 0.0f : expf(x - M);
            }
            wgt[s] = e;
            W += e;
        }
#pragma unroll
        for (int s = 0; s < MAX_SHARDS; ++s) wgt[s] = W > 0.0f ? wgt[s] / W : 0.0f;
    }
    __syncthreads();
    const int d4 = threadIdx.x;                  // 128 x float4 = 512 dims
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int s = 0; s < MAX_SHARDS; ++s) {
        if (s >= n_parts || wgt[s] == 0.0f) continue;
        const float4 v = reinterpret_cast<const float4 *>(p.o[s] + row * CSA2_LATENT)[d4];
        acc.x = fmaf(wgt[s], v.x, acc.x);
        acc.y = fmaf(wgt[s], v.y, acc.y);
        acc.z = fmaf(wgt[s], v.z, acc.z);
        acc.w = fmaf(wgt[s], v.w, acc.w);
    }
    (void)heads;
    const size_t o = row * CSA2_LATENT + 4 * d4;
    if (out_is_fp32) {
        *reinterpret_cast<float4 *>((float *)out + o) = acc;
    } else {
        __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y), hi = __floats2bfloat162_rn(acc.z, acc.w);
        *reinterpret_cast<uint2 *>((__nv_bfloat16 *)out + o) =
            make_uint2(*reinterpret_cast<uint32_t *>(&lo), *reinterpret_cast<uint32_t *>(&hi));
    }
}

}  // namespace

cudaError_t launch_shard_merge(const CacheView &c, const int32_t *entry_offset, int n_shards, const ShardLists &l,
                               int expand, int32_t *out, int32_t *pool_len, cudaStream_t st)
{
    static DeviceOnce once;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess)
        e = once.run(dev, [] {
            return cudaFuncSetAttribute(shard_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)MERGE_SMEM);
        });
    if (e != cudaSuccess) return e;
    const int k = expand ? CSA2_MAX_BLOCKS : CSA2_TOPK;
    LaunchScope scope(CSA2_KERNEL_COMBINE, st);
    return launch_pdl(shard_merge_kernel, dim3(c.batch), dim3(MT), MERGE_SMEM, st, c, entry_offset, n_shards, l, k,
                      expand, out, pool_len);
}

cudaError_t launch_combine(int n_parts, const PartList &p, int batch, int heads, void *out, int out_is_fp32,
                           cudaStream_t st)
{
    LaunchScope scope(CSA2_KERNEL_COMBINE, st);
    return launch_pdl(combine_kernel, dim3((unsigned)(batch * heads)), dim3(128), 0, st, n_parts, p, heads, out,
                      out_is_fp32);
}

}  // namespace csa2

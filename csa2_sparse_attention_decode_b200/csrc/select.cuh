// Exact top-k selection over order-preserving 32-bit keys held in shared
// memory, for one CTA or one thread-block cluster of NC CTAs (each CTA owns a
// contiguous range of the elements).  Score descending, ties to the lower
// index, output in ascending index order.
//
// Method (a radix select):
//   1. the cluster-wide min and max key give the leading bits every key
//      shares; no pass is spent on them;
//   2. one 8-bit histogram pass over the next bits finds the bin that holds
//      the k-th largest key and how many keys of that bin to take (krem);
//   3. the keys of that bin (the candidates, usually a few hundred) are
//      compacted.  When the cluster holds few enough of them, each candidate
//      is ranked directly (one warp per candidate) against all candidates
//      (key desc, index asc) and marked when its rank is below krem.  Otherwise further 8-bit
//      passes over the candidates (or all keys, if they overflowed) find the
//      exact threshold key T, and the first krem keys equal to T in index
//      order are taken;
//   4. the selected ids are written in ascending order: when every decision
//      is local (ranked candidates, or all elements taken) one pass compacts
//      each warp's selections in place; otherwise (ties at T resolved in
//      index order) a counting pass precedes the ordered compaction.
// Histograms, counts and candidates are exchanged over distributed shared
// memory.  Used by the top-k kernels of index.cu and by the fused pool
// rescoring kernel.
#pragma once
#include <cooperative_groups.h>

#include "common.cuh"

namespace csa2 {
namespace sel {

namespace cg = cooperative_groups;

constexpr int CAND = 2048;       // candidates a CTA keeps after the first pass
constexpr int RANK_MAX = 2048;   // cluster-wide candidates ranked directly
constexpr uint32_t RANK_WORK = 1024;   // at most this many comparisons per lane

// Order-preserving 32-bit key of an fp32 score (-0 folded onto +0).
__device__ __forceinline__ uint32_t ord_key(float x)
{
    uint32_t u = __float_as_uint(x);
    if (u == 0x80000000u) u = 0;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Shared-memory work areas the caller provides (dynamic shared memory).
struct Bufs {
    uint32_t *keys;              // [cnt] keys of this CTA's range, or nullptr: read `scores`
    const float *scores;         // global scores of this CTA's range (when keys == nullptr)
    uint32_t *cand_key, *cand_idx;    // [CAND]
    uint32_t *all_key, *all_idx;      // [RANK_MAX]
    uint32_t *bits;              // [bits_words] selection marks of candidates (local index)
    int bits_words;
};

// Where the selected ids go.
struct Out {
    int32_t *out;                // out[b*out_stride + pos] (plain / id-mapped mode)
    int out_stride;
    const int32_t *ids;          // optional map: the id of element i is ids[b*CSA2_POOL + i]
    int expand;                  // ids are block numbers: write their entries to pool
    int32_t *pool, *pool_len;
    int n_entries;               // entries of the request (expand mode)
    float *vals;                 // optional: the selected scores beside out (-inf padded)
    const int32_t *id_off;       // optional: (id_off[b] >> id_shift) is added to every written id
    int id_shift;
    // Optional: the plane row of the first element of each local run of 8
    // elements (shared memory, -1 if none).  Every selected element's latent
    // code and scale lines are then hinted into L2 for the attention's gather.
    const int32_t *run_rows = nullptr;
    const uint8_t *codes = nullptr, *scales = nullptr;
};

// Inverse of ord_key (a -0 score comes back as +0).
__device__ __forceinline__ float key_score(uint32_t key)
{
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

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

// Selects the top min(k, n) of the n elements of request b; CTA r of the NC
// holds elements [r*chunk, r*chunk + chunk) of them, this one [lo, lo + cnt)
// with lo = rank*chunk.  kmin / kmax: this thread's min / max over the keys
// it staged (any split of the range over the threads; a thread without keys
// passes kmin = 0xffffffff, kmax = 0).  NT = threads per CTA (a multiple of 32, at least 256).
// range (optional, the same in every CTA of the cluster): the cluster-wide
// {min key, max key, a lower bound of the threshold, number of disjoint key
// groups the bound is the smallest maximum of}, worked out by the caller;
// then kmin / kmax are unused and the first exchange round is skipped.
template <int NC, int NT>
__device__ __forceinline__ void select_core(const Bufs &bf, int b, int n, int chunk, int lo, int cnt, int k,
                                            uint32_t kmin, uint32_t kmax, const Out &o,
                                            const uint32_t *range = nullptr)
{
    constexpr int NW = NT / 32;
    __shared__ __align__(16) uint32_t hist[2][256];
    __shared__ __align__(16) uint32_t whist[NW][256];
    __shared__ uint32_t scratch[32];
    __shared__ uint32_t wsum[NW][4];
    __shared__ __align__(16) uint32_t s_cnt[4];
    __shared__ __align__(16) uint32_t s_mm[4];
    __shared__ __align__(16) uint32_t s_rk[NC][4];         // per-rank candidate counts, gathered by warp 0
    __shared__ uint32_t s_hsum[256];                       // cluster-wide histogram of a pass
    __shared__ uint32_t s_g[4];                            // cluster-wide reductions, formed by warp 0

    __shared__ uint32_t s_digit, s_above;
    const int rank = (NC > 1) ? (int)cg::this_cluster().block_rank() : 0;
    auto csync = [&]() {
        if constexpr (NC > 1) cluster_sync_aligned();
        else __syncthreads();
    };
    auto remote = [&](uint32_t *ptr, int r) -> uint32_t * {
        if constexpr (NC > 1) return cg::this_cluster().map_shared_rank(ptr, r);
        else return ptr;
    };
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int kk = min(k, n);
    const bool take_all = n <= k;
    const int seg = ((cnt + NW * 32 - 1) / (NW * 32)) * 32;     // elements per warp, multiple of 32
    auto key_at = [&](int e) -> uint32_t { return bf.keys ? bf.keys[e] : ord_key(bf.scores[e]); };

    uint32_t prefix = 0, pmask = 0, krem = (uint32_t)kk;
    bool ranked = false;                                    // candidates were ranked directly
    if (!take_all) {
        if (!range) {                                       // the range from one exchange round
            // Range of the keys that matter.  Every thread holding a key holds
            // one >= its own maximum, so when at least kk threads hold keys, the
            // smallest per-thread maximum lb is a lower bound of the threshold:
            // keys below it never need resolving, however far below they lie.
            const bool has = kmin <= kmax;
            uint32_t klb = has ? kmax : 0xffffffffu;
            uint32_t nthr = __popc(__ballot_sync(0xffffffffu, has));
#pragma unroll
            for (int off = 16; off; off >>= 1) {
                kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, off));
                kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, off));
                klb = min(klb, __shfl_xor_sync(0xffffffffu, klb, off));
            }
            if (lane == 0) {
                wsum[wid][0] = kmin;
                wsum[wid][1] = kmax;
                wsum[wid][2] = klb;
                wsum[wid][3] = nthr;
            }
            __syncthreads();
            if (wid == 0) {
                const bool in = lane < NW;
                const uint32_t a = __reduce_min_sync(0xffffffffu, in ? wsum[lane][0] : 0xffffffffu);
                const uint32_t z = __reduce_max_sync(0xffffffffu, in ? wsum[lane][1] : 0u);
                const uint32_t l = __reduce_min_sync(0xffffffffu, in ? wsum[lane][2] : 0xffffffffu);
                const uint32_t t = __reduce_add_sync(0xffffffffu, in ? wsum[lane][3] : 0u);
                if (lane == 0) {
                    s_mm[0] = a;
                    s_mm[1] = z;
                    s_mm[2] = l;
                    s_mm[3] = t;
                }
            }
            csync();
            if (wid == 0) {                                     // one 16-byte load per rank, reduced in the warp
                uint4 v = make_uint4(0xffffffffu, 0u, 0xffffffffu, 0u);
                if (lane < NC) v = *reinterpret_cast<const uint4 *>(remote(&s_mm[0], lane));
                const uint32_t a = __reduce_min_sync(0xffffffffu, v.x), z = __reduce_max_sync(0xffffffffu, v.y);
                const uint32_t l = __reduce_min_sync(0xffffffffu, v.z), t = __reduce_add_sync(0xffffffffu, v.w);
                if (lane == 0) {
                    s_g[0] = a;
                    s_g[1] = z;
                    s_g[2] = l;
                    s_g[3] = t;
                }
            }
            __syncthreads();
        }
        const uint32_t gmin = range ? range[0] : s_g[0], gmax = range ? range[1] : s_g[1];
        const uint32_t glb = range ? range[2] : s_g[2], gthr = range ? range[3] : s_g[3];
        const uint32_t low = gthr >= (uint32_t)kk ? glb : gmin;
        int hi = 32 - __clz(low ^ gmax);                    // bits [hi-1 .. 0] vary above `low`
        pmask = hi >= 32 ? 0u : ~((1u << hi) - 1u);
        prefix = gmax & pmask;
        bool use_cand = false;
        int n_cand = 0;
        for (int pass = 0; hi > 0; ++pass) {
            const int wdt = min(8, hi), shift = hi - wdt, buf = pass & 1;
            const uint32_t dmask = (1u << wdt) - 1u;
            for (int i = tid; i < NW * 64; i += NT) reinterpret_cast<uint4 *>(&whist[0][0])[i] = make_uint4(0, 0, 0, 0);
            __syncthreads();
            if (use_cand) {
                for (int ci = tid; ci < n_cand; ci += NT) {
                    const uint32_t key = bf.cand_key[ci];
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
                for (int w = 0; w < NW; ++w) t += whist[w][tid];
                hist[buf][tid] = t;
            }
            __syncthreads();
            csync();
            // Cluster-wide counts: thread t < 64 sums bins 4t .. 4t + 3 over
            // the CTAs with one 16-byte load each; then counts of bins >= b.
            if (tid < 64) {
                uint4 part[NC];
#pragma unroll
                for (int r = 0; r < NC; ++r) part[r] = reinterpret_cast<const uint4 *>(remote(&hist[buf][0], r))[tid];
                uint4 a = make_uint4(0, 0, 0, 0);
#pragma unroll
                for (int r = 0; r < NC; ++r) {
                    a.x += part[r].x;
                    a.y += part[r].y;
                    a.z += part[r].z;
                    a.w += part[r].w;
                }
                *reinterpret_cast<uint4 *>(&s_hsum[4 * tid]) = a;
            }
            __syncthreads();
            const uint32_t hv = tid < 256 ? s_hsum[255 - tid] : 0u;
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
                // The keys of the threshold bin: usually a few hundred.
                if (tid == 0) s_cnt[2] = 0;
                __syncthreads();
                for (int it = 0; it < seg; it += 32) {
                    const int e = wid * seg + it + lane;
                    const uint32_t key = e < cnt ? key_at(e) : 0u;
                    const bool m = e < cnt && (key & pmask) == prefix;
                    const uint32_t mb = __ballot_sync(0xffffffffu, m);
                    uint32_t base = 0;
                    if (lane == 0 && mb) base = atomicAdd(&s_cnt[2], (uint32_t)__popc(mb));
                    base = __shfl_sync(0xffffffffu, base, 0);
                    const uint32_t pos = base + __popc(mb & ((1u << lane) - 1u));
                    if (m && pos < (uint32_t)CAND) {
                        bf.cand_key[pos] = key;
                        bf.cand_idx[pos] = (uint32_t)e;
                    }
                }
                __syncthreads();
                n_cand = (int)s_cnt[2];
                use_cand = n_cand <= CAND;
                // Cluster-wide candidate count.  An overflowing CTA reports
                // CAND + 1: more than RANK_MAX in total, and the sum over the
                // cluster cannot wrap.
                static_assert(NC * (CAND + 1) < (1 << 30) && CAND + 1 > RANK_MAX, "candidate count encoding");
                if (tid == 0) s_cnt[3] = use_cand ? (uint32_t)n_cand : (uint32_t)(CAND + 1);
                csync();
                if (wid == 0) {                             // every rank's count, their sum and maximum
                    const uint32_t v = lane < NC ? *remote(&s_cnt[3], lane) : 0u;
                    const uint32_t tot = __reduce_add_sync(0xffffffffu, v), mo = __reduce_max_sync(0xffffffffu, v);
                    if (lane < NC) s_rk[lane][0] = v;
                    if (lane == 0) {
                        s_g[0] = tot;
                        s_g[1] = mo;
                    }
                }
                __syncthreads();
                const uint32_t total = s_g[0], most = s_g[1];
                // Rank directly when the comparisons per lane stay small (the
                // same decision in every CTA of the cluster).
                const uint32_t work = ((most + NW - 1) / NW) * ((total + 31) / 32);
                if (total <= (uint32_t)RANK_MAX && work <= RANK_WORK && chunk <= 32 * bf.bits_words) {
                    // Rank every local candidate against all candidates of the cluster.
                    const uint32_t *ak = bf.cand_key, *ai = nullptr;
                    if constexpr (NC > 1) {
                        // Candidate g of the cluster: CTA r's number g - off[r]
                        // (all remote loads independent of one another).
                        for (uint32_t g = tid; g < total; g += NT) {
                            int r = 0;
                            uint32_t off = 0;
                            while (r < NC - 1 && g >= off + s_rk[r][0]) off += s_rk[r++][0];
                            const uint32_t i = g - off;
                            bf.all_key[g] = remote(bf.cand_key, r)[i];
                            bf.all_idx[g] = (uint32_t)(r * chunk) + remote(bf.cand_idx, r)[i];
                        }
                        ak = bf.all_key;
                        ai = bf.all_idx;
                    }
                    for (int i = tid; i < bf.bits_words; i += NT) bf.bits[i] = 0;
                    __syncthreads();
                    // One warp per local candidate; its lanes split the comparisons.
                    for (int ci = wid; ci < n_cand; ci += NW) {
                        const uint32_t key = bf.cand_key[ci], li = bf.cand_idx[ci], gi = (uint32_t)lo + li;
                        uint32_t above = 0;
                        for (uint32_t j = lane; j < total; j += 32) {
                            const uint32_t kj = ak[j];
                            const uint32_t ij = (NC > 1) ? ai[j] : (uint32_t)lo + bf.cand_idx[j];
                            above += (kj > key) || (kj == key && ij < gi);
                        }
                        above = __reduce_add_sync(0xffffffffu, above);
                        if (lane == 0 && above < krem) atomicOr(&bf.bits[li >> 5], 1u << (li & 31));
                    }
                    __syncthreads();
                    ranked = true;
                    break;
                }
            }
        }
    }
    // Selected: every key above the threshold bin (ranked) / key T (radix),
    // plus the chosen keys of that bin (ranked: marked; radix: the first
    // krem keys equal to T in index order).
    const uint32_t T = prefix;
    const uint32_t q_take = ranked ? 0xffffffffu : krem;
    auto classify = [&](int e, bool valid, bool &g, bool &q) {
        const uint32_t key = valid ? key_at(e) : 0u;
        if (take_all) {
            g = valid;
            q = false;
        } else if (ranked) {
            const uint32_t top = key & pmask;
            g = valid && top > T;
            q = valid && top == T && ((bf.bits[e >> 5] >> (e & 31)) & 1u);
        } else {
            g = valid && key > T;
            q = valid && key == T;
        }
    };
    const uint32_t lt_mask = (1u << lane) - 1u;
    auto write_one = [&](int gi, uint32_t pos) {
        // A range that does not hold the keys (one left by a scan that
        // aborted) could choose more than kk: the slots bound the stores.
        if (pos >= (uint32_t)kk) return;
        if (o.expand) {
            static_assert(CSA2_BLOCK == 8, "a block's entries are two int4");
            int32_t *dst = o.pool + (size_t)b * CSA2_POOL + (size_t)pos * CSA2_BLOCK;
            const int e0 = gi * CSA2_BLOCK, ne = o.n_entries;
            auto id = [&](int j) { return e0 + j < ne ? e0 + j : -1; };
            if ((reinterpret_cast<uintptr_t>(o.pool) & 15) == 0) {     // two 16-byte stores per block
                reinterpret_cast<int4 *>(dst)[0] = make_int4(id(0), id(1), id(2), id(3));
                reinterpret_cast<int4 *>(dst)[1] = make_int4(id(4), id(5), id(6), id(7));
            } else {
                for (int j = 0; j < CSA2_BLOCK; ++j) dst[j] = id(j);
            }
        } else {
            const int id = o.ids ? o.ids[(size_t)b * CSA2_POOL + gi] : gi;
            o.out[(size_t)b * o.out_stride + pos] = (o.id_off && id >= 0) ? id + (o.id_off[b] >> o.id_shift) : id;
            if (o.vals) o.vals[(size_t)b * o.out_stride + pos] = key_score(key_at(gi - lo));
            if (o.run_rows) {
                const int li = gi - lo, r0 = o.run_rows[li >> 3];
                if (r0 >= 0) {
                    const size_t row = (size_t)r0 + (li & 7);
                    prefetch_l2(o.codes + row * CSA2_CODE_BYTES);
                    prefetch_l2(o.codes + row * CSA2_CODE_BYTES + 128);
                    prefetch_l2(o.scales + row * CSA2_SCALE_BYTES);
                }
            }
        }
    };
    auto pad_tail = [&]() {
        if (rank == 0) {
            if (o.expand) {
                for (int i = kk * CSA2_BLOCK + tid; i < CSA2_POOL; i += NT) o.pool[(size_t)b * CSA2_POOL + i] = -1;
                if (n == 0 && tid == 0) o.pool_len[b] = 0;
            } else {
                for (int i = kk + tid; i < k; i += NT) {
                    o.out[(size_t)b * o.out_stride + i] = -1;
                    if (o.vals) o.vals[(size_t)b * o.out_stride + i] = -INFINITY;
                }
            }
        }
    };
    if ((ranked || take_all) && bf.keys && !o.vals) {
        // Every decision is local: one pass compacts each warp's chosen
        // elements in place (over keys it has already read), then the
        // warps' and CTAs' counts place them.  (Not with scores out: the
        // compaction overwrites the keys.)
        // (The pool length, known to the thread holding the last element, is
        // stored after the cluster barriers: a global store before one would
        // hold up its release.)
        uint32_t c = 0;
        int pool_len_out = -1;
        for (int it = 0; it < seg; it += 32) {
            const int e = wid * seg + it + lane;
            const bool valid = e < cnt;
            bool g, q;
            classify(e, valid, g, q);
            const bool chosen = g || q;
            const uint32_t bal = __ballot_sync(0xffffffffu, chosen);
            if (chosen) bf.keys[wid * seg + c + __popc(bal & lt_mask)] = (uint32_t)e;
            c += __popc(bal);
            if (o.expand && valid && lo + e == n - 1)
                pool_len_out = kk * CSA2_BLOCK - (chosen ? n * CSA2_BLOCK - o.n_entries : 0);
        }
        if (lane == 0) wsum[wid][1] = c;
        __syncthreads();
        if (wid == 0) {                                     // exclusive prefix over the warps
            const uint32_t x = lane < NW ? wsum[lane][1] : 0u;
            uint32_t y = x;
#pragma unroll
            for (int o2 = 1; o2 < 32; o2 <<= 1) {
                const uint32_t t = __shfl_up_sync(0xffffffffu, y, o2);
                if (lane >= o2) y += t;
            }
            if (lane < NW) wsum[lane][0] = y - x;
            if (lane == 31) s_cnt[0] = y;
        }
        __syncthreads();
        csync();
        if (wid == 0) {                                     // the counts of the lower ranks, summed
            const uint32_t v = lane < rank ? *remote(&s_cnt[0], lane) : 0u;
            const uint32_t pre = __reduce_add_sync(0xffffffffu, v);
            if (lane == 0) s_g[0] = pre;
        }
        __syncthreads();
        const uint32_t base = wsum[wid][0] + s_g[0];
        // Nobody reads this CTA's shared memory after this point.
        if constexpr (NC > 1) asm volatile("barrier.cluster.arrive.aligned;" ::: "memory");
        const uint32_t nw = wsum[wid][1];
        for (uint32_t j = lane; j < nw; j += 32) write_one(lo + (int)bf.keys[wid * seg + j], base + j);
        if (pool_len_out >= 0) o.pool_len[b] = pool_len_out;
        pad_tail();
        if constexpr (NC > 1) asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
        return;
    }
    uint32_t ngt = 0, neq = 0;
    for (int it = 0; it < seg; it += 32) {
        const int e = wid * seg + it + lane;
        bool g, q;
        classify(e, e < cnt, g, q);
        ngt += __popc(__ballot_sync(0xffffffffu, g));
        neq += __popc(__ballot_sync(0xffffffffu, q));
    }
    if (lane == 0) {
        wsum[wid][0] = ngt;
        wsum[wid][1] = neq;
    }
    __syncthreads();
    if (wid == 0) {                                         // exclusive prefixes over the warps
        const uint32_t x0 = lane < NW ? wsum[lane][0] : 0u, x1 = lane < NW ? wsum[lane][1] : 0u;
        uint32_t y0 = x0, y1 = x1;
#pragma unroll
        for (int o2 = 1; o2 < 32; o2 <<= 1) {
            const uint32_t t0 = __shfl_up_sync(0xffffffffu, y0, o2), t1 = __shfl_up_sync(0xffffffffu, y1, o2);
            if (lane >= o2) {
                y0 += t0;
                y1 += t1;
            }
        }
        __syncwarp();
        if (lane < NW) {
            wsum[lane][0] = y0 - x0;
            wsum[lane][1] = y1 - x1;
        }
        if (lane == 31) {
            s_cnt[0] = y0;
            s_cnt[1] = y1;
        }
    }
    __syncthreads();
    csync();
    if (wid == 0) {                                         // the lower ranks' counts, summed
        uint2 v = make_uint2(0u, 0u);
        if (lane < rank) v = *reinterpret_cast<const uint2 *>(remote(&s_cnt[0], lane));
        const uint32_t p0 = __reduce_add_sync(0xffffffffu, v.x), p1 = __reduce_add_sync(0xffffffffu, v.y);
        if (lane == 0) {
            s_g[0] = p0;
            s_g[1] = p1;
        }
    }
    __syncthreads();
    uint32_t gt_b = s_g[0] + wsum[wid][0], eq_b = s_g[1] + wsum[wid][1];
    // Nobody reads another CTA's shared memory after this point: arrive now,
    // wait only after the output stores (a release after them would wait
    // for them).
    if constexpr (NC > 1) asm volatile("barrier.cluster.arrive.aligned;" ::: "memory");
    for (int it = 0; it < seg; it += 32) {
        const int e = wid * seg + it + lane;
        const bool valid = e < cnt;
        bool g, q;
        classify(e, valid, g, q);
        const uint32_t bg = __ballot_sync(0xffffffffu, g), bq = __ballot_sync(0xffffffffu, q);
        const uint32_t my_gt = gt_b + __popc(bg & lt_mask), my_eq = eq_b + __popc(bq & lt_mask);
        const int gi = lo + e;
        const bool chosen = g || (q && my_eq < q_take);
        if (chosen) write_one(gi, my_gt + min(my_eq, q_take));
        if (o.expand && valid && gi == n - 1)
            o.pool_len[b] = kk * CSA2_BLOCK - (chosen ? n * CSA2_BLOCK - o.n_entries : 0);
        gt_b += __popc(bg);
        eq_b += __popc(bq);
    }
    pad_tail();
    // No CTA may leave while another still reads its shared memory.
    if constexpr (NC > 1) asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
    else __syncthreads();
}

}  // namespace sel
}  // namespace csa2

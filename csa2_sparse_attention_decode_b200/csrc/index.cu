// Indexer kernels: score = sum_h w_h * ReLU(q_h . k) over FP8 keys or block
// summaries, and an exact radix top-k (score descending, ties to the lower
// index) whose output is the selected ids in ascending order.
//
// Sources: 0539edu.com/news/5732216 §3 (indexer 32 heads x 128, top_k 512,
// hierarchical 2048 blocks x 8 positions -> 16384 candidates; Full builds the
// pool, Reindex searches inside it).
#include "common.cuh"
#include "index.cuh"

namespace csa2 {

// ------------------------------------------------------------------ scoring
__device__ __forceinline__ int rows_of(const CacheView &c, int src, int b, const int32_t *pool_len)
{
    int n = n_entries_of(c, b);
    if (src == ROWS_KEYS) return n;
    if (src == ROWS_SUMMARIES) return (n + CSA2_BLOCK - 1) / CSA2_BLOCK;
    return max(0, min(pool_len[b], CSA2_POOL));
}

// Address of row r (nullptr if invalid; error word set).
__device__ __forceinline__ const uint8_t *row_addr(const CacheView &c, int src, int b, int r, int n_entries,
                                                   const int32_t *pool)
{
    if (src == ROWS_SUMMARIES) {
        uint8_t *pg = entry_page(c, b, r * CSA2_BLOCK);
        return pg ? pg + CSA2_PAGE_SUMM_OFF + (r & 7) * CSA2_KEY_DIM : nullptr;
    }
    int e = r;
    if (src == ROWS_POOL) {
        e = pool[(size_t)b * CSA2_POOL + r];
        if (e < 0 || e >= n_entries) {
            set_error(c.error, CSA2_DEV_BAD_INDEX);
            return nullptr;
        }
    }
    uint8_t *pg = entry_page(c, b, e);
    return pg ? pg + CSA2_PAGE_KEYS_OFF + (e & (CSA2_PAGE_ENTRIES - 1)) * CSA2_KEY_DIM : nullptr;
}

constexpr int SC_ROWS = 32;
constexpr int SC_THREADS = 128;
constexpr int SC_KSTRIDE = CSA2_KEY_DIM + 4;

// CTA: 32 rows of one request; thread tid: rows 2*(tid/8), +1 and heads
// 4*(tid%8) .. +3.
__global__ void __launch_bounds__(SC_THREADS) score_rows_kernel(CacheView c, int src, const uint16_t *q_idx,
                                                         const float *w, const int32_t *pool,
                                                         const int32_t *pool_len, float *scores,
                                                         int64_t score_stride)
{
    __shared__ __align__(16) float q_s[CSA2_KEY_DIM][CSA2_IDX_HEADS];
    __shared__ __align__(16) float k_s[SC_ROWS][SC_KSTRIDE];
    __shared__ float w_s[CSA2_IDX_HEADS];
    int b = blockIdx.y;
    int n_rows = rows_of(c, src, b, pool_len);
    int r0 = blockIdx.x * SC_ROWS;
    if (r0 >= n_rows) return;
    int n_entries = n_entries_of(c, b);
    int tid = threadIdx.x;
    const uint16_t *qb = q_idx + (size_t)b * CSA2_IDX_HEADS * CSA2_KEY_DIM;
    for (int i = tid; i < CSA2_IDX_HEADS * CSA2_KEY_DIM; i += SC_THREADS) {
        int h = i / CSA2_KEY_DIM, d = i % CSA2_KEY_DIM;
        q_s[d][h] = __uint_as_float((uint32_t)qb[i] << 16);
    }
    if (tid < CSA2_IDX_HEADS) w_s[tid] = w[(size_t)b * CSA2_IDX_HEADS + tid];
    // Stage 32 rows x 128 FP8 -> fp32 (two 16-byte chunks per thread).
    for (int ch = tid; ch < SC_ROWS * 8; ch += SC_THREADS) {
        int r = ch >> 3, part = ch & 7;
        float4 *dst = reinterpret_cast<float4 *>(&k_s[r][16 * part]);
        const uint8_t *src_row = (r0 + r < n_rows) ? row_addr(c, src, b, r0 + r, n_entries, pool) : nullptr;
        if (src_row) {
            uint4 v = *reinterpret_cast<const uint4 *>(src_row + 16 * part);
            uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int j = 0; j < 4; ++j)
                dst[j] = make_float4(e4m3_to_f32(wv[j] & 0xff), e4m3_to_f32((wv[j] >> 8) & 0xff),
                                     e4m3_to_f32((wv[j] >> 16) & 0xff), e4m3_to_f32(wv[j] >> 24));
        } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) dst[j] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    __syncthreads();
    int rp = tid >> 3, hg = tid & 7;
    float acc[2][4] = {};
    const float *ka = k_s[2 * rp], *kb = k_s[2 * rp + 1];
#pragma unroll 4
    for (int d = 0; d < CSA2_KEY_DIM; d += 4) {
        float4 a = *reinterpret_cast<const float4 *>(ka + d);
        float4 bb = *reinterpret_cast<const float4 *>(kb + d);
        float av[4] = {a.x, a.y, a.z, a.w}, bv[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
        for (int dd = 0; dd < 4; ++dd) {
            float4 q = *reinterpret_cast<const float4 *>(&q_s[d + dd][4 * hg]);
            acc[0][0] = fmaf(av[dd], q.x, acc[0][0]);
            acc[0][1] = fmaf(av[dd], q.y, acc[0][1]);
            acc[0][2] = fmaf(av[dd], q.z, acc[0][2]);
            acc[0][3] = fmaf(av[dd], q.w, acc[0][3]);
            acc[1][0] = fmaf(bv[dd], q.x, acc[1][0]);
            acc[1][1] = fmaf(bv[dd], q.y, acc[1][1]);
            acc[1][2] = fmaf(bv[dd], q.z, acc[1][2]);
            acc[1][3] = fmaf(bv[dd], q.w, acc[1][3]);
        }
    }
    float s[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        s[r] = 0.0f;
#pragma unroll
        for (int h = 0; h < 4; ++h) s[r] = fmaf(w_s[4 * hg + h], fmaxf(acc[r][h], 0.0f), s[r]);
#pragma unroll
        for (int o = 1; o < 8; o <<= 1) s[r] += __shfl_xor_sync(0xffffffffu, s[r], o);
    }
    if (hg == 0) {
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            int row = r0 + 2 * rp + r;
            if (row < n_rows) scores[(size_t)b * score_stride + row] = s[r];
        }
    }
}

// ------------------------------------------------------------------ top-k
// Order-preserving 32-bit key of an fp32 score (-0 folded onto +0).
__device__ __forceinline__ uint32_t ord_key(float x)
{
    uint32_t u = __float_as_uint(x);
    if (u == 0x80000000u) u = 0;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

constexpr int SEL_THREADS = 1024;

// Inclusive scan of v over the 1024 threads; returns the inclusive prefix and
// writes the block total into *total.  Uses scratch[32].
__device__ __forceinline__ uint32_t block_scan_incl(uint32_t v, uint32_t *scratch, uint32_t *total)
{
    int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        uint32_t t = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += t;
    }
    if (lane == 31) scratch[wid] = v;
    __syncthreads();
    if (wid == 0) {
        uint32_t t = scratch[lane];
        uint32_t x = t;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        scratch[lane] = x - t;       // exclusive prefix of warp totals
        if (lane == 31) scratch[32] = x;
    }
    __syncthreads();
    uint32_t r = v + scratch[wid];
    *total = scratch[32];
    __syncthreads();
    return r;
}

// One CTA per request.  Selects the top min(k, n) of scores[b][0..n) and
// writes the selected ids ascending to out[b][0..k) (-1 padded).  The id of
// element i is i, or ids[b][i] when ids != nullptr.  With expand != 0 the
// selected ids are block numbers: the pool of their entries (ascending, ids
// < n_entries) is written to pool[b][0..16384) and its length to pool_len[b].
__global__ void __launch_bounds__(SEL_THREADS) select_topk_kernel(CacheView c, int src, const float *scores,
                                                                  int64_t score_stride, const int32_t *pool_len_in,
                                                                  const int32_t *ids, int k, int32_t *out,
                                                                  int out_stride, int expand, int32_t *pool,
                                                                  int32_t *pool_len)
{
    __shared__ uint32_t hist[256];
    __shared__ uint32_t scratch[33];
    __shared__ uint32_t s_digit, s_above;
    __shared__ int32_t sel[CSA2_MAX_BLOCKS];
    int b = blockIdx.x;
    int tid = threadIdx.x;
    int n_entries = n_entries_of(c, b);
    int n = (src == ROWS_KEYS) ? n_entries
          : (src == ROWS_SUMMARIES) ? (n_entries + CSA2_BLOCK - 1) / CSA2_BLOCK
                              : max(0, min(pool_len_in[b], CSA2_POOL));
    const float *s = scores + (size_t)b * score_stride;
    int kk = min(k, n);
    bool take_all = n <= k;
    uint32_t prefix = 0, pmask = 0, krem = (uint32_t)kk;
    if (!take_all) {
        for (int shift = 24; shift >= 0; shift -= 8) {
            if (tid < 256) hist[tid] = 0;
            __syncthreads();
            // Uniform trip count so whole warps stay converged for the match.
            for (int base = 0; base < n; base += SEL_THREADS) {
                int i = base + tid;
                uint32_t key = i < n ? ord_key(s[i]) : 0u;
                bool match = (i < n) && (key & pmask) == prefix;
                uint32_t dig = (key >> shift) & 255u;
                uint32_t mm = __match_any_sync(0xffffffffu, match ? dig : 0x100u + (tid & 31));
                if (match && (__ffs(mm) - 1) == (tid & 31)) atomicAdd(&hist[dig], (uint32_t)__popc(mm));
            }
            __syncthreads();
            // Suffix counts: thread t holds bin 255 - t.
            uint32_t hv = tid < 256 ? hist[255 - tid] : 0u;
            uint32_t tot;
            uint32_t incl = block_scan_incl(hv, scratch, &tot);   // = count of bins >= 255 - t
            if (tid < 256) {
                uint32_t above = incl - hv;
                if (incl >= krem && above < krem) {
                    s_digit = 255u - tid;
                    s_above = above;
                }
            }
            __syncthreads();
            prefix |= s_digit << shift;
            pmask |= 255u << shift;
            krem -= s_above;
            __syncthreads();
        }
    }
    // Ordered compaction: selected = key > T, or key == T among the first krem.
    uint32_t T = prefix;
    uint32_t base_gt = 0, base_eq = 0;
    for (int t0 = 0; t0 < n; t0 += SEL_THREADS * 4) {
        int i0 = t0 + 4 * tid;
        uint32_t gtf = 0, eqf = 0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            int i = i0 + j;
            if (i < n) {
                uint32_t key = ord_key(s[i]);
                if (take_all || key > T) gtf |= 1u << j;
                else if (key == T) eqf |= 1u << j;
            }
        }
        uint32_t packed = (uint32_t)__popc(gtf) | ((uint32_t)__popc(eqf) << 16);
        uint32_t tot;
        uint32_t incl = block_scan_incl(packed, scratch, &tot);
        uint32_t ex = incl - packed;
        uint32_t gt_b = base_gt + (ex & 0xffffu), eq_b = base_eq + (ex >> 16);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            bool g = (gtf >> j) & 1u, e = (eqf >> j) & 1u;
            if (g || (e && eq_b < krem)) {
                uint32_t pos = gt_b + min(eq_b, krem);
                int i = i0 + j;
                int id = ids ? ids[(size_t)b * CSA2_POOL + i] : i;
                if (expand) sel[pos] = id;
                else out[(size_t)b * out_stride + pos] = id;
            }
            gt_b += g;
            eq_b += e;
        }
        base_gt += tot & 0xffffu;
        base_eq += tot >> 16;
    }
    __syncthreads();
    if (!expand) {
        for (int i = kk + tid; i < k; i += SEL_THREADS) out[(size_t)b * out_stride + i] = -1;
        return;
    }
    // Pool of the selected blocks: entries 8*blk + j (< n_entries); only the
    // highest block can be partial, and it comes last in ascending order.
    for (int i = tid; i < CSA2_POOL; i += SEL_THREADS) {
        int bi = i >> 3, j = i & 7;
        int e = -1;
        if (bi < kk) {
            e = sel[bi] * CSA2_BLOCK + j;
            if (e >= n_entries) e = -1;
        }
        pool[(size_t)b * CSA2_POOL + i] = e;
    }
    if (tid == 0) {
        int len = kk * CSA2_BLOCK;
        if (kk > 0) len -= max(0, (sel[kk - 1] + 1) * CSA2_BLOCK - n_entries);
        pool_len[b] = len;
    }
}

// ------------------------------------------------------------------ launchers
cudaError_t launch_score(const CacheView &c, int src, const uint16_t *q_idx, const float *w, const int32_t *pool,
                         const int32_t *pool_len, float *scores, int64_t stride, int max_rows, cudaStream_t st)
{
    if (max_rows <= 0) return cudaSuccess;
    dim3 grid((max_rows + SC_ROWS - 1) / SC_ROWS, c.batch);
    int kid = src == ROWS_KEYS ? CSA2_KERNEL_FLAT_SCORE : src == ROWS_SUMMARIES ? CSA2_KERNEL_BLOCK_SCORE
                                                                                : CSA2_KERNEL_POOL_SCORE;
    LaunchScope scope(kid, st);
    score_rows_kernel<<<grid, SC_THREADS, 0, st>>>(c, src, q_idx, w, pool, pool_len, scores, stride);
    return cudaGetLastError();
}

cudaError_t launch_select(const CacheView &c, int src, const float *scores, int64_t stride, const int32_t *pool_len_in,
                          const int32_t *ids, int k, int32_t *out, int out_stride, int expand, int32_t *pool,
                          int32_t *pool_len, cudaStream_t st)
{
    LaunchScope scope(CSA2_KERNEL_SELECT, st);
    select_topk_kernel<<<c.batch, SEL_THREADS, 0, st>>>(c, src, scores, stride, pool_len_in, ids, k, out, out_stride,
                                                        expand, pool, pool_len);
    return cudaGetLastError();
}

}  // namespace csa2

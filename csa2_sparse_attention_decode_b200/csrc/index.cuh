// Launch entry points of the indexer kernels (host side).
#pragma once
#include <cudaTypedefs.h>

#include "common.cuh"

namespace csa2 {
// Host-side validation of a cache descriptor shared by every entry point:
// non-null fields, positive sizes, at most 2^30 entries per request, and
// the pool / SWA ring 256-byte and pending 16-byte aligned.
csa2_status check_cache(const csa2_cache *c);

// What a scan or a selection runs over: every key of the requests, their
// block summaries, or (selection only) a given score matrix with row lengths.
enum RowSource { ROWS_KEYS = 0, ROWS_SUMMARIES = 1, ROWS_GIVEN = 2 };

// 2-D TMA view of a 128-byte-row plane of the pool (keys or summaries):
// `rows` rows, boxes of box_rows rows, 128-byte swizzled.  Host side.
bool make_plane_map(CUtensorMap *m, void *base, long long rows, int box_rows);

// Row scores of the block summaries (src ROWS_SUMMARIES) or of the keys
// (ROWS_KEYS) of every request into scores[b * stride + row].  With range,
// also folds the keys into range[b * RANGE_SLOTS + s] = {largest key,
// smallest key, smallest maximum of a group of range_group(n) rows, tag}
// (order-preserving keys, atomic max / min, each warp into one of the
// request's slots; the words must hold the empty range {0, ~0, ~0, tag} or
// a wider one beforehand, as the selection leaves them).
constexpr int RANGE_SLOTS = 32;
constexpr uint32_t RANGE_TAG = 0x43534132u;     // the last word of a slot a selection reset
// Rows per group for the lower bound of a request of n rows: the largest of
// 32, 16 and 8 that still gives at least CSA2_MAX_BLOCKS groups (each group
// holds a key at least as large as the bound, so with that many groups the
// bound is at most the top-2048 threshold); 8 when none does.
__host__ __device__ __forceinline__ int range_group(int n)
{
    return n >= 32 * CSA2_MAX_BLOCKS ? 32 : n >= 16 * CSA2_MAX_BLOCKS ? 16 : 8;
}
cudaError_t launch_score(const CacheView &c, int src, const uint16_t *q_idx, const float *w, float *scores,
                         int64_t stride, cudaStream_t st, uint4 *range = nullptr);
// Top-k selection of the rows' scores.  With range (the scan's, above), the
// selection takes its bounds from there when every slot of the request
// carries the tag, and then resets the slots to the tagged empty range for
// the next scan.
cudaError_t launch_select(const CacheView &c, int src, const float *scores, int64_t stride, const int32_t *pool_len_in,
                          const int32_t *ids, int k, int32_t *out, int out_stride, int expand, int32_t *pool,
                          int32_t *pool_len, int max_n, cudaStream_t st, float *vals = nullptr,
                          const int32_t *id_off = nullptr, int id_shift = 0, uint4 *range = nullptr);
// Exact rescoring of the pool fused with its top-512 selection (one cluster
// per request); writes the selected pool ids, ascending, -1 padded, and
// optionally their scores (-inf padded) with id_off[b] added to every id.
cudaError_t launch_pool_select(const CacheView &c, const uint16_t *q_idx, const float *w, const int32_t *pool,
                               const int32_t *pool_len, int32_t *topk, cudaStream_t st, float *topk_scores = nullptr,
                               const int32_t *id_off = nullptr);
cudaError_t launch_prefill(const CacheView &c, int req, int m, int tok_begin, int n_tok, int n_tok_final,
                           const float *lat, const float *key, const float *gate, cudaStream_t st);
cudaError_t launch_append(const CacheView &c, const float *lat, const float *key, const float *gate,
                          const int32_t *n_new, cudaStream_t st);

// Attention with the split merge inside a cluster (distributed shared memory):
// the csa2_attend path.  Needs no scratch.  With lse != nullptr it also
// writes ln sum_j exp(scale * q.v_j) per (request, head) ([batch][heads]).
cudaError_t launch_attend(const CacheView &c, int heads, const uint16_t *q, const int32_t *topk, float scale,
                          void *out, int out_is_fp32, uint32_t flags, cudaStream_t st, float *lse = nullptr);
// Internal attention flag (beside CSA2_ATTEND_INPUTS_SETTLED): no window keys.
constexpr uint32_t ATT_NO_WINDOW = 1u << 8;
// Sequence-sharded decode (shard.cu): global top-k over the shards' lists,
// keeping this shard's part.  expand = 1: block lists -> pool; 0: entry
// lists -> topk.
constexpr int MAX_SHARDS = 8;
struct ShardLists {
    const int32_t *ids[MAX_SHARDS];
    const float *scores[MAX_SHARDS];
};
cudaError_t launch_shard_merge(const CacheView &c, const int32_t *entry_offset, int n_shards, const ShardLists &l,
                               int expand, int32_t *out, int32_t *pool_len, cudaStream_t st);
struct PartList {
    const float *o[MAX_SHARDS];
    const float *lse[MAX_SHARDS];
};
cudaError_t launch_combine(int n_parts, const PartList &p, int batch, int heads, void *out, int out_is_fp32,
                           cudaStream_t st);
// Attention with the scaled split partials exchanged through global scratch
// `part_o` ([batch][5][heads][512] fp32): the csa2_attend_noalloc path.
cudaError_t launch_attend_umma(const CacheView &c, int heads, const uint16_t *q, const int32_t *topk, float scale,
                               void *out, int out_is_fp32, uint32_t flags, float *part_o, cudaStream_t st);

constexpr int ATT_KEYS_PER_SPLIT = 128;
constexpr int ATT_SPLITS = (CSA2_TOPK + CSA2_SWA) / ATT_KEYS_PER_SPLIT;   // 5: four top-k tiles + the window
}  // namespace csa2

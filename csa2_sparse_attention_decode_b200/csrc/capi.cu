// extern "C" entry points of libcsa2: host-side validation, workspace layout
// and kernel dispatch.  See include/csa2.h for the contract of each call.
#include <atomic>
#include <cstdio>

#include "common.cuh"
#include "index.cuh"

using namespace csa2;

namespace {

std::atomic<unsigned long long> g_launches{0};
cudaEvent_t g_prof[CSA2_KERNEL_COUNT][2] = {};

}  // namespace

void csa2::note_launch(int kernel, cudaStream_t st, bool before)
{
    if (!before) g_launches.fetch_add(1, std::memory_order_relaxed);
    if (kernel < 0 || kernel >= CSA2_KERNEL_COUNT) return;
    cudaEvent_t ev = g_prof[kernel][before ? 0 : 1];
    if (!ev) return;
    // Under stream capture a plain record only marks a dependency; an
    // external record becomes an event node that fires on every replay.
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    cudaStreamIsCapturing(st, &cs);
    if (cs == cudaStreamCaptureStatusActive)
        cudaEventRecordWithFlags(ev, st, cudaEventRecordExternal);
    else
        cudaEventRecord(ev, st);
}

csa2_status csa2::check_cache(const csa2_cache *c)
{
    auto al = [](const void *p, size_t a) { return ((uintptr_t)p % a) == 0; };
    if (!c || !c->pool || !c->page_table || !c->n_tokens || !c->m || !c->swa || !c->pending || !c->error)
        return CSA2_ERR_INVALID_ARG;
    if (c->batch <= 0 || c->n_pages <= 0 || c->max_pages <= 0) return CSA2_ERR_INVALID_ARG;
    if ((int64_t)c->max_pages * CSA2_PAGE_ENTRIES > (int64_t)1 << 30) return CSA2_ERR_INVALID_ARG;
    if (!al(c->pool, 256) || !al(c->swa, 256) || !al(c->pending, 16)) return CSA2_ERR_INVALID_ARG;
    return CSA2_OK;
}

namespace {

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Workspace layout (all regions 256-byte aligned):
//   scores   [batch][row_stride] f32  row scores of the block or flat scan
//   blocks   [batch][2048]       i32  selected blocks (FULL)
// The pool's scores stay in shared memory (pool_select.cu) and attention
// merges its splits inside a cluster (attend.cu): neither needs more.
struct Workspace {
    float *scores;
    int32_t *blocks;
    uint4 *range;           // per request: the block scan's key range, folded by its CTAs
    int64_t row_stride;
    size_t bytes;
};

Workspace layout(void *base, int32_t batch, int32_t max_entries)
{
    Workspace w{};
    w.row_stride = ((int64_t)max_entries + 3) & ~(int64_t)3;
    size_t off = 0;
    auto take = [&](size_t n) { size_t o = off; off = align256(off + n); return (char *)base + o; };
    w.scores = (float *)take(sizeof(float) * (size_t)batch * (size_t)w.row_stride);
    w.blocks = (int32_t *)take(sizeof(int32_t) * (size_t)batch * CSA2_MAX_BLOCKS);
    w.range = (uint4 *)take(sizeof(uint4) * RANGE_SLOTS * (size_t)batch);
    w.bytes = off;
    return w;
}

bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

csa2_status from_cuda(cudaError_t e) { return e == cudaSuccess ? CSA2_OK : CSA2_ERR_CUDA; }

}  // namespace

extern "C" {

size_t csa2_page_bytes(void) { return CSA2_PAGE_BYTES; }
size_t csa2_swa_bytes(void) { return CSA2_SWA_BYTES; }

size_t csa2_workspace_bytes(int32_t batch, int32_t max_entries)
{
    if (batch <= 0 || max_entries < 0) return 0;
    return layout(nullptr, batch, max_entries).bytes;
}

csa2_status csa2_prefill(const csa2_cache *cache, int32_t req, int32_t m_host, int32_t tok_begin, int32_t n_tok,
                         int32_t n_tok_final, const float *lat, const float *key, const float *gate,
                         csa2_stream_t stream)
{
    CSA2_TRACE("csa2_prefill");
    csa2_status st = check_cache(cache);
    if (st != CSA2_OK) return st;
    if (req < 0 || req >= cache->batch || (m_host != 1 && m_host != 2)) return CSA2_ERR_INVALID_ARG;
    if (tok_begin < 0 || n_tok < 0 || tok_begin % m_host != 0 || tok_begin + n_tok > n_tok_final)
        return CSA2_ERR_INVALID_ARG;
    if ((int64_t)(tok_begin + n_tok) / m_host > (int64_t)cache->max_pages * CSA2_PAGE_ENTRIES)
        return CSA2_ERR_INVALID_ARG;
    if (n_tok > 0 && (!lat || !key || !gate)) return CSA2_ERR_INVALID_ARG;
    if (!aligned(lat, 16) || !aligned(key, 16)) return CSA2_ERR_INVALID_ARG;
    return from_cuda(launch_prefill(make_view(cache), req, m_host, tok_begin, n_tok, n_tok_final, lat, key, gate,
                                    (cudaStream_t)stream));
}

csa2_status csa2_append(const csa2_cache *cache, const float *lat, const float *key, const float *gate,
                        const int32_t *n_new, csa2_stream_t stream)
{
    CSA2_TRACE("csa2_append");
    csa2_status st = check_cache(cache);
    if (st != CSA2_OK) return st;
    if (!lat || !key || !gate || !n_new) return CSA2_ERR_INVALID_ARG;
    if (!aligned(lat, 16) || !aligned(key, 16)) return CSA2_ERR_INVALID_ARG;
    return from_cuda(launch_append(make_view(cache), lat, key, gate, n_new, (cudaStream_t)stream));
}

csa2_status csa2_index(const csa2_cache *cache, csa2_index_mode mode, const uint16_t *q_idx, const float *w,
                       int32_t *pool, int32_t *pool_len, int32_t *topk, void *ws, size_t ws_bytes,
                       csa2_stream_t stream)
{
    CSA2_TRACE("csa2_index");
    csa2_status st = check_cache(cache);
    if (st != CSA2_OK) return st;
    if (!q_idx || !w || !topk || !ws || !aligned(ws, 256) || !aligned(q_idx, 16)) return CSA2_ERR_INVALID_ARG;
    if (mode != CSA2_INDEX_FLAT && mode != CSA2_INDEX_FULL && mode != CSA2_INDEX_REINDEX) return CSA2_ERR_INVALID_ARG;
    if (mode != CSA2_INDEX_FLAT && (!pool || !pool_len)) return CSA2_ERR_INVALID_ARG;
    const int max_entries = cache->max_pages * CSA2_PAGE_ENTRIES;
    Workspace W = layout(ws, cache->batch, max_entries);
    if (ws_bytes < W.bytes) return CSA2_ERR_INVALID_ARG;
    CacheView c = make_view(cache);
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e = cudaSuccess;
    if (mode == CSA2_INDEX_FLAT) {
        e = launch_score(c, ROWS_KEYS, q_idx, w, W.scores, W.row_stride, s);
        if (e == cudaSuccess)
            e = launch_select(c, ROWS_KEYS, W.scores, W.row_stride, nullptr, nullptr, CSA2_TOPK, topk, CSA2_TOPK,
                              0, nullptr, nullptr, max_entries, s);
        return from_cuda(e);
    }
    if (mode == CSA2_INDEX_FULL) {
        const int max_blocks = (max_entries + CSA2_BLOCK - 1) / CSA2_BLOCK;
        e = launch_score(c, ROWS_SUMMARIES, q_idx, w, W.scores, W.row_stride, s, W.range);
        if (e == cudaSuccess)
            e = launch_select(c, ROWS_SUMMARIES, W.scores, W.row_stride, nullptr, nullptr, CSA2_MAX_BLOCKS,
                              W.blocks, CSA2_MAX_BLOCKS, 1, pool, pool_len, max_blocks, s, nullptr, nullptr, 0,
                              W.range);
        if (e != cudaSuccess) return from_cuda(e);
    }
    return from_cuda(launch_pool_select(c, q_idx, w, pool, pool_len, topk, s));
}

csa2_status csa2_topk(const float *scores, int64_t stride, const int32_t *n, int32_t batch, int32_t k,
                      int32_t *out, csa2_stream_t stream)
{
    CSA2_TRACE("csa2_topk");
    if (!scores || !n || !out || batch <= 0 || batch > 65535 || k < 1 || k > CSA2_MAX_BLOCKS || stride < 1)
        return CSA2_ERR_INVALID_ARG;
    if (stride > ((int64_t)1 << 31) / batch) return CSA2_ERR_INVALID_ARG;
    CacheView c = {};
    c.batch = batch;
    const int max_n = stride > (int64_t)(1 << 30) ? (1 << 30) : (int)stride;
    return from_cuda(launch_select(c, ROWS_GIVEN, scores, stride, n, nullptr, k, out, k, 0, nullptr, nullptr, max_n,
                                   (cudaStream_t)stream));
}

csa2_status csa2_attend(const csa2_cache *cache, int32_t heads, const uint16_t *q, const int32_t *topk, float scale,
                        void *out, int32_t out_is_fp32, uint32_t flags, void *ws, size_t ws_bytes,
                        csa2_stream_t stream)
{
    CSA2_TRACE("csa2_attend");
    csa2_status st = check_cache(cache);
    if (st != CSA2_OK) return st;
    if (heads <= 0 || heads > 128 || !q || !topk || !out || !ws || !aligned(ws, 256)) return CSA2_ERR_INVALID_ARG;
    if (!aligned(out, 16) || !aligned(q, 16)) return CSA2_ERR_INVALID_ARG;
    const int max_entries = cache->max_pages * CSA2_PAGE_ENTRIES;
    Workspace W = layout(ws, cache->batch, max_entries);
    if (ws_bytes < W.bytes) return CSA2_ERR_INVALID_ARG;
    if (flags & ~CSA2_ATTEND_INPUTS_SETTLED) return CSA2_ERR_INVALID_ARG;
    return from_cuda(launch_attend(make_view(cache), heads, q, topk, scale, out, out_is_fp32, flags,
                                   (cudaStream_t)stream));
}

// ------------------------------------------------------------ sequence shards
csa2_status csa2_shard_blocks(const csa2_cache *shard, const int32_t *entry_offset, const uint16_t *q_idx,
                              const float *w, int32_t *block_ids, float *block_scores, void *ws, size_t ws_bytes,
                              csa2_stream_t stream)
{
    CSA2_TRACE("csa2_shard_blocks");
    csa2_status st = check_cache(shard);
    if (st != CSA2_OK) return st;
    if (!entry_offset || !q_idx || !w || !block_ids || !block_scores || !ws || !aligned(ws, 256) ||
        !aligned(q_idx, 16))
        return CSA2_ERR_INVALID_ARG;
    const int max_entries = shard->max_pages * CSA2_PAGE_ENTRIES;
    Workspace W = layout(ws, shard->batch, max_entries);
    if (ws_bytes < W.bytes) return CSA2_ERR_INVALID_ARG;
    CacheView c = make_view(shard);
    cudaStream_t s = (cudaStream_t)stream;
    const int max_blocks = (max_entries + CSA2_BLOCK - 1) / CSA2_BLOCK;
    cudaError_t e = launch_score(c, ROWS_SUMMARIES, q_idx, w, W.scores, W.row_stride, s, W.range);
    if (e == cudaSuccess)
        e = launch_select(c, ROWS_SUMMARIES, W.scores, W.row_stride, nullptr, nullptr, CSA2_MAX_BLOCKS, block_ids,
                          CSA2_MAX_BLOCKS, 0, nullptr, nullptr, max_blocks, s, block_scores, entry_offset, 3,
                          W.range);
    return from_cuda(e);
}

static_assert(MAX_SHARDS == CSA2_MAX_SHARDS, "one shard limit for the ABI and the kernels");

namespace {
csa2_status shard_lists(int32_t n_shards, const int32_t *const *ids, const float *const *scores, ShardLists &l)
{
    if (n_shards < 1 || n_shards > CSA2_MAX_SHARDS || !ids || !scores) return CSA2_ERR_INVALID_ARG;
    l = ShardLists{};
    for (int i = 0; i < n_shards; ++i) {
        if (!ids[i] || !scores[i]) return CSA2_ERR_INVALID_ARG;
        l.ids[i] = ids[i];
        l.scores[i] = scores[i];
    }
    return CSA2_OK;
}
}  // namespace

csa2_status csa2_shard_pool(const csa2_cache *shard, const int32_t *entry_offset, int32_t n_shards,
                            const int32_t *const *cand_ids, const float *const *cand_scores, int32_t *pool,
                            int32_t *pool_len, csa2_stream_t stream)
{
    CSA2_TRACE("csa2_shard_pool");
    csa2_status st = check_cache(shard);
    if (st != CSA2_OK) return st;
    ShardLists l;
    if ((st = shard_lists(n_shards, cand_ids, cand_scores, l)) != CSA2_OK) return st;
    if (!entry_offset || !pool || !pool_len) return CSA2_ERR_INVALID_ARG;
    return from_cuda(launch_shard_merge(make_view(shard), entry_offset, n_shards, l, 1, pool, pool_len,
                                        (cudaStream_t)stream));
}

csa2_status csa2_shard_rescore(const csa2_cache *shard, const int32_t *entry_offset, const uint16_t *q_idx,
                               const float *w, const int32_t *pool, const int32_t *pool_len, int32_t *ids,
                               float *scores, csa2_stream_t stream)
{
    CSA2_TRACE("csa2_shard_rescore");
    csa2_status st = check_cache(shard);
    if (st != CSA2_OK) return st;
    if (!entry_offset || !q_idx || !w || !pool || !pool_len || !ids || !scores || !aligned(q_idx, 16))
        return CSA2_ERR_INVALID_ARG;
    return from_cuda(launch_pool_select(make_view(shard), q_idx, w, pool, pool_len, ids, (cudaStream_t)stream,
                                        scores, entry_offset));
}

csa2_status csa2_shard_topk(const csa2_cache *shard, const int32_t *entry_offset, int32_t n_shards,
                            const int32_t *const *cand_ids, const float *const *cand_scores, int32_t *topk,
                            csa2_stream_t stream)
{
    CSA2_TRACE("csa2_shard_topk");
    csa2_status st = check_cache(shard);
    if (st != CSA2_OK) return st;
    ShardLists l;
    if ((st = shard_lists(n_shards, cand_ids, cand_scores, l)) != CSA2_OK) return st;
    if (!entry_offset || !topk) return CSA2_ERR_INVALID_ARG;
    return from_cuda(launch_shard_merge(make_view(shard), entry_offset, n_shards, l, 0, topk, nullptr,
                                        (cudaStream_t)stream));
}

csa2_status csa2_attend_partial(const csa2_cache *cache, int32_t heads, const uint16_t *q, const int32_t *topk,
                                float scale, int32_t with_window, float *o, float *lse, uint32_t flags,
                                csa2_stream_t stream)
{
    CSA2_TRACE("csa2_attend_partial");
    csa2_status st = check_cache(cache);
    if (st != CSA2_OK) return st;
    if (heads <= 0 || heads > 128 || !q || !topk || !o || !lse) return CSA2_ERR_INVALID_ARG;
    if (!aligned(o, 16) || !aligned(q, 16)) return CSA2_ERR_INVALID_ARG;
    if (flags & ~CSA2_ATTEND_INPUTS_SETTLED) return CSA2_ERR_INVALID_ARG;
    if (!with_window) flags |= ATT_NO_WINDOW;
    return from_cuda(launch_attend(make_view(cache), heads, q, topk, scale, o, 1, flags, (cudaStream_t)stream, lse));
}

csa2_status csa2_combine(int32_t n_parts, const float *const *o_parts, const float *const *lse_parts, int32_t batch,
                         int32_t heads, void *out, int32_t out_is_fp32, csa2_stream_t stream)
{
    CSA2_TRACE("csa2_combine");
    if (n_parts < 1 || n_parts > CSA2_MAX_SHARDS || !o_parts || !lse_parts || !out) return CSA2_ERR_INVALID_ARG;
    if (batch <= 0 || heads <= 0 || heads > 128 || (int64_t)batch * heads > 0x7fffffff || !aligned(out, 16))
        return CSA2_ERR_INVALID_ARG;
    PartList p{};
    for (int i = 0; i < n_parts; ++i) {
        if (!o_parts[i] || !lse_parts[i] || !aligned(o_parts[i], 16)) return CSA2_ERR_INVALID_ARG;
        p.o[i] = o_parts[i];
        p.lse[i] = lse_parts[i];
    }
    return from_cuda(launch_combine(n_parts, p, batch, heads, out, out_is_fp32, (cudaStream_t)stream));
}

csa2_status csa2_get_device_error(const csa2_cache *cache, int32_t *code_out, csa2_stream_t stream)
{
    CSA2_TRACE("csa2_get_device_error");
    if (!cache || !cache->error || !code_out) return CSA2_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    int32_t v = 0;
    cudaError_t e = cudaMemcpyAsync(&v, cache->error, sizeof(int32_t), cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e == cudaSuccess) e = cudaMemsetAsync(cache->error, 0, sizeof(int32_t), s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return CSA2_ERR_CUDA;
    *code_out = v;
    return v == 0 ? CSA2_OK : CSA2_ERR_DEVICE_CHECK;
}

csa2_status csa2_set_profile_events(int32_t kernel, void *ev_start, void *ev_stop)
{
    if (kernel < 0 || kernel >= CSA2_KERNEL_COUNT || (!ev_start) != (!ev_stop)) return CSA2_ERR_INVALID_ARG;
    g_prof[kernel][0] = (cudaEvent_t)ev_start;
    g_prof[kernel][1] = (cudaEvent_t)ev_stop;
    return CSA2_OK;
}

uint64_t csa2_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char *csa2_status_string(csa2_status status)
{
    switch (status) {
    case CSA2_OK: return "ok";
    case CSA2_ERR_INVALID_ARG: return "invalid argument";
    case CSA2_ERR_UNSUPPORTED: return "unsupported";
    case CSA2_ERR_CUDA: return "CUDA error";
    case CSA2_ERR_DEVICE_CHECK: return "device-side data check failed";
    case CSA2_ERR_TIMEOUT: return "device wait timed out";
    }
    return "unknown status";
}

}  // extern "C"

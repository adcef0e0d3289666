/*
 * csa2.h -- C ABI of libcsa2, the B200 (sm_100a) CSA2 sparse-attention
 * decode step over a compressed, FP4-quantised global KV cache.
 *
 * The method (DeepSeek-V4.1-Flash CSA2) is described by:
 *   [blog-0539] 0539edu.com/news/5732216, §1 (each m tokens become one cache
 *               entry; main KV, indexer K and top-k indices are reused across
 *               layers) and §3 (layer modes Full / Reuse / Reindex; the
 *               config: fp4_e2m1 global KV with one e4m3 scale per 16
 *               channels, fp8 SWA KV with a 128-token window, indexer of
 *               32 heads x 128 dims with top_k 512, hierarchical selection of
 *               2048 blocks x 8 positions = a 16384-candidate pool; the Full
 *               layer builds the pool and Reindex layers search inside it).
 *   [daiw]      daiw.net/manual/deepseek-v4-flash/million-token-cost: decode
 *               reads the cache every step and is bandwidth-bound; the
 *               cache-size factor table (one 512-dim KV shared by all query
 *               heads).
 *   [nxbn]      m.nxbn.cn/news/78290 §3.1 (E2M1 = 2 exponent bits, 1 mantissa
 *               bit), §4.2 (gated weighted compression of m tokens).
 *
 * Conventions shared by every call:
 *   - All data pointers are DEVICE pointers owned by the caller.  The library
 *     never allocates, frees or synchronises, except csa2_get_device_error,
 *     which synchronises the given stream.
 *   - Every call enqueues asynchronously on `stream` (0 = legacy default).
 *   - The return value reports host-side argument validation
 *     (CSA2_ERR_INVALID_ARG, nothing enqueued) and launch errors
 *     (CSA2_ERR_CUDA).  Errors found in the DATA on the device (a page id
 *     outside the pool, an entry index beyond a request's pages, a top-k index
 *     beyond the request's entries, a bad m or n_new) never trap: the kernel
 *     skips that element and records the first such code in cache->error;
 *     read it with csa2_get_device_error.
 *   - Multi-byte values are little-endian; bf16 values are passed as their
 *     16-bit patterns (uint16_t).
 */
#ifndef CSA2_H
#define CSA2_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *csa2_stream_t;   /* == cudaStream_t */

/* ---- method constants ([blog-0539] §3 config) ------------------------- */
#define CSA2_LATENT        512    /* shared latent (K = V) dim ([daiw])         */
#define CSA2_SCALE_GROUP   16     /* channels per e4m3 scale                    */
#define CSA2_CODE_BYTES    256    /* FP4 codes per entry: 512 x 4 bit           */
#define CSA2_SCALE_BYTES   32     /* e4m3 scales per entry: 512 / 16            */
#define CSA2_KEY_DIM       128    /* indexer head_dim; FP8 key bytes per entry  */
#define CSA2_IDX_HEADS     32     /* indexer query_heads                        */
#define CSA2_BLOCK         8      /* positions_per_block                        */
#define CSA2_MAX_BLOCKS    2048   /* max_blocks                                 */
#define CSA2_POOL          16384  /* candidate_pool_size = 2048 x 8             */
#define CSA2_TOPK          512    /* top_k                                      */
#define CSA2_SWA           128    /* swa_window_size                            */

/* ---- cache layout -------------------------------------------------------
 * Global KV lives in one pool of n_pages pages of 64 entries.  Entry e of
 * request b lives in page page_table[b * max_pages + (e >> 6)], slot e & 63.
 * The pool is stored as four planes, one per field, each holding that field
 * for every page in page-id order (so consecutive pages are contiguous within
 * a plane, and a scan over consecutive pages is one sequential stream):
 *   codes     plane at 0                : [n_pages][64][256] u8  FP4 e2m1
 *             codes; byte j = channel 2j (low nibble) | channel 2j+1 (high
 *             nibble); bit 3 of a nibble = sign
 *   scales    plane at n_pages * 16384  : [n_pages][64][32]  u8  e4m3 scale
 *             of channels 16i .. 16i+15
 *   keys      plane at n_pages * 18432  : [n_pages][64][128] u8  FP8 e4m3
 *             indexer key
 *   summaries plane at n_pages * 26624  : [n_pages][8][128]  u8  FP8 e4m3
 *             mean of the keys of block (e >> 3)
 * Pool size: n_pages * CSA2_PAGE_BYTES.  The plane offsets are multiples of
 * 256 bytes.  Per request, the SWA ring holds the last min(n_tokens, 128)
 * raw tokens: codes [128][512] u8 e4m3, then scale [128] f32 (a power of
 * two); token position t sits in slot t % 128.                               */
#define CSA2_PAGE_ENTRIES      64
#define CSA2_PAGE_CODES_BYTES  16384
#define CSA2_PAGE_SCALES_BYTES 2048
#define CSA2_PAGE_KEYS_BYTES   8192
#define CSA2_PAGE_SUMM_BYTES   1024
#define CSA2_PAGE_BYTES        27648
#define CSA2_PLANE_CODES(n_pages)  ((size_t)0)
#define CSA2_PLANE_SCALES(n_pages) ((size_t)(n_pages) * 16384)
#define CSA2_PLANE_KEYS(n_pages)   ((size_t)(n_pages) * 18432)
#define CSA2_PLANE_SUMM(n_pages)   ((size_t)(n_pages) * 26624)
#define CSA2_SWA_CODES_OFF     0
#define CSA2_SWA_SCALE_OFF     65536
#define CSA2_SWA_BYTES         66048
#define CSA2_PENDING_STRIDE    656    /* floats: latent 512 | key 128 | gate 1 | pad */

typedef enum {
    CSA2_OK = 0,
    CSA2_ERR_INVALID_ARG = 1,
    CSA2_ERR_UNSUPPORTED = 2,
    CSA2_ERR_CUDA = 3,
    CSA2_ERR_DEVICE_CHECK = 4,
    CSA2_ERR_TIMEOUT = 5
} csa2_status;

/* Device error word values (cache->error). */
#define CSA2_DEV_OK              0
#define CSA2_DEV_BAD_PAGE        1   /* page id outside [0, n_pages)            */
#define CSA2_DEV_CAPACITY        2   /* entry index >= max_pages * 64           */
#define CSA2_DEV_BAD_INDEX       3   /* top-k / pool index outside the request  */
#define CSA2_DEV_BAD_REQUEST     4   /* m not in {1,2}, n_new not in [0,2], ... */
#define CSA2_DEV_TIMEOUT         5   /* a bounded in-kernel wait gave up        */

typedef enum {
    CSA2_INDEX_FLAT = 0,     /* exact top-512 over every entry                   */
    CSA2_INDEX_FULL = 1,     /* hierarchical: blocks -> pool -> top-512; writes pool */
    CSA2_INDEX_REINDEX = 2   /* rescore a given pool, top-512                    */
} csa2_index_mode;

/* A batch of requests' caches.  The struct itself is host memory and is read
 * only during the call; every pointer in it is a device pointer owned by the
 * caller and must stay valid until the enqueued work completes. */
typedef struct {
    void          *pool;        /* n_pages * CSA2_PAGE_BYTES, 256-byte aligned          */
    int32_t        n_pages;
    const int32_t *page_table;  /* [batch][max_pages]                                   */
    int32_t        max_pages;   /* pages per request; entry capacity = 64 * max_pages   */
    int32_t       *n_tokens;    /* [batch] tokens seen; entries = n_tokens / m          */
    const int32_t *m;           /* [batch] compression ratio, 1 or 2                    */
    void          *swa;         /* [batch] * CSA2_SWA_BYTES, 256-byte aligned           */
    float         *pending;     /* [batch][CSA2_PENDING_STRIDE]: an m=2 request's odd token */
    int32_t       *error;       /* one device word; 0 = no data error                   */
    int32_t        batch;
} csa2_cache;

/* Sizes ------------------------------------------------------------------ */
size_t csa2_page_bytes(void);   /* CSA2_PAGE_BYTES */
size_t csa2_swa_bytes(void);    /* CSA2_SWA_BYTES  */

/* Bytes of workspace csa2_index and csa2_attend need for `batch` requests of
 * at most `max_entries` entries: the scan's row scores, the selected blocks
 * and 512 bytes per request for the range of the scan's scores (attention
 * needs none of it).  The range words are kept between calls: a fresh
 * workspace needs no initialisation (its first selection finds the range
 * itself), and any call's results are exact whatever they hold.  0 for batch <= 0 or max_entries < 0.
 * The caller allocates it (256-byte aligned) and may share one workspace
 * between calls that run in stream order. */
size_t csa2_workspace_bytes(int32_t batch, int32_t max_entries);

/* Bulk build (prefill side) ----------------------------------------------
 * Compress and pack tokens [tok_begin, tok_begin + n_tok) of request `req`
 * ([blog-0539] §1: m tokens -> one entry; [nxbn] §4.2: entry = sum_i
 * softmax(g)_i x_i over the m tokens of a group, for the latent and the
 * indexer key alike; m = 1 copies).  Writes the FP4 codes + e4m3 scales,
 * the FP8 key, recomputes the summaries of every block it touches, writes
 * tokens at positions >= n_tok_final - 128 into the SWA ring, keeps an m=2
 * request's unpaired last token in `pending`, and sets
 * n_tokens[req] = tok_begin + n_tok.
 *   lat  [n_tok][512] f32, key [n_tok][128] f32, gate [n_tok] f32 (device).
 *   tok_begin must be a multiple of m (read from m_host, which must equal
 *   cache->m[req]); calls for one request go in increasing tok_begin. */
csa2_status csa2_prefill(const csa2_cache *cache, int32_t req, int32_t m_host,
                         int32_t tok_begin, int32_t n_tok, int32_t n_tok_final,
                         const float *lat, const float *key, const float *gate,
                         csa2_stream_t stream);

/* Decode-step append ([blog-0539] §1, §3; [nxbn] §4.2) -------------------
 * Request b appends n_new[b] in {0,1,2} raw tokens: lat [batch][2][512],
 * key [batch][2][128], gate [batch][2] (f32, rows past n_new ignored).
 * Every new token enters the SWA ring as FP8 with a per-token power-of-two
 * scale; m=1 turns each token into an entry; m=2 pairs the pending odd token
 * (if any) with the new ones, completing entries and keeping a leftover
 * token pending.  Each new entry is packed as FP4 e2m1 + e4m3 per-16 scales
 * with its key in FP8, the summary of its block is recomputed, and
 * n_tokens[b] += n_new[b]. */
csa2_status csa2_append(const csa2_cache *cache, const float *lat, const float *key,
                        const float *gate, const int32_t *n_new, csa2_stream_t stream);

/* Indexer ([blog-0539] §3 indexer and hierarchical blocks, and the passage
 * that follows: Full builds the pool, Reindex searches only inside it) ----
 * score(row) = sum_h w_h * ReLU(q_idx_h . row) with q_idx bf16 [batch][32][128]
 * and w f32 [batch][32], rows being FP8 keys or block summaries.
 *   FLAT:    top-min(512, N) entries of all N.
 *   FULL:    top-min(2048, ceil(N/8)) blocks by summary score; their entries
 *            (ascending) form pool[b][0 .. pool_len[b]) (rest -1); exact
 *            rescoring of the pool's keys; top-min(512, pool_len).
 *   REINDEX: the pool/pool_len given (as written by a FULL call) is
 *            rescored with this layer's q_idx/w; top-min(512, pool_len).
 * topk[b][512] receives entry indices in ascending order, -1 padded.  Order
 * of selection: score descending, ties to the lower index.  pool and
 * pool_len are [batch][16384] / [batch] int32; unused (may be NULL) in FLAT
 * mode.  ws / ws_bytes: workspace of at least csa2_workspace_bytes(). */
csa2_status csa2_index(const csa2_cache *cache, csa2_index_mode mode,
                       const uint16_t *q_idx, const float *w,
                       int32_t *pool, int32_t *pool_len, int32_t *topk,
                       void *ws, size_t ws_bytes, csa2_stream_t stream);

/* The indexer's selection step on its own ([blog-0539] §3: top_k 512 of the
 * scored rows; top 2048 blocks in the hierarchical mode) ------------------
 * For each row b < batch: the top min(k, n[b]) of scores[b*stride + 0 ..
 * n[b]), score descending, ties to the lower index (-0 equals +0), written
 * as indices in ascending order to out[b*k ..], -1 padded to k.
 *   scores f32 device [batch][stride]; n int32 device [batch], each in
 *   0..stride (values outside are clamped); k in 1..2048; out int32 device
 *   [batch][k].  Scores must not be NaN.  Each row is selected by one
 *   CTA or by a cluster of 4, 8 or 16 CTAs (each CTA holding up to 32768
 *   elements), whichever a cost model of the batch's resident waves favours.
 *   No workspace. */
csa2_status csa2_topk(const float *scores, int64_t stride, const int32_t *n, int32_t batch, int32_t k,
                      int32_t *out, csa2_stream_t stream);

/* Sparse MQA decode attention ([daiw] decode step and factor table: one
 * 512-dim latent shared by all heads, used as both K and V) --------------
 * For every head h of request b:
 *   o_h = sum_j softmax_j(scale * q_h . v_j) v_j
 * over j in {valid topk[b][*] entries (FP4 e2m1 x e4m3 scale)} plus the
 * min(n_tokens[b], 128) SWA tokens (FP8 x power-of-two scale), one softmax,
 * no de-duplication.  q bf16 [batch][heads][512]; heads in 1..128.
 * out [batch][heads][512] is bf16 (out_is_fp32 = 0) or f32 (= 1).  A request
 * with no keys gets a zero output.  Reuse layers call this with their
 * group's topk and their own q (and may pass CSA2_ATTEND_INPUTS_SETTLED). */
csa2_status csa2_attend(const csa2_cache *cache, int32_t heads, const uint16_t *q,
                        const int32_t *topk, float scale, void *out, int32_t out_is_fp32,
                        uint32_t flags, void *ws, size_t ws_bytes, csa2_stream_t stream);

/* csa2_attend flags.  CSA2_ATTEND_INPUTS_SETTLED: topk, the cache rows it
 * names and n_tokens were last written by work that finished before the
 * kernel launched just before this call on `stream` (for example a Reuse
 * layer, whose indices come from its group's Full layer).  The kernel may
 * then gather and dequantise those rows while that previous kernel is still
 * running; only q is read after it completes.  Without the flag every input
 * is read after the previous kernel completes. */
#define CSA2_ATTEND_INPUTS_SETTLED 1u

/* Sequence-sharded decode of long requests --------------------------------
 * The pages describe decode on one device; they do not split a request.
 * These calls split each request's entries over G shards (normally one per
 * GPU), so that G devices share one long request's block scan, pool
 * rescoring and gathers, and they reproduce the unsharded result: the
 * selections are exactly those of csa2_index FULL / REINDEX (the global top-k
 * of a union of per-shard top-k lists equals the top-k of the whole, under
 * the same order: score descending, ties to the lower global index), and the
 * attention equals csa2_attend's up to fp32 rounding of the final merge.
 *
 * Shards.  Shard s of request b holds the request's global entries
 * [entry_offset[b], entry_offset[b] + N_s) in a csa2_cache of its own (its
 * n_tokens / m = N_s; its page table lists only its pages).  entry_offset is
 * a device int32 array [batch], a multiple of 8 (of 64 to keep pages whole);
 * a bad offset sets CSA2_DEV_BAD_REQUEST and the request selects nothing.
 * Shards are numbered in increasing offset and cover the request without
 * gaps.  Only the LAST shard holds the SWA window and takes appends; its
 * n_tokens must count at least min(total tokens, 128) tokens so that its
 * window is the request's.  Exchanged lists are passed as host arrays of
 * n_shards device pointers, in shard order, each to a [batch][k] array (the
 * buffers of an all-gather, or peers' memory mapped into this process); at
 * most CSA2_MAX_SHARDS shards.
 *
 * One Full layer on shard s:
 *   1. csa2_shard_blocks    local top-2048 blocks by summary score
 *   2. exchange             every shard's block ids + scores to every shard
 *   3. csa2_shard_pool      global top-2048 blocks; this shard's ones -> its pool
 *   4. csa2_shard_rescore   exact pool rescoring, local top-512
 *   5. exchange             every shard's top-512 ids + scores
 *   6. csa2_shard_topk      global top-512; this shard's entries -> its topk
 *   7. csa2_attend_partial  attention over its topk (+ window on the last
 *                           shard): normalised output and log-sum-exp
 *   8. exchange             outputs and log-sum-exps
 *   9. csa2_combine         log-sum-exp merge of the shards' outputs
 * A Reindex layer runs steps 4-9 on the Full layer's shard pool; a Reuse
 * layer runs steps 7-9 with its group's shard topk.                        */
#define CSA2_MAX_SHARDS 8

/* Step 1.  The top min(2048, ceil(N_s/8)) blocks of this shard by summary
 * score (as csa2_index FULL scores them): block_ids [batch][2048] gets
 * GLOBAL block numbers (local + entry_offset/8) ascending, -1 padded;
 * block_scores [batch][2048] their f32 scores, -inf padded.  ws: workspace
 * of csa2_workspace_bytes() for this shard's cache. */
csa2_status csa2_shard_blocks(const csa2_cache *shard, const int32_t *entry_offset,
                              const uint16_t *q_idx, const float *w,
                              int32_t *block_ids, float *block_scores,
                              void *ws, size_t ws_bytes, csa2_stream_t stream);

/* Step 3.  Over the n_shards lists of step 1 (cand_ids[s] / cand_scores[s],
 * each [batch][2048]): the global top-2048 blocks; those inside this shard
 * are expanded, ascending, into its pool [batch][16384] as LOCAL entry
 * indices (entries past N_s become -1), pool_len [batch] counts them. */
csa2_status csa2_shard_pool(const csa2_cache *shard, const int32_t *entry_offset, int32_t n_shards,
                            const int32_t *const *cand_ids, const float *const *cand_scores,
                            int32_t *pool, int32_t *pool_len, csa2_stream_t stream);

/* Step 4.  Exact rescoring of this shard's pool (csa2_index REINDEX's
 * arithmetic) and its top min(512, pool_len): ids [batch][512] get GLOBAL
 * entry indices ascending, -1 padded; scores [batch][512] f32, -inf padded. */
csa2_status csa2_shard_rescore(const csa2_cache *shard, const int32_t *entry_offset,
                               const uint16_t *q_idx, const float *w,
                               const int32_t *pool, const int32_t *pool_len,
                               int32_t *ids, float *scores, csa2_stream_t stream);

/* Step 6.  Over the n_shards lists of step 4 (each [batch][512]): the global
 * top-512 entries; those inside this shard go to topk [batch][512] as LOCAL
 * entry indices, ascending, -1 padded. */
csa2_status csa2_shard_topk(const csa2_cache *shard, const int32_t *entry_offset, int32_t n_shards,
                            const int32_t *const *cand_ids, const float *const *cand_scores,
                            int32_t *topk, csa2_stream_t stream);

/* Step 7.  csa2_attend over the valid topk entries, plus the window only
 * when with_window != 0, returning the pieces a merge needs:
 * o [batch][heads][512] f32, normalised over this call's keys (zero without
 * keys), and lse [batch][heads] f32 = ln sum_j exp(scale * q_h . v_j)
 * (-inf without keys).  flags as csa2_attend.  No workspace. */
csa2_status csa2_attend_partial(const csa2_cache *cache, int32_t heads, const uint16_t *q,
                                const int32_t *topk, float scale, int32_t with_window,
                                float *o, float *lse, uint32_t flags, csa2_stream_t stream);

/* Step 9.  out[b][h] = sum_s exp(lse_s - L) o_s[b][h] with
 * L = ln sum_s exp(lse_s) over the n_parts (1..CSA2_MAX_SHARDS) partial
 * results o_parts[s] [batch][heads][512] f32 and lse_parts[s]
 * [batch][heads] f32 (host arrays of device pointers); zero where every
 * lse is -inf.  out is bf16 (out_is_fp32 = 0) or f32 (= 1). */
csa2_status csa2_combine(int32_t n_parts, const float *const *o_parts, const float *const *lse_parts,
                         int32_t batch, int32_t heads, void *out, int32_t out_is_fp32,
                         csa2_stream_t stream);

/* Attention without a workspace ------------------------------------------
 * The pages have no counterpart to this call; it exists for callers that
 * cannot allocate device memory -- for instance code embedded in a host
 * framework that owns all device memory through its own pool and gives
 * plugins no way to allocate, or a serving loop that must not allocate once
 * it runs, because an allocation can synchronise the device.  It computes
 * what csa2_attend computes, with the same arguments minus ws, ws_bytes and
 * flags, using the attention variant that exchanges its per-split partials
 * through device memory: those partials live in one fixed array inside the
 * library.  Results agree with csa2_attend up to the order of the final
 * fp32 sum over the five splits.
 *   - Limit: batch * heads <= CSA2_ATTEND_NOALLOC_MAX_ROWS (512).  Larger
 *     calls return CSA2_ERR_UNSUPPORTED and enqueue nothing.
 *   - The array (512 x 5 x 512 floats, about 5.2 MB) exists on every GPU
 *     that loads the library and stays allocated until the process exits.
 *   - The first call on a device is set-up: with that device current it
 *     looks up the array's device address (cudaGetSymbolAddress), and CUDA,
 *     which loads a library's device code lazily by default, loads the
 *     module that holds the array at that moment -- allocating the array's
 *     device memory and possibly synchronising the device.  Make that first
 *     call on each device while setting up, before any stream capture and
 *     before the loop that must not allocate.  Later calls allocate and free
 *     nothing.
 *   - All calls share the one array and each overwrites every partial it
 *     reads, so nothing carries over between calls; but two calls whose GPU
 *     work can overlap (different streams, or concurrent host threads
 *     without ordering) race on it -- order them on one stream. */
#define CSA2_ATTEND_NOALLOC_MAX_ROWS 512
csa2_status csa2_attend_noalloc(const csa2_cache *cache, int32_t heads, const uint16_t *q,
                                const int32_t *topk, float scale, void *out, int32_t out_is_fp32,
                                csa2_stream_t stream);

/* Diagnostics ------------------------------------------------------------
 * Kernels that csa2_set_profile_events can bracket with CUDA events. */
typedef enum {
    CSA2_KERNEL_BLOCK_SCORE = 0,   /* FULL: scoring of the block summaries     */
    CSA2_KERNEL_FLAT_SCORE = 1,    /* FLAT: scoring of every key               */
    CSA2_KERNEL_POOL_SCORE = 2,    /* FULL / REINDEX: exact pool rescoring     */
    CSA2_KERNEL_SELECT = 3,        /* radix top-k                              */
    CSA2_KERNEL_ATTEND = 4,        /* split-KV attention partials              */
    CSA2_KERNEL_COMBINE = 5,       /* shard merges and csa2_combine            */
    CSA2_KERNEL_COUNT = 6
} csa2_kernel_id;

/* When ev_start / ev_stop (cudaEvent_t, created by the caller with timing
 * enabled) are non-NULL, every later launch of `kernel` is preceded by
 * cudaEventRecord(ev_start) and followed by cudaEventRecord(ev_stop) on the
 * stream it is launched on, so the pair brackets the most recent launch.
 * Pass NULLs to stop.  Process-wide setting; not thread-safe. */
csa2_status csa2_set_profile_events(int32_t kernel, void *ev_start, void *ev_stop);

/* Self-test of the bounded waits: launches one CTA that waits on a barrier
 * nothing completes; after `polls` polls (1..65536) it gives up and writes
 * CSA2_DEV_TIMEOUT to the device word *error_word (if it holds 0), as every
 * kernel of the library does when a wait runs out.  Nothing faults or
 * hangs.  For tests of the timeout reporting path. */
csa2_status csa2_selftest_wait_timeout(int32_t *error_word, uint32_t polls, csa2_stream_t stream);

/* Number of kernels this library has launched in this process so far. */
uint64_t csa2_launch_count(void);

/* Synchronises `stream`, copies cache->error into *code_out and resets the
 * device word to 0. */
csa2_status csa2_get_device_error(const csa2_cache *cache, int32_t *code_out,
                                  csa2_stream_t stream);

const char *csa2_status_string(csa2_status status);

#ifdef __cplusplus
}
#endif
#endif /* CSA2_H */

/*
 * CSA2 decode oracle: plain, slow, obviously-correct CPU definitions of every
 * step of the CSA2 sparse-attention decode path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library may call, link or
 * include this file; only the tests, the smoke check and the CPU-baseline leg
 * of the benchmark use it.  It shares no code, header, table or constant with
 * the CUDA path: every format and constant below is restated here from the
 * pages that define the method.
 *
 * Sources (cited by page and section):
 *   [blog-0539]  0539edu.com/news/5732216 "长上下文推理的显存瓶颈" -- §1 (three
 *                multiplicative dimensions: m tokens -> 1 entry, cross-layer
 *                reuse of KV / indexer K / top-k), §3 (CSA2 layer modes, the
 *                JSON/TOML config: fp4_e2m1 global KV with an e4m3 scale per
 *                16 channels, fp8 SWA KV with a 128-token window, indexer
 *                32 heads x 128 dims, top_k 512, hierarchical 2048 blocks x 8
 *                positions = 16384 candidates).
 *   [nxbn]       m.nxbn.cn/news/78290 §3.1 (E2M1: 1 sign, 2 exponent,
 *                1 mantissa bit), §4.2 (gated weighted compression).
 *   [daiw]       daiw.net/manual/deepseek-v4-flash/million-token-cost,
 *                "解码时每步要读多少" (attention reads the cache each step) and
 *                the "缓存大小的四个因子" table (one 512-dim KV shared by all
 *                query heads, i.e. MQA with K = V = latent).
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *   - e2m1 / e4m3 rounding: round to nearest, ties to the even code,
 *     saturating to the largest finite magnitude; the sign is kept (-0 -> 0x8).
 *   - FP4 scale: s = e4m3(amax/6) with amax/6 an IEEE fp32 division; if s is
 *     zero every code is 0x0; otherwise code = e2m1(x / s) (fp32 division).
 *   - Nibble order: byte j holds channel 2j (low nibble) and 2j+1 (high).
 *   - Indexer key: e4m3(x), no scale.
 *   - SWA token: e4m3(x * 2^-e) with e the smallest integer such that
 *     amax <= 448 * 2^e; the fp32 scale 2^e is stored beside the codes.
 *   - Compression (m = 2): p = softmax(g) in fp64, rounded to fp32;
 *     entry = fmaf(p1, x1, p0 * x0) with the fp32 product rounded first.
 *   - Block summary: fp32 sum of the dequantised FP8 keys present in the
 *     block (exact), divided by their count (fp32), then e4m3.
 *   - Indexer score: sum_h w_h * ReLU(q_h . k); accumulated in fp64, rounded
 *     once to fp32; selection decides on that fp32 value.
 *   - Top-k: order by (score desc, index asc); output ascending, -1 padded.
 *   - Attention: one softmax over the selected FP4 entries plus the SWA
 *     tokens (no de-duplication), logits = scale * (q . v), K = V = latent;
 *     fp64 throughout.  An empty key set gives a zero output.
 *
 * Build: gcc -O2 -ffp-contract=off -fPIC -shared (never -ffast-math).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---- method constants, restated from [blog-0539] §3 ---------------------- */
#define OR_LATENT      512   /* shared latent dim ([daiw] factor table)      */
#define OR_SCALE_GROUP 16    /* channels per e4m3 scale                       */
#define OR_IDX_DIM     128   /* indexer head_dim                              */
#define OR_IDX_HEADS   32    /* indexer query_heads                           */
#define OR_BLOCK       8     /* positions_per_block                           */
#define OR_MAX_BLOCKS  2048  /* max_blocks                                    */
#define OR_POOL        16384 /* candidate_pool_size = 2048 x 8                */
#define OR_TOPK        512   /* top_k                                         */
#define OR_SWA         128   /* swa_window_size                               */

/* ======================================================================
 * Number formats
 * ====================================================================== */

/* E2M1 ([nxbn] §3.1): bit 3 sign, bits 2..1 exponent (bias 1), bit 0
 * mantissa.  Exponent field 0 is subnormal: m * 0.5. */
double orc_e2m1_decode(uint8_t code)
{
    int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    double mag = (e == 0) ? m * 0.5 : (1.0 + m / 2.0) * ldexp(1.0, e - 1);
    return s ? -mag : mag;
}

/* E4M3 (the "e4m3" of [blog-0539] §3): bit 7 sign, bits 6..3 exponent
 * (bias 7), bits 2..0 mantissa; exponent 0 is subnormal m/8 * 2^-6;
 * 0x7F / 0xFF are NaN, there is no infinity. */
double orc_e4m3_decode(uint8_t code)
{
    int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
    if (e == 15 && m == 7) return NAN;
    double mag = (e == 0) ? (m / 8.0) * ldexp(1.0, -6) : (1.0 + m / 8.0) * ldexp(1.0, e - 7);
    return s ? -mag : mag;
}

/* Nearest magnitude code by search over the ascending table of finite
 * magnitudes mags[0..n-1] (code == table position); ties go to the even
 * code; anything at or above the top magnitude saturates to it. */
static int nearest_code(const double *mags, int n, double a)
{
    if (a >= mags[n - 1]) return n - 1;
    int lo = 0, hi = n - 1;                 /* invariant: mags[lo] <= a < mags[hi] */
    while (hi - lo > 1) {
        int mid = (lo + hi) / 2;
        if (mags[mid] <= a) lo = mid; else hi = mid;
    }
    double dlo = a - mags[lo], dhi = mags[hi] - a;
    if (dlo < dhi) return lo;
    if (dhi < dlo) return hi;
    return (lo % 2 == 0) ? lo : hi;
}

static double g_e2m1_mag[8];
static double g_e4m3_mag[127];
static int g_tables_ready = 0;

static void init_tables(void)
{
    if (g_tables_ready) return;
    for (int c = 0; c < 8; ++c) g_e2m1_mag[c] = orc_e2m1_decode((uint8_t)c);
    for (int c = 0; c < 127; ++c) g_e4m3_mag[c] = orc_e4m3_decode((uint8_t)c);
    g_tables_ready = 1;
}

uint8_t orc_e2m1_encode(float x)
{
    init_tables();
    uint8_t sign = signbit(x) ? 0x8 : 0x0;
    return (uint8_t)(sign | nearest_code(g_e2m1_mag, 8, fabs((double)x)));
}

uint8_t orc_e4m3_encode(float x)
{
    init_tables();
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    return (uint8_t)(sign | nearest_code(g_e4m3_mag, 127, fabs((double)x)));
}

float orc_bf16_to_float(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* ======================================================================
 * Append: compression and packing  ([blog-0539] §1, §3; [nxbn] §4.2)
 * ====================================================================== */

/* m tokens -> one entry: e = sum_i softmax(g)_i x_i.  m = 1 is the identity. */
void orc_compress(int m, const float *x, const float *g, int dim, float *out)
{
    if (m == 1) {
        memcpy(out, x, sizeof(float) * (size_t)dim);
        return;
    }
    double gmax = g[0] > g[1] ? g[0] : g[1];
    double e0 = exp((double)g[0] - gmax), e1 = exp((double)g[1] - gmax);
    float p0 = (float)(e0 / (e0 + e1));
    float p1 = (float)(e1 / (e0 + e1));
    for (int d = 0; d < dim; ++d) {
        float t = p0 * x[d];
        out[d] = fmaf(p1, x[dim + d], t);
    }
}

/* 512-dim latent -> 256 code bytes (two e2m1 per byte) + 32 e4m3 scales. */
void orc_pack_latent(const float *e, uint8_t *codes, uint8_t *scales)
{
    uint8_t nib[OR_LATENT];
    for (int g = 0; g < OR_LATENT / OR_SCALE_GROUP; ++g) {
        const float *x = e + g * OR_SCALE_GROUP;
        float amax = 0.0f;
        for (int i = 0; i < OR_SCALE_GROUP; ++i) {
            float a = fabsf(x[i]);
            if (a > amax) amax = a;
        }
        float sf = amax / 6.0f;
        uint8_t sc = orc_e4m3_encode(sf);
        float s = (float)orc_e4m3_decode(sc);
        scales[g] = sc;
        for (int i = 0; i < OR_SCALE_GROUP; ++i)
            nib[g * OR_SCALE_GROUP + i] = (s == 0.0f) ? 0 : orc_e2m1_encode(x[i] / s);
    }
    for (int j = 0; j < OR_LATENT / 2; ++j)
        codes[j] = (uint8_t)(nib[2 * j] | (nib[2 * j + 1] << 4));
}

void orc_unpack_latent(const uint8_t *codes, const uint8_t *scales, double *out)
{
    for (int d = 0; d < OR_LATENT; ++d) {
        uint8_t byte = codes[d / 2];
        uint8_t c = (d % 2 == 0) ? (byte & 0xF) : (byte >> 4);
        out[d] = orc_e2m1_decode(c) * orc_e4m3_decode(scales[d / OR_SCALE_GROUP]);
    }
}

void orc_quant_key(const float *k, uint8_t *out)
{
    for (int i = 0; i < OR_IDX_DIM; ++i) out[i] = orc_e4m3_encode(k[i]);
}

/* Summary of one block: mean of the c dequantised FP8 keys present. */
void orc_block_summary(const uint8_t *keys, int c, uint8_t *out)
{
    for (int i = 0; i < OR_IDX_DIM; ++i) {
        double sum = 0.0;
        for (int j = 0; j < c; ++j) sum += orc_e4m3_decode(keys[j * OR_IDX_DIM + i]);
        float mean = (float)sum / (float)c;    /* the sum is exact in fp32 */
        out[i] = orc_e4m3_encode(mean);
    }
}

/* SWA token: per-token power-of-two scale, then e4m3. */
void orc_swa_quant(const float *x, uint8_t *codes, float *scale)
{
    float amax = 0.0f;
    for (int d = 0; d < OR_LATENT; ++d) {
        float a = fabsf(x[d]);
        if (a > amax) amax = a;
    }
    int e = 0;
    if (amax > 0.0f) {
        e = (int)ceil(log2((double)amax / 448.0));
        while ((double)amax > 448.0 * ldexp(1.0, e)) ++e;
        while ((double)amax <= 448.0 * ldexp(1.0, e - 1)) --e;
    }
    *scale = ldexpf(1.0f, e);
    for (int d = 0; d < OR_LATENT; ++d) codes[d] = orc_e4m3_encode(ldexpf(x[d], -e));
}

/* Bulk build of one request's entries [e_begin, e_end) from its raw tokens.
 * tok_* hold tokens [m*e_begin, m*e_end) (row-major, latent 512 / key 128 /
 * gate 1).  Any output pointer may be NULL to skip that field. */
void orc_build_entries(int m, int e_begin, int e_end,
                       const float *tok_lat, const float *tok_key, const float *tok_gate,
                       uint8_t *codes, uint8_t *scales, uint8_t *keys8)
{
    float lat[2 * OR_LATENT], key[2 * OR_IDX_DIM], ent[OR_LATENT], ek[OR_IDX_DIM];
    for (int e = e_begin; e < e_end; ++e) {
        int r = (e - e_begin) * m;
        for (int i = 0; i < m; ++i) {
            if (codes || scales)
                memcpy(lat + i * OR_LATENT, tok_lat + (size_t)(r + i) * OR_LATENT, sizeof(float) * OR_LATENT);
            memcpy(key + i * OR_IDX_DIM, tok_key + (size_t)(r + i) * OR_IDX_DIM, sizeof(float) * OR_IDX_DIM);
        }
        const float *g = tok_gate + r;
        size_t o = (size_t)(e - e_begin);
        if (codes || scales) {
            orc_compress(m, lat, g, OR_LATENT, ent);
            uint8_t c[OR_LATENT / 2], s[OR_LATENT / OR_SCALE_GROUP];
            orc_pack_latent(ent, c, s);
            if (codes) memcpy(codes + o * (OR_LATENT / 2), c, OR_LATENT / 2);
            if (scales) memcpy(scales + o * (OR_LATENT / OR_SCALE_GROUP), s, OR_LATENT / OR_SCALE_GROUP);
        }
        if (keys8) {
            orc_compress(m, key, g, OR_IDX_DIM, ek);
            orc_quant_key(ek, keys8 + o * OR_IDX_DIM);
        }
    }
}

/* Summaries of all blocks of a request with N entries (keys8 is [N][128]). */
void orc_build_summaries(const uint8_t *keys8, int n_entries, uint8_t *summ)
{
    int nb = (n_entries + OR_BLOCK - 1) / OR_BLOCK;
    for (int b = 0; b < nb; ++b) {
        int c = n_entries - b * OR_BLOCK;
        if (c > OR_BLOCK) c = OR_BLOCK;
        orc_block_summary(keys8 + (size_t)b * OR_BLOCK * OR_IDX_DIM, c, summ + (size_t)b * OR_IDX_DIM);
    }
}

/* ======================================================================
 * Indexer  ([blog-0539] §3 indexer + hierarchical block, and the passage
 * after it: the Full layer builds the pool, Reindex layers search inside it)
 * ====================================================================== */

/* sum_h w_h * ReLU(q_h . k), exact products, fp64 accumulation. */
double orc_index_score_f64(const uint16_t *q, const float *w, const uint8_t *k8)
{
    double kv[OR_IDX_DIM];
    for (int i = 0; i < OR_IDX_DIM; ++i) kv[i] = orc_e4m3_decode(k8[i]);
    double s = 0.0;
    for (int h = 0; h < OR_IDX_HEADS; ++h) {
        double dot = 0.0;
        for (int i = 0; i < OR_IDX_DIM; ++i)
            dot += (double)orc_bf16_to_float(q[h * OR_IDX_DIM + i]) * kv[i];
        if (dot > 0.0) s += (double)w[h] * dot;
    }
    return s;
}

void orc_score_rows(const uint16_t *q, const float *w, const uint8_t *rows, int n,
                    float *s32, double *s64)
{
    for (int i = 0; i < n; ++i) {
        double s = orc_index_score_f64(q, w, rows + (size_t)i * OR_IDX_DIM);
        if (s64) s64[i] = s;
        if (s32) s32[i] = (float)s;
    }
}

typedef struct { float s; int32_t i; } scored_t;

static int by_score_then_index(const void *pa, const void *pb)
{
    const scored_t *a = (const scored_t *)pa, *b = (const scored_t *)pb;
    if (a->s > b->s) return -1;
    if (a->s < b->s) return 1;
    return (a->i < b->i) ? -1 : (a->i > b->i);
}

static int ascending_int(const void *pa, const void *pb)
{
    int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    return (a > b) - (a < b);
}

/* Exact top-k by full sort: (score desc, index asc); ids[i] names element i
 * (NULL means ids[i] = i).  Writes min(k, n) ids ascending, then -1 padding
 * up to k.  Returns min(k, n). */
int orc_topk(const float *s, const int32_t *ids, int n, int k, int32_t *out)
{
    scored_t *v = (scored_t *)malloc(sizeof(scored_t) * (size_t)(n > 0 ? n : 1));
    for (int i = 0; i < n; ++i) {
        v[i].s = (s[i] == 0.0f) ? 0.0f : s[i];   /* -0 is +0 */
        v[i].i = ids ? ids[i] : i;
    }
    qsort(v, (size_t)n, sizeof(scored_t), by_score_then_index);
    int kk = n < k ? n : k;
    for (int i = 0; i < kk; ++i) out[i] = v[i].i;
    qsort(out, (size_t)kk, sizeof(int32_t), ascending_int);
    for (int i = kk; i < k; ++i) out[i] = -1;
    free(v);
    return kk;
}

/* Flat mode: top-512 over every entry of the request. */
int orc_index_flat(const uint16_t *q, const float *w, const uint8_t *keys8, int n_entries,
                   int32_t *topk)
{
    float *s = (float *)malloc(sizeof(float) * (size_t)(n_entries > 0 ? n_entries : 1));
    orc_score_rows(q, w, keys8, n_entries, s, NULL);
    int r = orc_topk(s, NULL, n_entries, OR_TOPK, topk);
    free(s);
    return r;
}

/* Pool of the selected blocks: every existing entry of each block, in
 * ascending order (blocks given ascending, -1 padded).  Returns its length. */
int orc_expand_pool(const int32_t *blocks, int n_blocks, int n_entries, int32_t *pool)
{
    int len = 0;
    for (int i = 0; i < n_blocks; ++i) {
        if (blocks[i] < 0) continue;
        for (int j = 0; j < OR_BLOCK; ++j) {
            int e = blocks[i] * OR_BLOCK + j;
            if (e < n_entries) pool[len++] = e;
        }
    }
    for (int i = len; i < OR_POOL; ++i) pool[i] = -1;
    return len;
}

/* Exact rescoring of a pool and its top-512 (also the whole Reindex mode). */
int orc_index_pool(const uint16_t *q, const float *w, const uint8_t *keys8,
                   const int32_t *pool, int pool_len, int32_t *topk)
{
    float *s = (float *)malloc(sizeof(float) * (size_t)(pool_len > 0 ? pool_len : 1));
    for (int i = 0; i < pool_len; ++i)
        s[i] = (float)orc_index_score_f64(q, w, keys8 + (size_t)pool[i] * OR_IDX_DIM);
    int r = orc_topk(s, pool, pool_len, OR_TOPK, topk);
    free(s);
    return r;
}

/* Full mode, hierarchical: block summaries -> top-min(2048, nb) blocks ->
 * pool of up to 16384 entries -> exact scores -> top-512.  blocks_out may be
 * NULL.  Returns the pool length. */
int orc_index_full(const uint16_t *q, const float *w, const uint8_t *keys8, const uint8_t *summ,
                   int n_entries, int32_t *blocks_out, int32_t *pool, int32_t *topk)
{
    int nb = (n_entries + OR_BLOCK - 1) / OR_BLOCK;
    float *s = (float *)malloc(sizeof(float) * (size_t)(nb > 0 ? nb : 1));
    int32_t blocks[OR_MAX_BLOCKS];
    orc_score_rows(q, w, summ, nb, s, NULL);
    orc_topk(s, NULL, nb, OR_MAX_BLOCKS, blocks);
    free(s);
    if (blocks_out) memcpy(blocks_out, blocks, sizeof(blocks));
    int len = orc_expand_pool(blocks, OR_MAX_BLOCKS, n_entries, pool);
    orc_index_pool(q, w, keys8, pool, len, topk);
    return len;
}

/* ======================================================================
 * Attention  ([daiw] "解码时每步要读多少" and the factor table: one 512-dim
 * KV shared by all query heads; [blog-0539] §3: FP4 global KV + FP8 SWA-128)
 * ====================================================================== */

/* o_h = sum_j softmax_j(scale * q_h . v_j) v_j over n_sel FP4 rows and n_swa
 * FP8 rows.  q is bf16 [H][512]; out is fp64 [H][512].  When lse is not
 * NULL it receives, per head, the log of the softmax denominator measured
 * from zero: ln sum_j exp(scale * q_h . v_j) (-inf for an empty key set). */
void orc_attend_lse(int H, const uint16_t *q, int n_sel, const uint8_t *codes, const uint8_t *scales,
                    int n_swa, const uint8_t *swa_codes, const float *swa_scale, double scale,
                    double *out, double *lse)
{
    int n = n_sel + n_swa;
    double *v = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1) * OR_LATENT);
    double *p = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    for (int j = 0; j < n_sel; ++j)
        orc_unpack_latent(codes + (size_t)j * (OR_LATENT / 2), scales + (size_t)j * (OR_LATENT / OR_SCALE_GROUP),
                          v + (size_t)j * OR_LATENT);
    for (int j = 0; j < n_swa; ++j)
        for (int d = 0; d < OR_LATENT; ++d)
            v[(size_t)(n_sel + j) * OR_LATENT + d] =
                orc_e4m3_decode(swa_codes[(size_t)j * OR_LATENT + d]) * (double)swa_scale[j];
    for (int h = 0; h < H; ++h) {
        double *o = out + (size_t)h * OR_LATENT;
        for (int d = 0; d < OR_LATENT; ++d) o[d] = 0.0;
        if (lse) lse[h] = -INFINITY;
        if (n == 0) continue;
        double qd[OR_LATENT];
        for (int d = 0; d < OR_LATENT; ++d) qd[d] = orc_bf16_to_float(q[h * OR_LATENT + d]);
        double mx = -INFINITY;
        for (int j = 0; j < n; ++j) {
            double dot = 0.0;
            for (int d = 0; d < OR_LATENT; ++d) dot += qd[d] * v[(size_t)j * OR_LATENT + d];
            p[j] = scale * dot;
            if (p[j] > mx) mx = p[j];
        }
        double l = 0.0;
        for (int j = 0; j < n; ++j) { p[j] = exp(p[j] - mx); l += p[j]; }
        if (lse) lse[h] = mx + log(l);
        for (int j = 0; j < n; ++j) {
            double pj = p[j] / l;
            for (int d = 0; d < OR_LATENT; ++d) o[d] += pj * v[(size_t)j * OR_LATENT + d];
        }
    }
    free(v);
    free(p);
}

void orc_attend(int H, const uint16_t *q, int n_sel, const uint8_t *codes, const uint8_t *scales,
                int n_swa, const uint8_t *swa_codes, const float *swa_scale, double scale,
                double *out)
{
    orc_attend_lse(H, q, n_sel, codes, scales, n_swa, swa_codes, swa_scale, scale, out, NULL);
}

/* Merge of attention results over disjoint parts of one key set: part s
 * holds o_s (normalised over its keys) and lse_s = ln of its softmax
 * denominator.  The whole set's denominator is sum_s exp(lse_s), so
 *   o = sum_s exp(lse_s - L) o_s,   L = ln sum_s exp(lse_s),
 * evaluated with the largest lse_s factored out.  Parts with lse_s = -inf
 * (no keys) weigh nothing; with no keys at all the output is zero.
 * o_parts [P][rows][512], lse_parts [P][rows], out [rows][512], fp64. */
void orc_lse_combine(int n_parts, int rows, const double *o_parts, const double *lse_parts, double *out)
{
    for (int r = 0; r < rows; ++r) {
        double mx = -INFINITY;
        for (int s = 0; s < n_parts; ++s)
            if (lse_parts[(size_t)s * rows + r] > mx) mx = lse_parts[(size_t)s * rows + r];
        double *o = out + (size_t)r * OR_LATENT;
        for (int d = 0; d < OR_LATENT; ++d) o[d] = 0.0;
        if (mx == -INFINITY) continue;
        double den = 0.0;
        for (int s = 0; s < n_parts; ++s) den += exp(lse_parts[(size_t)s * rows + r] - mx);
        for (int s = 0; s < n_parts; ++s) {
            const double ws = exp(lse_parts[(size_t)s * rows + r] - mx) / den;
            const double *os = o_parts + ((size_t)s * rows + r) * OR_LATENT;
            for (int d = 0; d < OR_LATENT; ++d) o[d] += ws * os[d];
        }
    }
}

/* ======================================================================
 * Array conveniences for the Python wrapper (element-wise loops only)
 * ====================================================================== */
void orc_e2m1_encode_n(const float *x, long n, uint8_t *out)
{
    for (long i = 0; i < n; ++i) out[i] = orc_e2m1_encode(x[i]);
}
void orc_e4m3_encode_n(const float *x, long n, uint8_t *out)
{
    for (long i = 0; i < n; ++i) out[i] = orc_e4m3_encode(x[i]);
}
void orc_e4m3_decode_n(const uint8_t *c, long n, double *out)
{
    for (long i = 0; i < n; ++i) out[i] = orc_e4m3_decode(c[i]);
}
void orc_e2m1_decode_n(const uint8_t *c, long n, double *out)
{
    for (long i = 0; i < n; ++i) out[i] = orc_e2m1_decode(c[i]);
}
void orc_swa_quant_n(const float *x, long n_tok, uint8_t *codes, float *scale)
{
    for (long t = 0; t < n_tok; ++t)
        orc_swa_quant(x + t * OR_LATENT, codes + t * OR_LATENT, scale + t);
}

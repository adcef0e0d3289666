// Append / bulk-build kernels: gated m -> 1 compression, FP4 e2m1 packing
// with e4m3 per-16-channel scales, FP8 indexer keys, block summaries, the
// FP8 SWA ring and an m=2 request's pending token.
//
// Sources: 0539edu.com/news/5732216 §1 (m tokens -> one entry) and §3 (the
// fp4_e2m1 / e4m3_per_16_channel / fp8 SWA-128 config); m.nxbn.cn/news/78290
// §4.2 (gated weighted compression), §3.1 (E2M1).
//
// Every value written here must match the CPU definition bit for bit, so the
// arithmetic is spelled out with explicitly rounded intrinsics (no FMA
// contraction): p = softmax(g) in fp64 rounded to fp32, entry =
// fma(p1, x1, p0 * x0); scale = e4m3(amax / 6); code = e2m1(x / scale).
#include "common.cuh"

namespace csa2 {

// Softmax weights of a 2-token group, fp64 then rounded to fp32.
__device__ __forceinline__ void gate_weights(float g0, float g1, float &p0, float &p1)
{
    double gm = g0 > g1 ? (double)g0 : (double)g1;
    double e0 = exp((double)g0 - gm), e1 = exp((double)g1 - gm);
    p0 = (float)(e0 / (e0 + e1));
    p1 = (float)(e1 / (e0 + e1));
}

// One warp packs one entry.  x0/x1 point at the group's token rows (x1 unused
// when m == 1); lane l owns latent channels 16l..16l+15 (= scale group l) and
// key channels 4l..4l+3.
__device__ __forceinline__ void pack_entry_warp(const float *lat0, const float *lat1,
                                                const float *key0, const float *key1,
                                                int m, float p0, float p1,
                                                const CacheView &c, int pid, int slot, int lane)
{
    float x[16];
#pragma unroll
    for (int i = 0; i < 16; i += 4) {
        float4 a = *reinterpret_cast<const float4 *>(lat0 + 16 * lane + i);
        if (m == 2) {
            float4 b = *reinterpret_cast<const float4 *>(lat1 + 16 * lane + i);
            a.x = __fmaf_rn(p1, b.x, __fmul_rn(p0, a.x));
            a.y = __fmaf_rn(p1, b.y, __fmul_rn(p0, a.y));
            a.z = __fmaf_rn(p1, b.z, __fmul_rn(p0, a.z));
            a.w = __fmaf_rn(p1, b.w, __fmul_rn(p0, a.w));
        }
        x[i] = a.x; x[i + 1] = a.y; x[i + 2] = a.z; x[i + 3] = a.w;
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(x[i]));
    uint8_t sc = f32_to_e4m3(__fdiv_rn(amax, 6.0f));
    float s = e4m3_to_f32(sc);
    uint32_t lo = 0, hi = 0;
    if (s != 0.0f) {
#pragma unroll
        for (int i = 0; i < 8; ++i) lo |= f32_to_e2m1(__fdiv_rn(x[i], s)) << (4 * i);
#pragma unroll
        for (int i = 0; i < 8; ++i) hi |= f32_to_e2m1(__fdiv_rn(x[8 + i], s)) << (4 * i);
    }
    *reinterpret_cast<uint2 *>(codes_row(c, pid, slot) + 8 * lane) = make_uint2(lo, hi);
    scales_row(c, pid, slot)[lane] = sc;

    float4 k = *reinterpret_cast<const float4 *>(key0 + 4 * lane);
    if (m == 2) {
        float4 k1 = *reinterpret_cast<const float4 *>(key1 + 4 * lane);
        k.x = __fmaf_rn(p1, k1.x, __fmul_rn(p0, k.x));
        k.y = __fmaf_rn(p1, k1.y, __fmul_rn(p0, k.y));
        k.z = __fmaf_rn(p1, k1.z, __fmul_rn(p0, k.z));
        k.w = __fmaf_rn(p1, k1.w, __fmul_rn(p0, k.w));
    }
    uint32_t kw = (uint32_t)f32_to_e4m3(k.x) | ((uint32_t)f32_to_e4m3(k.y) << 8) |
                  ((uint32_t)f32_to_e4m3(k.z) << 16) | ((uint32_t)f32_to_e4m3(k.w) << 24);
    *reinterpret_cast<uint32_t *>(keys_row(c, pid, slot) + 4 * lane) = kw;
}

// One warp quantises one raw token into its SWA slot.
__device__ __forceinline__ void swa_token_warp(const float *lat, uint8_t *swa, int slot, int lane)
{
    float x[16];
#pragma unroll
    for (int i = 0; i < 16; i += 4) {
        float4 a = *reinterpret_cast<const float4 *>(lat + 16 * lane + i);
        x[i] = a.x; x[i + 1] = a.y; x[i + 2] = a.z; x[i + 3] = a.w;
    }
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(x[i]));
#pragma unroll
    for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    int e = amax > 0.0f ? swa_exponent(amax) : 0;
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
        w[i] = (uint32_t)f32_to_e4m3(ldexpf(x[4 * i], -e)) |
               ((uint32_t)f32_to_e4m3(ldexpf(x[4 * i + 1], -e)) << 8) |
               ((uint32_t)f32_to_e4m3(ldexpf(x[4 * i + 2], -e)) << 16) |
               ((uint32_t)f32_to_e4m3(ldexpf(x[4 * i + 3], -e)) << 24);
    *reinterpret_cast<uint4 *>(swa + CSA2_SWA_CODES_OFF + slot * CSA2_LATENT + 16 * lane) =
        make_uint4(w[0], w[1], w[2], w[3]);
    if (lane == 0)
        reinterpret_cast<float *>(swa + CSA2_SWA_SCALE_OFF)[slot] = ldexpf(1.0f, e);
}

// Summary of block `blk` of request b: e4m3(mean of the c present FP8 keys).
// 128 threads, thread i = channel i.
__device__ __forceinline__ void block_summary(const CacheView &c, int b, int blk, int n_entries, int i)
{
    int cnt = min(CSA2_BLOCK, n_entries - blk * CSA2_BLOCK);
    if (cnt <= 0) return;
    const int pid = entry_pid(c, b, blk * CSA2_BLOCK);
    if (pid < 0) return;
    int slot0 = (blk * CSA2_BLOCK) & (CSA2_PAGE_ENTRIES - 1);
    float sum = 0.0f;   // exact: e4m3 values are multiples of 2^-9 below 2^9
    for (int j = 0; j < cnt; ++j) sum += e4m3_to_f32(keys_row(c, pid, slot0 + j)[i]);
    summ_row(c, pid, blk & 7)[i] = f32_to_e4m3(__fdiv_rn(sum, (float)cnt));
}

// ------------------------------------------------------------------ prefill
// Grid: one CTA of 8 warps per 8 entries; warp w packs entry e_first + 8*bid + w.
__global__ void __launch_bounds__(256) prefill_entries_kernel(CacheView c, int req, int m, int e_first,
                                                              int n_ent, const float *lat, const float *key,
                                                              const float *gate)
{
    int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int le = blockIdx.x * 8 + w;
    if (le >= n_ent) return;
    int e = e_first + le;
    const int pid = entry_pid(c, req, e);
    if (pid < 0) return;
    int r0 = le * m;
    float p0 = 1.0f, p1 = 0.0f;
    if (m == 2) gate_weights(gate[r0], gate[r0 + 1], p0, p1);
    const float *l0 = lat + (size_t)r0 * CSA2_LATENT, *k0 = key + (size_t)r0 * CSA2_KEY_DIM;
    pack_entry_warp(l0, l0 + CSA2_LATENT, k0, k0 + CSA2_KEY_DIM, m, p0, p1, c, pid, e & (CSA2_PAGE_ENTRIES - 1),
                    lane);
}

__global__ void __launch_bounds__(128) prefill_summary_kernel(CacheView c, int req, int blk_first, int n_entries)
{
    block_summary(c, req, blk_first + blockIdx.x, n_entries, threadIdx.x);
}

// Tokens [t_first, t_first + n) of the chunk (chunk-relative row r0) into SWA;
// one warp per token.  Also stores an m=2 request's unpaired last token and
// finally publishes n_tokens.
__global__ void __launch_bounds__(256) prefill_swa_kernel(CacheView c, int req, int tok_begin, int t_first,
                                                          int n, const float *lat, const float *key,
                                                          const float *gate, int pend_row, int n_tok_total)
{
    int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int i = blockIdx.x * 8 + w;
    if (i < n) {
        int t = t_first + i;
        swa_token_warp(lat + (size_t)(t - tok_begin) * CSA2_LATENT, swa_base(c, req), t % CSA2_SWA, lane);
    }
    if (blockIdx.x == 0 && pend_row >= 0) {
        float *pd = c.pending + (size_t)req * CSA2_PENDING_STRIDE;
        for (int j = threadIdx.x; j < CSA2_LATENT; j += blockDim.x) pd[j] = lat[(size_t)pend_row * CSA2_LATENT + j];
        for (int j = threadIdx.x; j < CSA2_KEY_DIM; j += blockDim.x)
            pd[CSA2_LATENT + j] = key[(size_t)pend_row * CSA2_KEY_DIM + j];
        if (threadIdx.x == 0) pd[CSA2_LATENT + CSA2_KEY_DIM] = gate[pend_row];
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) c.n_tokens[req] = n_tok_total;
}

// ------------------------------------------------------------------ append
// One CTA (8 warps) per request.
__global__ void __launch_bounds__(256) append_kernel(CacheView c, const float *lat, const float *key,
                                                     const float *gate, const int32_t *n_new_arr)
{
    // pending + up to 2 new tokens; rows padded to 644 floats so every row
    // (and its key part at +512) is 16-byte aligned for the float4 loads.
    __shared__ __align__(16) float s_tok[3][CSA2_LATENT + CSA2_KEY_DIM + 4];
    __shared__ int s_ent[2];
    int b = blockIdx.x;
    int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    grid_dependency_wait();
    allow_dependents();
    int n0 = c.n_tokens[b];
    int m = c.m[b];
    int k = n_new_arr[b];
    if (k < 0 || k > 2 || (m != 1 && m != 2)) {
        if (threadIdx.x == 0) set_error(c.error, CSA2_DEV_BAD_REQUEST);
        return;
    }
    if (k == 0) return;
    const int W = CSA2_LATENT + CSA2_KEY_DIM + 1;
    bool has_pend = (m == 2) && (n0 & 1);
    // Stage the token sequence: [pending?] new0 [new1].
    int nt = (has_pend ? 1 : 0) + k;
    for (int j = threadIdx.x; j < W; j += blockDim.x) {
        int t = 0;
        if (has_pend) s_tok[t++][j] = c.pending[(size_t)b * CSA2_PENDING_STRIDE + j];
        for (int i = 0; i < k; ++i, ++t) {
            float v;
            if (j < CSA2_LATENT) v = lat[((size_t)b * 2 + i) * CSA2_LATENT + j];
            else if (j < CSA2_LATENT + CSA2_KEY_DIM) v = key[((size_t)b * 2 + i) * CSA2_KEY_DIM + (j - CSA2_LATENT)];
            else v = gate[(size_t)b * 2 + i];
            s_tok[t][j] = v;
        }
    }
    __syncthreads();
    // SWA: every new token (warps 0, 1).
    if (w < k) {
        int t = n0 + w;
        swa_token_warp(&s_tok[(has_pend ? 1 : 0) + w][0], swa_base(c, b), t % CSA2_SWA, lane);
    }
    // Entries: m=1 -> one per new token; m=2 -> one per complete pair.
    int n_ent = (m == 1) ? k : nt / 2;
    int e0 = n0 / m;
    if (w >= 2 && w - 2 < n_ent) {
        int i = w - 2;
        int e = e0 + i;
        const int pid = entry_pid(c, b, e);
        if (pid >= 0) {
            const float *t0 = &s_tok[i * m][0];
            const float *t1 = (m == 2) ? &s_tok[i * m + 1][0] : t0;
            float p0 = 1.0f, p1 = 0.0f;
            if (m == 2) gate_weights(t0[CSA2_LATENT + CSA2_KEY_DIM], t1[CSA2_LATENT + CSA2_KEY_DIM], p0, p1);
            pack_entry_warp(t0, t1, t0 + CSA2_LATENT, t1 + CSA2_LATENT, m, p0, p1, c, pid,
                            e & (CSA2_PAGE_ENTRIES - 1), lane);
        }
    }
    if (threadIdx.x < 2) s_ent[threadIdx.x] = ((int)threadIdx.x < n_ent) ? e0 + (int)threadIdx.x : -1;
    // Leftover odd token of an m=2 request becomes the pending token.
    bool leftover = (m == 2) && (nt & 1);
    __syncthreads();
    if (leftover) {
        float *pd = c.pending + (size_t)b * CSA2_PENDING_STRIDE;
        for (int j = threadIdx.x; j < W; j += blockDim.x) pd[j] = s_tok[nt - 1][j];
    }
    // Summaries of the blocks that received an entry (entries written above are
    // visible to the whole CTA after the barrier).
    int n_entries_after = (n0 + k) / m;
    if (threadIdx.x < CSA2_KEY_DIM) {
        int blk_a = s_ent[0] >= 0 ? s_ent[0] / CSA2_BLOCK : -1;
        int blk_b = s_ent[1] >= 0 ? s_ent[1] / CSA2_BLOCK : -1;
        if (blk_a >= 0) block_summary(c, b, blk_a, n_entries_after, threadIdx.x);
        if (blk_b >= 0 && blk_b != blk_a) block_summary(c, b, blk_b, n_entries_after, threadIdx.x);
    }
    if (threadIdx.x == 0) c.n_tokens[b] = n0 + k;
}

// ------------------------------------------------------------------ launchers
cudaError_t launch_prefill(const CacheView &c, int req, int m, int tok_begin, int n_tok, int n_tok_final,
                           const float *lat, const float *key, const float *gate, cudaStream_t st)
{
    int tok_end = tok_begin + n_tok;
    int e_first = tok_begin / m;
    int n_ent = tok_end / m - e_first;
    if (n_ent > 0) {
        {
            LaunchScope scope(-1, st);
            prefill_entries_kernel<<<(n_ent + 7) / 8, 256, 0, st>>>(c, req, m, e_first, n_ent, lat, key, gate);
        }
        int b0 = e_first / CSA2_BLOCK, b1 = (e_first + n_ent - 1) / CSA2_BLOCK;
        LaunchScope scope(-1, st);
        prefill_summary_kernel<<<b1 - b0 + 1, 128, 0, st>>>(c, req, b0, e_first + n_ent);
    }
    int t_first = max(tok_begin, n_tok_final - CSA2_SWA);
    int n_swa = max(0, tok_end - t_first);
    int pend_row = (m == 2 && (tok_end & 1) && tok_end == n_tok_final) ? (tok_end - 1 - tok_begin) : -1;
    LaunchScope scope(-1, st);
    prefill_swa_kernel<<<max(1, (n_swa + 7) / 8), 256, 0, st>>>(c, req, tok_begin, t_first, n_swa, lat, key,
                                                               gate, pend_row, tok_end);
    return cudaGetLastError();
}

cudaError_t launch_append(const CacheView &c, const float *lat, const float *key, const float *gate,
                          const int32_t *n_new, cudaStream_t st)
{
    LaunchScope scope(-1, st);
    return launch_pdl(append_kernel, dim3(c.batch), dim3(256), 0, st, c, lat, key, gate, n_new);
}

}  // namespace csa2

// Sparse MQA decode attention over the selected FP4 entries plus the FP8 SWA
// window, split over key chunks (flash-decode), then a log-sum-exp combine.
//
// Sources: daiw.net/manual/deepseek-v4-flash/million-token-cost, decode
// section (attention reads the cached keys every step) and the cache-size
// factor table (one 512-dim KV shared by all query heads: K = V = latent);
// 0539edu.com/news/5732216 §3 (fp4_e2m1 global KV with per-16 e4m3 scales,
// fp8 SWA with a 128-token window).
#include "common.cuh"
#include "index.cuh"

namespace csa2 {

constexpr int AT_KT = ATT_KEYS_PER_SPLIT;   // keys per split (64)
constexpr int AT_HG = 16;                    // heads per CTA
constexpr int AT_VSTRIDE = CSA2_LATENT + 4;  // floats per staged key row
constexpr size_t AT_SMEM = sizeof(float) * ((size_t)AT_KT * AT_VSTRIDE + AT_HG * CSA2_LATENT + AT_HG * AT_KT);

__constant__ float c_e2m1[16] = {0.f, 0.5f, 1.f, 1.5f, 2.f, 3.f, 4.f, 6.f,
                                 -0.f, -0.5f, -1.f, -1.5f, -2.f, -3.f, -4.f, -6.f};

// Grid (splits, head groups, batch); 256 threads.  Split s < 8 covers top-k
// slots 64s..64s+63; splits 8, 9 cover SWA slots 0..63, 64..127.
// Partials: part_ml[b][s][h] = (max logit, sum of exp), part_o[b][s][h][512]
// = sum_j exp(logit_j - max) v_j.
__global__ void __launch_bounds__(256) attend_split_kernel(CacheView c, int heads, const uint16_t *q,
                                                           const int32_t *topk, float scale, float *part_o,
                                                           float *part_ml)
{
    extern __shared__ __align__(16) float smem[];
    float *v_s = smem;                                   // [64][516]
    float *q_s = v_s + AT_KT * AT_VSTRIDE;               // [16][512]
    float *p_s = q_s + AT_HG * CSA2_LATENT;              // [16][64]
    __shared__ int s_valid[AT_KT];
    const int s = blockIdx.x, hg0 = blockIdx.y * AT_HG, b = blockIdx.z;
    const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
    const int n_tok = c.n_tokens[b];
    const int n_entries = n_entries_of(c, b);
    const int nv = min(n_tok, CSA2_SWA);
    const bool is_swa = s >= CSA2_TOPK / AT_KT;

    // q for this head group (zero past `heads`).
    for (int i = tid; i < AT_HG * CSA2_LATENT; i += 256) {
        int h = hg0 + i / CSA2_LATENT;
        q_s[i] = h < heads ? __uint_as_float((uint32_t)q[((size_t)b * heads + h) * CSA2_LATENT + i % CSA2_LATENT] << 16)
                           : 0.0f;
    }
    // Dequantise the 64 keys of this split: warp w handles rows w, w+8, ...;
    // lane l handles channels l + 32i.
    for (int j = w; j < AT_KT; j += 8) {
        float *row = v_s + j * AT_VSTRIDE;
        bool valid = false;
        if (!is_swa) {
            int e = topk[(size_t)b * CSA2_TOPK + s * AT_KT + j];
            if (e >= n_entries) {
                if (lane == 0) set_error(c.error, CSA2_DEV_BAD_INDEX);
            } else if (e >= 0) {
                const uint8_t *pg = entry_page(c, b, e);
                if (pg) {
                    valid = true;
                    int slot = e & (CSA2_PAGE_ENTRIES - 1);
                    const uint8_t *codes = pg + CSA2_PAGE_CODES_OFF + slot * CSA2_CODE_BYTES;
                    const uint8_t *scl = pg + CSA2_PAGE_SCALES_OFF + slot * CSA2_SCALE_BYTES;
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        int ch = lane + 32 * i;
                        uint8_t byte = codes[ch >> 1];
                        uint8_t nib = (ch & 1) ? (byte >> 4) : (byte & 15);
                        row[ch] = c_e2m1[nib] * e4m3_to_f32(scl[ch >> 4]);
                    }
                }
            }
        } else {
            int slot = (s - CSA2_TOPK / AT_KT) * AT_KT + j;
            if (slot < nv) {
                valid = true;
                const uint8_t *sw = swa_base(c, b);
                float sc = reinterpret_cast<const float *>(sw + CSA2_SWA_SCALE_OFF)[slot];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    int ch = lane + 32 * i;
                    row[ch] = e4m3_to_f32(sw[CSA2_SWA_CODES_OFF + slot * CSA2_LATENT + ch]) * sc;
                }
            }
        }
        if (!valid) {
#pragma unroll
            for (int i = 0; i < 16; ++i) row[lane + 32 * i] = 0.0f;
        }
        if (lane == 0) s_valid[j] = valid;
    }
    __syncthreads();

    // Logits: warp w -> heads 2w, 2w+1; lane -> keys lane, lane+32.
    float acc[2][2] = {};
    {
        const float *va = v_s + lane * AT_VSTRIDE, *vb = v_s + (lane + 32) * AT_VSTRIDE;
        const float *qa = q_s + (2 * w) * CSA2_LATENT, *qb = q_s + (2 * w + 1) * CSA2_LATENT;
#pragma unroll 4
        for (int d = 0; d < CSA2_LATENT; d += 4) {
            float4 x = *reinterpret_cast<const float4 *>(va + d);
            float4 y = *reinterpret_cast<const float4 *>(vb + d);
            float4 p = *reinterpret_cast<const float4 *>(qa + d);
            float4 r = *reinterpret_cast<const float4 *>(qb + d);
            acc[0][0] += x.x * p.x + x.y * p.y + x.z * p.z + x.w * p.w;
            acc[0][1] += y.x * p.x + y.y * p.y + y.z * p.z + y.w * p.w;
            acc[1][0] += x.x * r.x + x.y * r.y + x.z * r.z + x.w * r.w;
            acc[1][1] += y.x * r.x + y.y * r.y + y.z * r.z + y.w * r.w;
        }
    }
    const bool va_ok = s_valid[lane], vb_ok = s_valid[lane + 32];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        float la = va_ok ? acc[hh][0] * scale : -INFINITY;
        float lb = vb_ok ? acc[hh][1] * scale : -INFINITY;
        float mx = fmaxf(la, lb);
#pragma unroll
        for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        float pa = va_ok ? expf(la - mx) : 0.0f;
        float pb = vb_ok ? expf(lb - mx) : 0.0f;
        float l = pa + pb;
#pragma unroll
        for (int o = 16; o; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
        p_s[(2 * w + hh) * AT_KT + lane] = pa;
        p_s[(2 * w + hh) * AT_KT + lane + 32] = pb;
        int h = hg0 + 2 * w + hh;
        if (lane == 0 && h < heads) {
            size_t o = (((size_t)b * ATT_SPLITS + s) * heads + h) * 2;
            part_ml[o] = mx;
            part_ml[o + 1] = l;
        }
    }
    __syncthreads();

    // o = P V: warp w -> heads 2w, 2w+1; lane -> channels 4*lane + 128*cc.
    float o[2][16] = {};
    for (int j = 0; j < AT_KT; ++j) {
        float pa = p_s[(2 * w) * AT_KT + j], pb = p_s[(2 * w + 1) * AT_KT + j];
        const float *vr = v_s + j * AT_VSTRIDE;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
            float4 v = *reinterpret_cast<const float4 *>(vr + 4 * lane + 128 * cc);
            o[0][4 * cc + 0] += pa * v.x; o[0][4 * cc + 1] += pa * v.y;
            o[0][4 * cc + 2] += pa * v.z; o[0][4 * cc + 3] += pa * v.w;
            o[1][4 * cc + 0] += pb * v.x; o[1][4 * cc + 1] += pb * v.y;
            o[1][4 * cc + 2] += pb * v.z; o[1][4 * cc + 3] += pb * v.w;
        }
    }
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        int h = hg0 + 2 * w + hh;
        if (h >= heads) continue;
        float *dst = part_o + (((size_t)b * ATT_SPLITS + s) * heads + h) * CSA2_LATENT;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
            *reinterpret_cast<float4 *>(dst + 4 * lane + 128 * cc) =
                make_float4(o[hh][4 * cc], o[hh][4 * cc + 1], o[hh][4 * cc + 2], o[hh][4 * cc + 3]);
    }
}

// Grid (heads, batch); 128 threads, 4 channels each.
__global__ void __launch_bounds__(128) attend_combine_kernel(int heads, const float *part_o, const float *part_ml,
                                                             void *out, int out_is_fp32)
{
    const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
    float m[ATT_SPLITS], M = -INFINITY;
#pragma unroll
    for (int s = 0; s < ATT_SPLITS; ++s) {
        m[s] = part_ml[(((size_t)b * ATT_SPLITS + s) * heads + h) * 2];
        M = fmaxf(M, m[s]);
    }
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float L = 0.0f;
    if (M != -INFINITY) {
#pragma unroll
        for (int s = 0; s < ATT_SPLITS; ++s) {
            if (m[s] == -INFINITY) continue;
            float f = expf(m[s] - M);
            L += f * part_ml[(((size_t)b * ATT_SPLITS + s) * heads + h) * 2 + 1];
            float4 v = *reinterpret_cast<const float4 *>(
                part_o + (((size_t)b * ATT_SPLITS + s) * heads + h) * CSA2_LATENT + 4 * tid);
            acc.x += f * v.x; acc.y += f * v.y; acc.z += f * v.z; acc.w += f * v.w;
        }
        float inv = 1.0f / L;
        acc.x *= inv; acc.y *= inv; acc.z *= inv; acc.w *= inv;
    }
    size_t o = ((size_t)b * heads + h) * CSA2_LATENT + 4 * tid;
    if (out_is_fp32) {
        *reinterpret_cast<float4 *>((float *)out + o) = acc;
    } else {
        __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y), hi = __floats2bfloat162_rn(acc.z, acc.w);
        __nv_bfloat162 *dst = reinterpret_cast<__nv_bfloat162 *>((__nv_bfloat16 *)out + o);
        dst[0] = lo;
        dst[1] = hi;
    }
}

cudaError_t launch_attend(const CacheView &c, int heads, const uint16_t *q, const int32_t *topk, float scale,
                          void *out, int out_is_fp32, float *part_o, float *part_ml, cudaStream_t st)
{
    static bool attr_done[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 64 || !attr_done[dev]) {
        e = cudaFuncSetAttribute(attend_split_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)AT_SMEM);
        if (e != cudaSuccess) return e;
        if (dev < 64) attr_done[dev] = true;
    }
    dim3 g1(ATT_SPLITS, (heads + AT_HG - 1) / AT_HG, c.batch);
    {
        LaunchScope scope(CSA2_KERNEL_ATTEND, st);
        attend_split_kernel<<<g1, 256, AT_SMEM, st>>>(c, heads, q, topk, scale, part_o, part_ml);
    }
    dim3 g2(heads, c.batch);
    {
        LaunchScope scope(CSA2_KERNEL_COMBINE, st);
        attend_combine_kernel<<<g2, 128, 0, st>>>(heads, part_o, part_ml, out, out_is_fp32);
    }
    return cudaGetLastError();
}

}  // namespace csa2

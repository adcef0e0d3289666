// Log-sum-exp combine of the attention partials (one per 128-key tile: four
// top-k tiles and the SWA window, computed in attend_umma.cu) into the
// output, and the attention launcher.
//
// Sources: daiw.net/manual/deepseek-v4-flash/million-token-cost, decode
// section (attention reads the cached keys every step) and the cache-size
// factor table (one 512-dim KV shared by all query heads: K = V = latent);
// 0539edu.com/news/5732216 §3 (fp4_e2m1 global KV with per-16 e4m3 scales,
// fp8 SWA with a 128-token window).
#include "common.cuh"
#include "index.cuh"

namespace csa2 {

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
    cudaError_t e = launch_attend_umma(c, heads, q, topk, scale, part_o, part_ml, st);
    if (e != cudaSuccess) return e;
    dim3 g2(heads, c.batch);
    LaunchScope scope(CSA2_KERNEL_COMBINE, st);
    attend_combine_kernel<<<g2, 128, 0, st>>>(heads, part_o, part_ml, out, out_is_fp32);
    return cudaGetLastError();
}

}  // namespace csa2

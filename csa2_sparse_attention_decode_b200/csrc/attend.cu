// The attention launcher.  The kernel (attend_dsm.cu) computes one partial
// per 128-key tile (four top-k tiles and the SWA window) and merges them in
// the same launch, inside a thread-block cluster; it needs no workspace.
//
// Sources: daiw.net/manual/deepseek-v4-flash/million-token-cost, decode
// section (attention reads the cached keys every step) and the cache-size
// factor table (one 512-dim KV shared by all query heads: K = V = latent);
// 0539edu.com/news/5732216 §3 (fp4_e2m1 global KV with per-16 e4m3 scales,
// fp8 SWA with a 128-token window).
#include "common.cuh"
#include "index.cuh"

namespace csa2 {

cudaError_t launch_attend(const CacheView &c, int heads, const uint16_t *q, const int32_t *topk, float scale,
                          void *out, int out_is_fp32, uint32_t flags, float *part_o, float *part_ml, cudaStream_t st)
{
    (void)part_o;
    (void)part_ml;
    return launch_attend_dsm(c, heads, q, topk, scale, out, out_is_fp32, flags, st);
}

}  // namespace csa2

// Sparse MQA decode attention on the 5th-generation tensor cores.
//
// Sources: daiw.net/manual/deepseek-v4-flash/million-token-cost, decode
// section (each step reads the selected keys) and the cache-size factor table
// (one 512-dim KV shared by all query heads, so K = V = latent);
// 0539edu.com/news/5732216 §3 (fp4_e2m1 global KV with an e4m3 scale per 16
// channels; fp8 SWA with a 128-token window).
//
// One CTA per (request, 128-key tile, 64-head group); tiles 0-3 are the
// top-512 entries, tile 4 the SWA window.  256 threads; threads i and i+128
// share key row i (each half of its channels / heads) while loading and
// tensor-memory row i afterwards.
//   1. q (bf16, 64 heads x 512) -> smem, K-major, 128-byte swizzle.
//   2. gather + dequantise 128 keys to bf16 (exact: e2m1 x e4m3 and
//      e4m3 x 2^e all fit bf16) -> smem V tile, K-major, swizzled.
//   3. S^T[128 keys x 64 heads] = V . Q^T           (32 MMAs, fp32 in TMEM)
//   4. softmax over the tile's keys per head (max and sum through a smem
//      transpose); P = exp(scale*S - m) is split into bf16 hi + lo parts so
//      the second product keeps ~16 bits of P.
//   5. O^T[512 x 64] = V^T . (P_hi + P_lo)^T       (4 x 16 MMAs; V reused as
//      an MN-major operand, P as MN-major [key][head])
//   6. the five tiles of a (request, head group) form one thread-block
//      cluster: they exchange the per-head max m and sum l over distributed
//      shared memory, write their partial o scaled by exp(m_tile - M) / L to
//      the workspace, and each CTA then sums one fifth of the output.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "index.cuh"
#include "umma.cuh"

#include <cooperative_groups.h>
namespace cg = cooperative_groups;

namespace csa2 {
using namespace umma;

namespace {

constexpr int KT = 128;                    // keys per tile
constexpr int HG = 64;                     // heads per CTA
constexpr int THREADS = 256;
constexpr int NTILES = ATT_SPLITS;         // 4 top-k tiles + the window = one cluster
constexpr int V_SLAB = KT * 128;           // 16 KB: 128 rows x 64 bf16
constexpr int V_BYTES = 8 * V_SLAB;        // 128 KB
constexpr int Q_SLAB = HG * 128;           // 8 KB
constexpr int Q_BYTES = 8 * Q_SLAB;        // 64 KB
constexpr int T_STRIDE = HG + 1;           // fp32 transpose row stride
constexpr size_t SMEM_BYTES = 1024 + V_BYTES + Q_BYTES + 4096;
// After the first product the q region (plus 4 KB) is reused: transpose
// [128][65] fp32 at +0 (33,280 B), P_hi at +36 KB, P_lo at +52 KB (both
// 1024-aligned; P_lo ends at +68 KB).
constexpr int T_OFF = 0, PHI_OFF = 36 * 1024, PLO_OFF = 52 * 1024;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t S_COL = 0, O_COL = 64;
constexpr uint32_t IDESC_S = idesc_f16(128, HG, true, false, false);
constexpr uint32_t IDESC_O = idesc_f16(128, HG, true, true, true);

// bf16 bits of the 8 e2m1 magnitudes (0, .5, 1, 1.5, 2, 3, 4, 6), split into
// low and high bytes for byte-permute lookups.
constexpr uint32_t E2M1_LO_A = 0xC0800000u, E2M1_LO_B = 0xC0804000u;   // codes 0-3, 4-7
constexpr uint32_t E2M1_HI_A = 0x3F3F3F00u, E2M1_HI_B = 0x40404040u;

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel)
{
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

// 8 e2m1 codes (one 32-bit word; channel c in bits 4c..4c+3) -> 8 bf16
// values as 4 bf16x2 words (channels 2i, 2i+1 in word i).  The 3-bit
// magnitude selects the low and high byte of the bf16 pattern from two
// 8-entry byte tables; the sign bit moves to bit 15.
__device__ __forceinline__ void e2m1x8_to_bf16(uint32_t w, uint32_t (&o)[4])
{
    const uint32_t sel_even = (w & 7u) | ((w >> 8 & 7u) << 4) | ((w >> 16 & 7u) << 8) | ((w >> 24 & 7u) << 12);
    const uint32_t sel_odd = (w >> 4 & 7u) | ((w >> 12 & 7u) << 4) | ((w >> 20 & 7u) << 8) | ((w >> 28 & 7u) << 12);
    const uint32_t le = prmt(E2M1_LO_A, E2M1_LO_B, sel_even), he = prmt(E2M1_HI_A, E2M1_HI_B, sel_even);
    const uint32_t lod = prmt(E2M1_LO_A, E2M1_LO_B, sel_odd), hod = prmt(E2M1_HI_A, E2M1_HI_B, sel_odd);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t ev = ((he >> (8 * i) & 0xffu) << 8) | (le >> (8 * i) & 0xffu);
        uint32_t od = ((hod >> (8 * i) & 0xffu) << 8) | (lod >> (8 * i) & 0xffu);
        ev |= (w >> (8 * i) & 0x8u) << 12;           // sign of channel 2i   -> bit 15
        od |= (w >> (8 * i) & 0x80u) << 8;           // sign of channel 2i+1 -> bit 15
        o[i] = ev | (od << 16);
    }
}

__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b)
{
    __nv_bfloat162 x = *reinterpret_cast<__nv_bfloat162 *>(&a), y = *reinterpret_cast<__nv_bfloat162 *>(&b);
    __nv_bfloat162 r = __hmul2(x, y);
    return *reinterpret_cast<uint32_t *>(&r);
}

__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, int32_t *err)
{
    if (mbar_wait(bar, parity)) return true;
    set_error(err, CSA2_DEV_TIMEOUT);
    return false;
}

__global__ void __cluster_dims__(NTILES, 1, 1) __launch_bounds__(THREADS, 1)
attend_umma_kernel(const __grid_constant__ CUtensorMap map_q, CacheView c, int heads, const int32_t *topk, float scale,
                   void *out, int out_is_fp32, uint32_t flags, float *part_o)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t *Vs = sm, *Qs = sm + V_BYTES;
    float *Ts = reinterpret_cast<float *>(Qs + T_OFF);
    __shared__ __align__(8) uint64_t bar_q, bar_s, bar_o;
    __shared__ uint32_t tmem_base;
    __shared__ float m_s[HG], l_s[HG], fac_s[HG], red_s[4][HG];
    __shared__ int tile_live[NTILES];
    cg::cluster_group cluster = cg::this_cluster();

    const int tile = blockIdx.x, hg0 = blockIdx.y * HG, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int row = tid & (KT - 1), half = tid >> 7;      // two threads per key / tensor-memory row
    if (warp == 0) tmem_alloc(&tmem_base, TMEM_COLS);
    if (tid == 32) tma_prefetch_map(&map_q);
    const bool early = (flags & CSA2_ATTEND_INPUTS_SETTLED) != 0;
    bool valid = false;
    // ---- 2. key `row`, channels [256*half, 256*half + 256) -> bf16 in slabs 4*half .. 4*half+3
    auto gather = [&]() {
        const int n_tok = c.n_tokens[b];
        const int n_entries = n_entries_of(c, b);
        const int nv = max(0, min(n_tok, CSA2_SWA));
        if (tile < CSA2_TOPK / KT) {
            const int e = topk[(size_t)b * CSA2_TOPK + tile * KT + row];
            if (e >= n_entries && half == 0) set_error(c.error, CSA2_DEV_BAD_INDEX);
            const int pid = (e >= 0 && e < n_entries) ? entry_pid(c, b, e) : -1;
            if (pid >= 0) {
                valid = true;
                const int slot = e & (CSA2_PAGE_ENTRIES - 1);
                const uint4 *codes = reinterpret_cast<const uint4 *>(codes_row(c, pid, slot)) + 8 * half;
                const uint4 sv = reinterpret_cast<const uint4 *>(scales_row(c, pid, slot))[half];
                uint4 cw[8];                               // 128 code bytes, loads issued together
    #pragma unroll
                for (int i = 0; i < 8; ++i) cw[i] = codes[i];
                const uint32_t sw[4] = {sv.x, sv.y, sv.z, sv.w};
    #pragma unroll
                for (int s4 = 0; s4 < 4; ++s4) {
                    const int slab = 4 * half + s4;
                    const uint32_t cwu[8] = {cw[2 * s4].x,     cw[2 * s4].y,     cw[2 * s4].z,     cw[2 * s4].w,
                                             cw[2 * s4 + 1].x, cw[2 * s4 + 1].y, cw[2 * s4 + 1].z, cw[2 * s4 + 1].w};
    #pragma unroll
                    for (int ch = 0; ch < 8; ++ch) {                                  // 8 channels per chunk
                        uint32_t o[4];
                        e2m1x8_to_bf16(cwu[ch], o);
                        // channels slab*64 + ch*8 .. +7 share scale byte slab*4 + ch/2
                        const int si = s4 * 4 + (ch >> 1);
                        const float sf = e4m3_to_f32((uint8_t)(sw[si >> 2] >> (8 * (si & 3))));
                        const uint32_t s2 = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(sf)) * 0x10001u;
    #pragma unroll
                        for (int i = 0; i < 4; ++i) o[i] = bf16x2_mul(o[i], s2);
                        *reinterpret_cast<uint4 *>(Vs + slab * V_SLAB + row * 128 + ((ch ^ (row & 7)) << 4)) =
                            make_uint4(o[0], o[1], o[2], o[3]);
                    }
                }
            }
        } else if (row < nv) {
            valid = true;
            const uint8_t *swa = swa_base(c, b);
            const float sc = reinterpret_cast<const float *>(swa + CSA2_SWA_SCALE_OFF)[row];
            const uint4 *codes = reinterpret_cast<const uint4 *>(swa + CSA2_SWA_CODES_OFF + row * CSA2_LATENT) + 16 * half;
            uint4 cv[16];
    #pragma unroll
            for (int i = 0; i < 16; ++i) cv[i] = codes[i];
    #pragma unroll
            for (int k = 0; k < 16; ++k) {                                          // 16 codes -> 2 chunks
                const int slab = 4 * half + (k >> 2), ch0 = 2 * (k & 3);
                const uint32_t cw[4] = {cv[k].x, cv[k].y, cv[k].z, cv[k].w};
                uint32_t o[8];
    #pragma unroll
                for (int i = 0; i < 4; ++i) {
                    __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(cw[i] & 0xffff), __NV_E4M3);
                    __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(cw[i] >> 16), __NV_E4M3);
                    __nv_bfloat162 a = __floats2bfloat162_rn(__half2float(__ushort_as_half(lo.x)) * sc,
                                                             __half2float(__ushort_as_half(lo.y)) * sc);
                    __nv_bfloat162 bq = __floats2bfloat162_rn(__half2float(__ushort_as_half(hi.x)) * sc,
                                                              __half2float(__ushort_as_half(hi.y)) * sc);
                    o[2 * i] = *reinterpret_cast<uint32_t *>(&a);
                    o[2 * i + 1] = *reinterpret_cast<uint32_t *>(&bq);
                }
                *reinterpret_cast<uint4 *>(Vs + slab * V_SLAB + row * 128 + ((ch0 ^ (row & 7)) << 4)) =
                    make_uint4(o[0], o[1], o[2], o[3]);
                *reinterpret_cast<uint4 *>(Vs + slab * V_SLAB + row * 128 + (((ch0 + 1) ^ (row & 7)) << 4)) =
                    make_uint4(o[4], o[5], o[6], o[7]);
            }
        }
        if (!valid) {
            for (int s4 = 0; s4 < 4; ++s4)
                for (int ch = 0; ch < 8; ++ch)
                    *reinterpret_cast<uint4 *>(Vs + (4 * half + s4) * V_SLAB + row * 128 + (ch << 4)) =
                        make_uint4(0, 0, 0, 0);
        }
    };
    if (early) gather();                                  // inputs settled: overlap the previous kernel
    grid_dependency_wait();                               // q (and, unless settled, the rest) may be fresh
    allow_dependents();
    const int nh = min(HG, heads - hg0);
    if (tid == 0) {
        mbar_init(&bar_q, 1);
        mbar_init(&bar_s, 1);
        mbar_init(&bar_o, 1);
        mbar_fence_init();
        // ---- 1. q -> smem by TMA: 8 boxes of 64 dims x 64 heads, 128-byte
        // swizzled (K-major operand layout); heads past `heads` read as zero.
        mbar_arrive_expect_tx(&bar_q, Q_BYTES);
        for (int slab = 0; slab < 8; ++slab) tma_load_3d(Qs + slab * Q_SLAB, &map_q, 64 * slab, hg0, b, &bar_q);
    }
    if (!early) gather();
    fence_proxy_async_smem();
    const bool live = __syncthreads_or(valid) != 0;      // any valid key in this tile
    fence_after_sync();
    const uint32_t tb = tmem_base;
    const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;

    if (live) {
        // ---- 3. S^T = V . Q^T
        if (tid == 0) {
            wait_bar(&bar_q, 0, c.error);
            const uint32_t va = smem_addr(Vs), qa = smem_addr(Qs);
#pragma unroll 4
            for (int kk = 0; kk < CSA2_LATENT / 16; ++kk) {
                const uint32_t off = (kk >> 2), in = (kk & 3) * 32;
                mma_ss(tb + S_COL, smem_desc(va + off * V_SLAB + in, 16, 1024),
                       smem_desc(qa + off * Q_SLAB + in, 16, 1024), IDESC_S, kk > 0 ? 1u : 0u);
            }
            mma_commit(&bar_s);
        }
        __syncwarp();
        wait_bar(&bar_s, 0, c.error);
        fence_after_sync();

        // ---- 4. softmax over the tile's keys, per head (thread: key `row`, heads 32*half ..)
        float lg[32];
        {
            uint32_t rr[32];
            tmem_ld32(tb + lane_base + S_COL + 32 * half, rr);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 32; ++j) lg[j] = valid ? __uint_as_float(rr[j]) * scale : -INFINITY;
        }
        // the q region is free from here on (the product above has completed)
#pragma unroll
        for (int j = 0; j < 32; ++j) Ts[row * T_STRIDE + 32 * half + j] = lg[j];
        __syncthreads();
        {
            const int h = tid & (HG - 1), part = tid >> 6;
            float mx = -INFINITY;
            for (int j = part * 32; j < part * 32 + 32; ++j) mx = fmaxf(mx, Ts[j * T_STRIDE + h]);
            red_s[part][h] = mx;
        }
        __syncthreads();
        if (tid < HG) m_s[tid] = fmaxf(fmaxf(red_s[0][tid], red_s[1][tid]), fmaxf(red_s[2][tid], red_s[3][tid]));
        __syncthreads();
        uint8_t *Ph = Qs + PHI_OFF, *Pl = Qs + PLO_OFF;
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
            const int cch = 4 * half + c4;                 // 8-head chunk of the P row
            uint32_t hi[4], lo[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int j0 = 8 * c4 + 2 * i, h0 = 32 * half + j0;
                const float p0 = valid ? __expf(lg[j0] - m_s[h0]) : 0.0f;
                const float p1 = valid ? __expf(lg[j0 + 1] - m_s[h0 + 1]) : 0.0f;
                Ts[row * T_STRIDE + h0] = p0;
                Ts[row * T_STRIDE + h0 + 1] = p1;
                const __nv_bfloat162 ph = __floats2bfloat162_rn(p0, p1);
                const float2 phf = __bfloat1622float2(ph);
                const __nv_bfloat162 pl = __floats2bfloat162_rn(p0 - phf.x, p1 - phf.y);
                hi[i] = *reinterpret_cast<const uint32_t *>(&ph);
                lo[i] = *reinterpret_cast<const uint32_t *>(&pl);
            }
            const uint32_t off = row * 128 + ((cch ^ (row & 7)) << 4);
            *reinterpret_cast<uint4 *>(Ph + off) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
            *reinterpret_cast<uint4 *>(Pl + off) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
        fence_proxy_async_smem();
        __syncthreads();
        fence_after_sync();
        // ---- 5. O^T = V^T . P^T (hi, then lo)
        if (tid == 0) {
            const uint32_t va = smem_addr(Vs), ph = smem_addr(Ph), pl = smem_addr(Pl);
            for (int cc = 0; cc < 4; ++cc) {
                for (int part = 0; part < 2; ++part) {
                    const uint32_t pb = part ? pl : ph;
#pragma unroll
                    for (int kk = 0; kk < KT / 16; ++kk) {
                        const uint64_t ad = smem_desc(va + (2 * cc) * V_SLAB + kk * 2048, V_SLAB, 1024);
                        const uint64_t bd = smem_desc(pb + kk * 2048, 8192, 1024);
                        mma_ss(tb + O_COL + 64 * cc, ad, bd, IDESC_O, (part | kk) ? 1u : 0u);
                    }
                }
            }
            mma_commit(&bar_o);
        }
        __syncwarp();
        // row sums of P per head while the MMAs run
        {
            const int h = tid & (HG - 1), part = tid >> 6;
            float sum = 0.0f;
            for (int j = part * 32; j < part * 32 + 32; ++j) sum += Ts[j * T_STRIDE + h];
            red_s[part][h] = sum;
        }
        __syncthreads();
        if (tid < HG) l_s[tid] = (red_s[0][tid] + red_s[1][tid]) + (red_s[2][tid] + red_s[3][tid]);
    } else {
        if (tid == 0) wait_bar(&bar_q, 0, c.error);          // no copy may be in flight at exit
        if (tid < HG) {
            m_s[tid] = -INFINITY;
            l_s[tid] = 0.0f;
        }
    }
    // ---- 6. combine the five tiles of this (request, head group) in-cluster:
    // exchange (m, l) over distributed shared memory; each tile writes its
    // partial already scaled by exp(m_tile - M) / L; then each CTA sums one
    // fifth of the output over the live tiles.
    cluster.sync();
    if (tid < HG) {
        float mr[NTILES], M = -INFINITY;
#pragma unroll
        for (int r = 0; r < NTILES; ++r) {
            mr[r] = cluster.map_shared_rank(&m_s[0], r)[tid];
            M = fmaxf(M, mr[r]);
        }
        float L = 0.0f;
#pragma unroll
        for (int r = 0; r < NTILES; ++r)
            if (mr[r] != -INFINITY) L += __expf(mr[r] - M) * cluster.map_shared_rank(&l_s[0], r)[tid];
        fac_s[tid] = (live && M != -INFINITY && L > 0.0f) ? __expf(m_s[tid] - M) / L : 0.0f;
        if (tid < NTILES) tile_live[tid] = cluster.map_shared_rank(&m_s[0], tid)[0] != -INFINITY;
    }
    __syncthreads();
    if (live) {
        wait_bar(&bar_o, 0, c.error);
        fence_after_sync();
        for (int cc = 0; cc < 4; ++cc) {
            uint32_t rr[32];
            tmem_ld32(tb + lane_base + O_COL + 64 * cc + 32 * half, rr);
            tmem_ld_wait();
            const int d = 128 * cc + row;
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int h = 32 * half + j;
                if (h < nh)
                    part_o[(((size_t)b * NTILES + tile) * heads + hg0 + h) * CSA2_LATENT + d] =
                        __uint_as_float(rr[j]) * fac_s[h];
            }
        }
    }
    cluster.sync();                                       // partials visible cluster-wide
    {
        const int total4 = HG * (CSA2_LATENT / 4);
        const int lo4 = tile * total4 / NTILES, hi4 = (tile + 1) * total4 / NTILES;
        for (int i = lo4 + tid; i < hi4; i += THREADS) {
            const int h = i / (CSA2_LATENT / 4), d4 = i % (CSA2_LATENT / 4);
            if (h >= nh) continue;
            float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int r = 0; r < NTILES; ++r) {
                if (!tile_live[r]) continue;
                const float4 v = *reinterpret_cast<const float4 *>(
                    part_o + (((size_t)b * NTILES + r) * heads + hg0 + h) * CSA2_LATENT + 4 * d4);
                acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
            }
            const size_t o = ((size_t)b * heads + hg0 + h) * CSA2_LATENT + 4 * d4;
            if (out_is_fp32) {
                *reinterpret_cast<float4 *>((float *)out + o) = acc;
            } else {
                __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y), hi = __floats2bfloat162_rn(acc.z, acc.w);
                uint2 pk = make_uint2(*reinterpret_cast<uint32_t *>(&lo), *reinterpret_cast<uint32_t *>(&hi));
                *reinterpret_cast<uint2 *>((__nv_bfloat16 *)out + o) = pk;
            }
        }
    }
    fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        fence_after_sync();
        tmem_dealloc(tb, TMEM_COLS);
    }
}

// q viewed as a 3-D bf16 tensor (512 dims, heads, batch); boxes of 64 dims x
// 64 heads, 128-byte swizzled.
bool make_q_map(CUtensorMap *m, const uint16_t *q, int heads, int batch)
{
    auto fn = tensor_map_encoder();
    if (!fn) return false;
    cuuint64_t dims[3] = {CSA2_LATENT, (cuuint64_t)heads, (cuuint64_t)batch};
    cuuint64_t strides[2] = {CSA2_LATENT * 2, (cuuint64_t)heads * CSA2_LATENT * 2};
    cuuint32_t box[3] = {64, HG, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, (void *)q, dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_attend_umma(const CacheView &c, int heads, const uint16_t *q, const int32_t *topk, float scale,
                               void *out, int out_is_fp32, uint32_t flags, float *part_o, cudaStream_t st)
{
    static DeviceOnce once;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess)
        e = once.run(dev, [] {
            return cudaFuncSetAttribute(attend_umma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        (int)SMEM_BYTES);
        });
    if (e != cudaSuccess) return e;
    CUtensorMap map_q;
    if (!make_q_map(&map_q, q, heads, c.batch)) return cudaErrorInvalidValue;
    dim3 grid(NTILES, (heads + HG - 1) / HG, c.batch);
    LaunchScope scope(CSA2_KERNEL_ATTEND, st);
    return launch_pdl(attend_umma_kernel, grid, dim3(THREADS), SMEM_BYTES, st, map_q, c, heads, topk, scale, out,
                      out_is_fp32, flags, part_o);
}

}  // namespace csa2

// Sparse MQA decode attention on the 5th-generation tensor cores, split over
// 128-key tiles and merged inside a thread-block cluster through distributed
// shared memory.
//
// Sources: daiw.net/manual/deepseek-v4-flash/million-token-cost, decode
// section (each step reads the selected keys) and the cache-size factor table
// (one 512-dim KV shared by all query heads, so K = V = latent);
// 0539edu.com/news/5732216 §3 (fp4_e2m1 global KV with an e4m3 scale per 16
// channels; fp8 SWA with a 128-token window).
//
// Grid (5 tiles, ceil(heads / 16) head groups, batch); the five tiles of one
// (request, head group) form a cluster.  Tiles 0-3 are the top-512 entries,
// tile 4 the SWA window.  512 threads: while gathering, thread t owns key row
// t & 127 and a quarter (t >> 7) of its 512 channels.
//   1. q (bf16, 16 heads x 512) -> smem by TMA, K-major, 128-byte swizzle.
//   2. gather + dequantise 128 keys to bf16 (exact: e2m1 x e4m3 and
//      e4m3 x 2^e all fit bf16) -> smem V tile, K-major, swizzled.
//   3. S^T[128 keys x 16 heads] = V . Q^T            (32 MMAs, fp32 in TMEM)
//   4. softmax per head over the tile's keys through a smem transpose;
//      P = exp(scale*S - m) is split into bf16 hi + lo parts (the second
//      product keeps ~16 bits of P), stored K-major as [head][key].
//   5. O^T[512 x 16] = V^T . (P_hi + P_lo)^T        (4 dim chunks x 2 x 8
//      MMAs; the V tile is read again as an MN-major operand)
//   6. merge: each live tile writes its partial O into its own shared
//      memory beside its per-head max m and sum l; after one cluster barrier
//      each CTA reads every tile's (m, l), forms the weights exp(m - M) / L
//      and sums one fifth of the output over the live tiles, reading their
//      buffers remotely.
// Partial mode (sequence-sharded decode): ATT_NO_WINDOW leaves the window
// tile empty, and `lse` receives ln sum_j exp(scale * q.v_j) per head.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <cooperative_groups.h>

#include "common.cuh"
#include "index.cuh"
#include "umma.cuh"

namespace cg = cooperative_groups;

namespace csa2 {
using namespace umma;

namespace {

constexpr int KT = 128;                     // keys per tile
constexpr int THREADS = 512;
constexpr int NTILES = ATT_SPLITS;          // 4 top-k tiles + the window = one cluster
constexpr int V_SLAB = KT * 128;            // 16 KB: 128 keys x 64 dims (bf16)
constexpr int V_BYTES = 8 * V_SLAB;         // 128 KB
constexpr uint32_t S_COL = 0, O_COL = 32;   // S^T: HG columns; O^T: 4 chunks x HG columns

// Sizes for HG heads per CTA (16 or 32).
template <int HG>
struct Cfg {
    static_assert(HG == 16 || HG == 32, "head group of 16 or 32");
    static constexpr int KC = THREADS / HG;            // softmax: chunks of KPT keys per head
    static constexpr int KPT = KT / KC;                // keys per softmax thread (4 or 8)
    static constexpr int SCOLS = HG / 4;               // S^T columns each warp moves to the transpose
    static constexpr int Q_SLAB = HG * 128;            // HG heads x 64 dims
    static constexpr int Q_BYTES = 8 * Q_SLAB;
    static constexpr int P_SLAB = HG * 128;            // HG heads x 64 keys
    static constexpr int P_BYTES = 2 * P_SLAB;
    static constexpr int T_STRIDE = HG + 1;            // fp32 transpose row stride
    static constexpr int T_BYTES = KT * T_STRIDE * 4;
    static constexpr int Q_OFF = V_BYTES, PHI_OFF = Q_OFF + Q_BYTES, PLO_OFF = PHI_OFF + P_BYTES,
                         T_OFF = PLO_OFF + P_BYTES;
    static constexpr size_t SMEM_BYTES = 1024 + T_OFF + T_BYTES;
    // The merge buffer [head][dim] (fp32) reuses the V tile once the second
    // product has completed.
    static_assert(HG * CSA2_LATENT * 4 <= V_BYTES, "merge buffer must fit the V tile");
    static constexpr uint32_t TMEM_COLS = (O_COL + 4 * HG <= 128) ? 128 : 256;
    static constexpr uint32_t IDESC_S = idesc_f16(128, HG, true, false, false);
    static constexpr uint32_t IDESC_O = idesc_f16(128, HG, true, true, false);
};

// Low and high bytes of the bf16 patterns of the 8 e2m1 magnitudes (0, .5,
// 1, 1.5, 2, 3, 4, 6) as byte-permute tables: codes 0-3 in A, 4-7 in B.
constexpr uint32_t E2M1_LO_A = 0xC0800000u, E2M1_LO_B = 0xC0804000u;
constexpr uint32_t E2M1_HI_A = 0x3F3F3F00u, E2M1_HI_B = 0x40404040u;

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel)
{
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

// 8 e2m1 codes (channel c in bits 4c..4c+3) -> 4 bf16x2 words, word i =
// channels 2i (low half) and 2i+1 (high half).  Even and odd channels are
// looked up separately: the four 3-bit magnitudes of a group become one
// byte-permute selector, and each channel's sign bit then sits exactly where
// bit 7 of its high byte goes (a shift of 4 for even channels, 0 for odd).
__device__ __forceinline__ void e2m1x8_to_bf16(uint32_t w, uint32_t (&o)[4])
{
    const uint32_t xe = w & 0x07070707u, xo = (w >> 4) & 0x07070707u;
    const uint32_t se = prmt(xe | (xe >> 4), 0u, 0x4420u);     // selector nibbles: channels 0, 2, 4, 6
    const uint32_t so = prmt(xo | (xo >> 4), 0u, 0x4420u);     // channels 1, 3, 5, 7
    const uint32_t le = prmt(E2M1_LO_A, E2M1_LO_B, se);
    const uint32_t he = prmt(E2M1_HI_A, E2M1_HI_B, se) | ((w << 4) & 0x80808080u);
    const uint32_t lo = prmt(E2M1_LO_A, E2M1_LO_B, so);
    const uint32_t ho = prmt(E2M1_HI_A, E2M1_HI_B, so) | (w & 0x80808080u);
    const uint32_t a = prmt(le, he, 0x5140u), bq = prmt(le, he, 0x7362u);   // [lo, hi] of channels 0,2 | 4,6
    const uint32_t c = prmt(lo, ho, 0x5140u), d = prmt(lo, ho, 0x7362u);    // channels 1,3 | 5,7
    o[0] = prmt(a, c, 0x5410u);
    o[1] = prmt(a, c, 0x7632u);
    o[2] = prmt(bq, d, 0x5410u);
    o[3] = prmt(bq, d, 0x7632u);
}

__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b)
{
    __nv_bfloat162 x = *reinterpret_cast<__nv_bfloat162 *>(&a), y = *reinterpret_cast<__nv_bfloat162 *>(&b);
    __nv_bfloat162 r = __hmul2(x, y);
    return *reinterpret_cast<uint32_t *>(&r);
}

// Tensor-memory load of as many columns as the array holds.
template <int N>
__device__ __forceinline__ void ld_cols(uint32_t a, uint32_t (&r)[N])
{
    if constexpr (N == 4) tmem_ld4(a, r);
    else if constexpr (N == 8) tmem_ld8(a, r);
    else if constexpr (N == 16) tmem_ld16(a, r);
    else tmem_ld32(a, r);
}
// 2 or 4 packed bf16 pairs to shared memory.
template <int N>
__device__ __forceinline__ void st_pairs(uint8_t *p, const uint32_t (&v)[N])
{
    if constexpr (N == 2) *reinterpret_cast<uint2 *>(p) = make_uint2(v[0], v[1]);
    else *reinterpret_cast<uint4 *>(p) = make_uint4(v[0], v[1], v[2], v[3]);
}

__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, int32_t *err)
{
    if (mbar_wait(bar, parity)) return true;
    set_error(err, CSA2_DEV_TIMEOUT);
    return false;
}

template <int HG>
__global__ void __cluster_dims__(NTILES, 1, 1) __launch_bounds__(THREADS, 1)
attend_dsm_kernel(const __grid_constant__ CUtensorMap map_q, CacheView c, int heads, const int32_t *topk, float scale,
                  void *out, int out_is_fp32, uint32_t flags, float *lse)
{
    using C = Cfg<HG>;
    constexpr int KC = C::KC, KPT = C::KPT, SCOLS = C::SCOLS, Q_SLAB = C::Q_SLAB, Q_BYTES = C::Q_BYTES;
    constexpr int P_SLAB = C::P_SLAB, T_STRIDE = C::T_STRIDE;
    constexpr uint32_t TMEM_COLS = C::TMEM_COLS, IDESC_S = C::IDESC_S, IDESC_O = C::IDESC_O;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t *Vs = sm, *Qs = sm + C::Q_OFF, *Ph = sm + C::PHI_OFF, *Pl = sm + C::PLO_OFF;
    float *Ts = reinterpret_cast<float *>(sm + C::T_OFF);
    float *Ob = reinterpret_cast<float *>(Vs);
    __shared__ __align__(8) uint64_t bar_q, bar_s, bar_o;
    __shared__ uint32_t tmem_base;
    __shared__ float m_s[HG], l_s[HG], red_m[KC][HG], red_l[KC][HG];
    __shared__ float mt_s[NTILES][HG], lt_s[NTILES][HG], fac_s[NTILES][HG];   // every tile's (m, l), weights
    __shared__ int tile_live[NTILES];
    cg::cluster_group cluster = cg::this_cluster();

    const int tile = blockIdx.x, hg0 = blockIdx.y * HG, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int row = tid & (KT - 1), qtr = tid >> 7;     // gather: key row, quarter of its channels
    if (warp == 0) {
        tmem_alloc(&tmem_base, TMEM_COLS);
        fence_before_sync();
    }
    if (tid == 32) tma_prefetch_map(&map_q);
    const bool early = (flags & CSA2_ATTEND_INPUTS_SETTLED) != 0;
    bool valid = false;
    // ---- 2. key `row`, channels [128*qtr, 128*qtr + 128) -> slabs 2*qtr, 2*qtr + 1
    auto gather = [&]() {
        const int n_tok = c.n_tokens[b];
        const int n_entries = n_entries_of(c, b);
        const int nv = (flags & ATT_NO_WINDOW) ? 0 : max(0, min(n_tok, CSA2_SWA));
        uint8_t *vrow = Vs + (2 * qtr) * V_SLAB + row * 128;
        const int sw = row & 7;
        if (tile < CSA2_TOPK / KT) {
            const int e = topk[(size_t)b * CSA2_TOPK + tile * KT + row];
            if (e >= n_entries && qtr == 0) set_error(c.error, CSA2_DEV_BAD_INDEX);
            const int pid = (e >= 0 && e < n_entries) ? entry_pid(c, b, e) : -1;
            if (pid >= 0) {
                valid = true;
                const int slot = e & (CSA2_PAGE_ENTRIES - 1);
                const uint4 *codes = reinterpret_cast<const uint4 *>(codes_row(c, pid, slot)) + 4 * qtr;
                const uint2 sv = reinterpret_cast<const uint2 *>(scales_row(c, pid, slot))[qtr];
                uint4 cw[4];                                   // 64 code bytes, loads issued together
#pragma unroll
                for (int i = 0; i < 4; ++i) cw[i] = codes[i];
                uint32_t s2[8];                                // scale of channels 16j.. as bf16x2
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const uint32_t byte = ((j < 4 ? sv.x : sv.y) >> (8 * (j & 3))) & 0xffu;
                    s2[j] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(e4m3_to_f32((uint8_t)byte))) * 0x10001u;
                }
#pragma unroll
                for (int k = 0; k < 16; ++k) {                 // word k: channels 128*qtr + 8k .. +7
                    const uint4 &v4 = cw[k >> 2];
                    const uint32_t wd = (k & 3) == 0 ? v4.x : (k & 3) == 1 ? v4.y : (k & 3) == 2 ? v4.z : v4.w;
                    uint32_t o[4];
                    e2m1x8_to_bf16(wd, o);
#pragma unroll
                    for (int i = 0; i < 4; ++i) o[i] = bf16x2_mul(o[i], s2[k >> 1]);
                    *reinterpret_cast<uint4 *>(vrow + (k >> 3) * V_SLAB + (((k & 7) ^ sw) << 4)) =
                        make_uint4(o[0], o[1], o[2], o[3]);
                }
            }
        } else if (row < nv) {
            valid = true;
            const uint8_t *swa = swa_base(c, b);
            const float sc = reinterpret_cast<const float *>(swa + CSA2_SWA_SCALE_OFF)[row];
            const uint4 *codes =
                reinterpret_cast<const uint4 *>(swa + CSA2_SWA_CODES_OFF + row * CSA2_LATENT) + 8 * qtr;
            uint4 cv[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) cv[i] = codes[i];
#pragma unroll
            for (int k = 0; k < 8; ++k) {                      // 16 channels: 128*qtr + 16k .. +15
                const uint32_t cw[4] = {cv[k].x, cv[k].y, cv[k].z, cv[k].w};
                uint32_t o[8];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    __half2_raw lo = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(cw[i] & 0xffff), __NV_E4M3);
                    __half2_raw hi = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(cw[i] >> 16), __NV_E4M3);
                    __nv_bfloat162 x = __floats2bfloat162_rn(__half2float(__ushort_as_half(lo.x)) * sc,
                                                             __half2float(__ushort_as_half(lo.y)) * sc);
                    __nv_bfloat162 y = __floats2bfloat162_rn(__half2float(__ushort_as_half(hi.x)) * sc,
                                                             __half2float(__ushort_as_half(hi.y)) * sc);
                    o[2 * i] = *reinterpret_cast<uint32_t *>(&x);
                    o[2 * i + 1] = *reinterpret_cast<uint32_t *>(&y);
                }
                uint8_t *dst = vrow + (k >> 2) * V_SLAB;
                const int ch0 = 2 * (k & 3);
                *reinterpret_cast<uint4 *>(dst + ((ch0 ^ sw) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
                *reinterpret_cast<uint4 *>(dst + (((ch0 + 1) ^ sw) << 4)) = make_uint4(o[4], o[5], o[6], o[7]);
            }
        }
        if (!valid) {
#pragma unroll
            for (int s = 0; s < 2; ++s)
#pragma unroll
                for (int ch = 0; ch < 8; ++ch)
                    *reinterpret_cast<uint4 *>(vrow + s * V_SLAB + (ch << 4)) = make_uint4(0, 0, 0, 0);
        }
    };
    if (early) gather();                                  // inputs settled: overlap the previous kernel
    grid_dependency_wait();                               // q (and, unless settled, the rest) may be fresh
    allow_dependents();
    const int nh = min(HG, heads - hg0);
    if (tid == 0) {
        mbar_init(&bar_q, 1);
        mbar_init(&bar_s, 1);
        mbar_init(&bar_o, 4);                                // one commit per issuing warp
        mbar_fence_init();
        // ---- 1. q -> smem by TMA: 8 boxes of 64 dims x HG heads, 128-byte
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
    const int h = tid & (HG - 1), kc = tid / HG;         // softmax: head, chunk of KPT keys

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

        // ---- 4. softmax.  Scaled logits -> transpose (thread: key `row`, SCOLS heads).
        {
            uint32_t rr[SCOLS];
            ld_cols(tb + lane_base + S_COL + SCOLS * (warp >> 2), rr);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < SCOLS; ++j)
                Ts[row * T_STRIDE + SCOLS * (warp >> 2) + j] = valid ? __uint_as_float(rr[j]) * scale : -INFINITY;
        }
        __syncthreads();
        {
            float mx = -INFINITY;
#pragma unroll
            for (int j = 0; j < KPT; ++j) mx = fmaxf(mx, Ts[(KPT * kc + j) * T_STRIDE + h]);
            red_m[kc][h] = mx;
        }
        __syncthreads();
        {
            float m = red_m[0][h];
#pragma unroll
            for (int r = 1; r < KC; ++r) m = fmaxf(m, red_m[r][h]);
            if (kc == 0) m_s[h] = m;
            float sum = 0.0f;
            uint32_t hi[KPT / 2], lo[KPT / 2];
#pragma unroll
            for (int i = 0; i < KPT / 2; ++i) {
                const float p0 = __expf(Ts[(KPT * kc + 2 * i) * T_STRIDE + h] - m);
                const float p1 = __expf(Ts[(KPT * kc + 2 * i + 1) * T_STRIDE + h] - m);
                sum += p0 + p1;
                const __nv_bfloat162 ph = __floats2bfloat162_rn(p0, p1);
                const float2 phf = __bfloat1622float2(ph);
                const __nv_bfloat162 pl = __floats2bfloat162_rn(p0 - phf.x, p1 - phf.y);
                hi[i] = *reinterpret_cast<const uint32_t *>(&ph);
                lo[i] = *reinterpret_cast<const uint32_t *>(&pl);
            }
            // P^T row h, keys KPT*kc ..: slab key/64, 16-byte chunk (key%64)/8
            // swizzled by h, then the byte of the key inside its chunk
            const int key0 = KPT * kc, k6 = key0 & 63;
            const uint32_t off = (key0 >> 6) * P_SLAB + h * 128 + ((((k6 >> 3) ^ (h & 7))) << 4) + (k6 & 7) * 2;
            st_pairs(Ph + off, hi);
            st_pairs(Pl + off, lo);
            red_l[kc][h] = sum;
        }
        fence_proxy_async_smem();
        __syncthreads();
        fence_after_sync();
        // ---- 5. O^T = V^T . P^T (hi, then lo), 128 dims per chunk; lane 0 of
        // warp cc issues chunk cc (four issuers, disjoint accumulators)
        if (lane == 0 && warp < 4) {
            const uint32_t va = smem_addr(Vs), ph = smem_addr(Ph), pl = smem_addr(Pl);
            const int cc = warp;
            {
                for (int part = 0; part < 2; ++part) {
                    const uint32_t pb = part ? pl : ph;
#pragma unroll
                    for (int kk = 0; kk < KT / 16; ++kk) {
                        const uint64_t ad = smem_desc(va + (2 * cc) * V_SLAB + kk * 2048, V_SLAB, 1024);
                        const uint64_t bd = smem_desc(pb + (kk >> 2) * P_SLAB + (kk & 3) * 32, 16, 1024);
                        mma_ss(tb + O_COL + HG * cc, ad, bd, IDESC_O, (part | kk) ? 1u : 0u);
                    }
                }
            }
            mma_commit(&bar_o);
        }
        __syncwarp();
        if (tid < HG) {
            float l = 0.0f;
#pragma unroll
            for (int r = 0; r < KC; ++r) l += red_l[r][tid];
            l_s[tid] = l;
        }
    } else {
        if (tid == 0) wait_bar(&bar_q, 0, c.error);          // no copy may be in flight at exit
        if (tid < HG) {
            m_s[tid] = -INFINITY;
            l_s[tid] = 0.0f;
        }
    }
    // ---- 6. merge the five tiles of this (request, head group).  Each live
    // tile leaves its unscaled partial O^T as [head][dim] fp32 in its V
    // region (free once the second product has completed) beside its
    // per-head (m, l); after one cluster barrier every CTA forms all five
    // tiles' weights exp(m_r - M) / L and sums its fifth of the output.
    if (live) {
        wait_bar(&bar_o, 0, c.error);
        fence_after_sync();
        uint32_t rr[HG];
        ld_cols(tb + lane_base + O_COL + HG * (warp >> 2), rr);
        tmem_ld_wait();
        const int d = 128 * (warp >> 2) + 32 * (warp & 3) + lane;
#pragma unroll
        for (int j = 0; j < HG; ++j) Ob[j * CSA2_LATENT + d] = __uint_as_float(rr[j]);
    }
    cluster.sync();                                       // (m, l) and partials visible cluster-wide
    if (tid < NTILES * HG) {
        const int r = tid / HG, hh = tid % HG;
        mt_s[r][hh] = cluster.map_shared_rank(&m_s[0], r)[hh];
        lt_s[r][hh] = cluster.map_shared_rank(&l_s[0], r)[hh];
    }
    __syncthreads();
    if (tid < HG) {
        float M = -INFINITY;
#pragma unroll
        for (int r = 0; r < NTILES; ++r) M = fmaxf(M, mt_s[r][tid]);
        float L = 0.0f;
#pragma unroll
        for (int r = 0; r < NTILES; ++r)
            if (mt_s[r][tid] != -INFINITY) L += __expf(mt_s[r][tid] - M) * lt_s[r][tid];
        const bool any = M != -INFINITY && L > 0.0f;
#pragma unroll
        for (int r = 0; r < NTILES; ++r)
            fac_s[r][tid] = (any && mt_s[r][tid] != -INFINITY) ? __expf(mt_s[r][tid] - M) / L : 0.0f;
        if (lse && tile == 0 && tid < nh) lse[(size_t)b * heads + hg0 + tid] = any ? M + logf(L) : -INFINITY;
        if (tid < NTILES) tile_live[tid] = mt_s[tid][0] != -INFINITY;
    }
    __syncthreads();
    {
        // This CTA's fifth of the HG x 512 outputs (NU float4 per thread):
        // every remote load is issued before any sum.
        constexpr int total4 = HG * (CSA2_LATENT / 4);
        constexpr int NU = ((total4 + NTILES - 1) / NTILES + THREADS - 1) / THREADS;
        const int lo4 = tile * total4 / NTILES, hi4 = (tile + 1) * total4 / NTILES;
        float4 v[NU][NTILES];
#pragma unroll
        for (int u = 0; u < NU; ++u) {
            const int i = lo4 + tid + u * THREADS;
#pragma unroll
            for (int r = 0; r < NTILES; ++r)
                v[u][r] = (i < hi4 && tile_live[r]) ? reinterpret_cast<const float4 *>(cluster.map_shared_rank(Ob, r))[i]
                                                    : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        float4 acc[NU];
#pragma unroll
        for (int u = 0; u < NU; ++u) {
            const int hh = min((lo4 + tid + u * THREADS) / (CSA2_LATENT / 4), HG - 1);
            acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int r = 0; r < NTILES; ++r) {
                const float f = fac_s[r][hh];
                acc[u].x = fmaf(f, v[u][r].x, acc[u].x);
                acc[u].y = fmaf(f, v[u][r].y, acc[u].y);
                acc[u].z = fmaf(f, v[u][r].z, acc[u].z);
                acc[u].w = fmaf(f, v[u][r].w, acc[u].w);
            }
        }
        // Every remote read of this CTA has returned: tell the cluster, and
        // wait for the others only after the output stores.
        asm volatile("barrier.cluster.arrive.aligned;" ::: "memory");
#pragma unroll
        for (int u = 0; u < NU; ++u) {
            const int i = lo4 + tid + u * THREADS;
            const int hh = i / (CSA2_LATENT / 4), d4 = i % (CSA2_LATENT / 4);
            if (i >= hi4 || hh >= nh) continue;
            const size_t o = ((size_t)b * heads + hg0 + hh) * CSA2_LATENT + 4 * d4;
            if (out_is_fp32) {
                *reinterpret_cast<float4 *>((float *)out + o) = acc[u];
            } else {
                __nv_bfloat162 lo = __floats2bfloat162_rn(acc[u].x, acc[u].y),
                               hi = __floats2bfloat162_rn(acc[u].z, acc[u].w);
                uint2 pk = make_uint2(*reinterpret_cast<uint32_t *>(&lo), *reinterpret_cast<uint32_t *>(&hi));
                *reinterpret_cast<uint2 *>((__nv_bfloat16 *)out + o) = pk;
            }
        }
    }
    // No CTA leaves while another may still read its partials.
    asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
    fence_before_sync();
    __syncthreads();
    if (warp == 0) {
        fence_after_sync();
        tmem_dealloc(tb, TMEM_COLS);
    }
}

// q viewed as a 3-D bf16 tensor (512 dims, heads, batch); boxes of 64 dims x
// hg heads, 128-byte swizzled.
bool make_q_map(CUtensorMap *m, const uint16_t *q, int heads, int batch, int hg)
{
    auto fn = tensor_map_encoder();
    if (!fn) return false;
    cuuint64_t dims[3] = {CSA2_LATENT, (cuuint64_t)heads, (cuuint64_t)batch};
    cuuint64_t strides[2] = {CSA2_LATENT * 2, (cuuint64_t)heads * CSA2_LATENT * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)hg, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, (void *)q, dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int HG>
cudaError_t launch_hg(const CacheView &c, int heads, const uint16_t *q, const int32_t *topk, float scale, void *out,
                      int out_is_fp32, uint32_t flags, cudaStream_t st, float *lse)
{
    CUtensorMap map_q;
    if (!make_q_map(&map_q, q, heads, c.batch, HG)) return cudaErrorInvalidValue;
    dim3 grid(NTILES, (heads + HG - 1) / HG, c.batch);
    LaunchScope scope(CSA2_KERNEL_ATTEND, st);
    return launch_pdl(attend_dsm_kernel<HG>, grid, dim3(THREADS), Cfg<HG>::SMEM_BYTES, st, map_q, c, heads, topk,
                      scale, out, out_is_fp32, flags, lse);
}

// Clusters of the 16-head kernel the device runs at once (0 if unknown).
int max_clusters_16()
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(NTILES, 1, 1);
    cfg.blockDim = dim3(THREADS, 1, 1);
    cfg.dynamicSmemBytes = Cfg<16>::SMEM_BYTES;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = NTILES;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, (void *)attend_dsm_kernel<16>, &cfg) != cudaSuccess) {
        cudaGetLastError();
        n = 0;
    }
    return n;
}

}  // namespace

// 16-head CTAs halve each CTA's softmax, partial and merge work (the
// latency of a small batch) but gather every key twice as often; they are
// used while all their clusters run on the device at once (one wave),
// 32-head CTAs beyond that.
cudaError_t launch_attend_dsm(const CacheView &c, int heads, const uint16_t *q, const int32_t *topk, float scale,
                              void *out, int out_is_fp32, uint32_t flags, cudaStream_t st, float *lse)
{
    static bool attr_done[64] = {};
    static int wave16[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    int wave = dev < 64 ? wave16[dev] : 0;
    if (dev >= 64 || !attr_done[dev]) {
        e = cudaFuncSetAttribute(attend_dsm_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)Cfg<16>::SMEM_BYTES);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(attend_dsm_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)Cfg<32>::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        wave = max_clusters_16();
        if (dev < 64) {
            wave16[dev] = wave;
            attr_done[dev] = true;
        }
    }
    const long long clusters16 = (long long)((heads + 15) / 16) * c.batch;
    if (clusters16 <= wave) return launch_hg<16>(c, heads, q, topk, scale, out, out_is_fp32, flags, st, lse);
    return launch_hg<32>(c, heads, q, topk, scale, out, out_is_fp32, flags, st, lse);
}

}  // namespace csa2

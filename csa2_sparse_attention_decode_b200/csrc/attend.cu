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
// Grid (5 tiles, ceil(heads / HG) head groups, batch); the five tiles of one
// (request, head group) form a cluster.  Tiles 0-3 are the top-512 entries,
// tile 4 the SWA window.  512 threads; thread t owns key row t & 127 while
// gathering (a quarter t >> 7 of its channels) and the same key as a tensor-
// memory lane afterwards.
//   1. q (bf16, HG heads x 512) -> smem by TMA, K-major, 128-byte swizzle.
//   2. gather + dequantise 128 keys to bf16 (exact: e2m1 x e4m3 and
//      e4m3 x 2^e all fit bf16) -> smem V tile, K-major, swizzled.  With
//      CSA2_ATTEND_INPUTS_SETTLED this runs before the dependency wait.
//   3. S^T[128 keys x HG heads] = V . Q^T  (32 MMAs from four issuers, one
//      channel quarter and one fp32 TMEM accumulator each, summed on read)
//   4. softmax per head over the tile's keys, in base 2: each warp takes the
//      maximum of its 32 keys (TMEM lanes) with one warp reduction, the four
//      lane groups meet in shared memory; P = 2^(x - m) is split into bf16
//      hi + lo (the second product keeps ~16 bits of P) and stored K-major as
//      2*HG rows [hi heads | lo heads] x 128 keys.
//   5. O^T[512 x 2HG] = V^T . [P_hi | P_lo]^T  (4 dim chunks x 8 MMAs; the hi
//      and lo products land in adjacent accumulator columns of one MMA)
//   6. merge: each tile stages its unnormalised partial O_r = hi + lo as
//      [head][dim] fp32 over the V tile beside its per-head (m_r, l_r = sum
//      p); after one cluster barrier each CTA forms one fifth of the output,
//      loading every tile's (m, l) and its five partial float4s in one round
//      of distributed-shared-memory loads:
//        out = sum_r 2^(m_r - M) O_r / sum_r l_r 2^(m_r - M),  M = max_r m_r.
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

// Sizes for HG heads per CTA (16, 24 or 32).
template <int HG>
struct Cfg {
    static_assert(HG == 16 || HG == 24 || HG == 32, "head group of 16, 24 or 32");
    static constexpr int CPT = HG / 4;                 // softmax: S^T columns (heads) per thread
    static constexpr int CPT_LD = CPT == 6 ? 8 : CPT;  // columns loaded for them (a supported width)
    // N of the first product: HG rounded up to a multiple of 16 (M = 128);
    // q rows past HG in a slab are never written and their S^T columns never read.
    static constexpr int SN = (HG + 15) / 16 * 16;
    static constexpr int Q_SLAB = SN * 128;            // SN rows (HG heads) x 64 dims
    static constexpr int Q_BOX_BYTES = 8 * HG * 128;   // what the eight q boxes bring
    static constexpr int Q_BYTES = 8 * Q_SLAB;
    static constexpr int P_ROWS = 2 * HG;              // hi rows, then lo rows
    static constexpr int P_SLAB = P_ROWS * 128;        // 2HG rows x 64 keys
    static constexpr int P_BYTES = 2 * P_SLAB;
    static constexpr int Q_OFF = V_BYTES, P_OFF = Q_OFF + Q_BYTES;
    static constexpr size_t SMEM_BYTES = 1024 + P_OFF + P_BYTES;
    // The staged output [head][dim] (fp32) reuses the V tile once the second
    // product has completed.
    static_assert(HG * CSA2_LATENT * 4 <= V_BYTES, "staging must fit the V tile");
    // S^T's four channel-quarter partials in columns [0, 4SN); O^T chunk c
    // in [O_COL c, O_COL c + 2HG) (O_COL: 2HG rounded up to 32 columns),
    // written only after every S^T column has been read.
    static constexpr int O_COL = (2 * HG + 31) / 32 * 32;
    static constexpr uint32_t TMEM_COLS = HG == 24 ? 256 : 8 * HG;
    static_assert(4 * O_COL <= (int)TMEM_COLS, "the O^T chunks fit the allocation");
    static_assert((TMEM_COLS & (TMEM_COLS - 1)) == 0 && TMEM_COLS >= 32, "allocation is a power of two");
    static_assert(4 * SN <= (int)TMEM_COLS && 8 * HG <= (int)TMEM_COLS, "the accumulators fit the allocation");
    static_assert(3 * CPT + CPT_LD <= SN, "softmax loads stay inside one S^T partial");
    static constexpr uint32_t IDESC_S = idesc_f16(128, SN, true, false, false);
    static constexpr uint32_t IDESC_O = idesc_f16(128, P_ROWS, true, true, false);
    static constexpr int TOTAL4 = HG * (CSA2_LATENT / 4);              // float4 of the output
    static constexpr int NU = (TOTAL4 / NTILES + 1 + THREADS - 1) / THREADS;   // per thread in the merge
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

// Tensor-memory load of as many columns as the array holds (4, 8, 16, 32,
// 48 or 64).
template <int N>
__device__ __forceinline__ void ld_cols(uint32_t a, uint32_t (&r)[N])
{
    if constexpr (N == 4) {
        tmem_ld4(a, r);
    } else if constexpr (N == 8) {
        tmem_ld8(a, r);
    } else if constexpr (N == 16) {
        tmem_ld16(a, r);
    } else if constexpr (N == 32) {
        tmem_ld32(a, r);
    } else if constexpr (N == 48) {
        uint32_t (&lo)[32] = *reinterpret_cast<uint32_t (*)[32]>(&r[0]);
        uint32_t (&hi)[16] = *reinterpret_cast<uint32_t (*)[16]>(&r[32]);
        tmem_ld32(a, lo);
        tmem_ld16(a + 32, hi);
    } else {
        static_assert(N == 64, "4 to 64 columns");
        uint32_t (&lo)[32] = *reinterpret_cast<uint32_t (*)[32]>(&r[0]);
        uint32_t (&hi)[32] = *reinterpret_cast<uint32_t (*)[32]>(&r[32]);
        tmem_ld32(a, lo);
        tmem_ld32(a + 32, hi);
    }
}

constexpr float LOG2E = 1.4426950408889634f, LN2 = 0.6931471805599453f;

// Maximum over the warp's 32 lanes (-inf lanes are ignored unless all are).
__device__ __forceinline__ float warp_max(float v)
{
    float m;
    asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;" : "=f"(m) : "f"(v));
    return m;
}
__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int off = 16; off; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}
// 2^x by the hardware approximation (the one __expf uses after scaling by
// log2 e); 2^-inf = 0.
__device__ __forceinline__ float exp2f_approx(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ bool wait_bar(uint64_t *bar, uint32_t parity, int32_t *err)
{
    if (mbar_wait(bar, parity)) return true;
    set_error(err, CSA2_DEV_TIMEOUT);
    return false;
}

// Byte offset of (row n, key k) in a K-major, 128-byte swizzled operand of
// 64-key slabs holding `rows` rows each.
__device__ __forceinline__ uint32_t kmajor_off(int n, int k, int slab_bytes)
{
    const int k6 = k & 63;
    return (uint32_t)((k >> 6) * slab_bytes + n * 128 + ((((k6 >> 3) ^ (n & 7))) << 4) + (k6 & 7) * 2);
}

template <int HG>
__global__ void __cluster_dims__(NTILES, 1, 1) __launch_bounds__(THREADS, 1)
attend_kernel(const __grid_constant__ CUtensorMap map_q, CacheView c, int heads, const int32_t *topk, const uint16_t *q,
              float scale, void *out, int out_is_fp32, uint32_t flags, float *lse)
{
    using C = Cfg<HG>;
    constexpr int CPT = C::CPT, Q_SLAB = C::Q_SLAB, P_SLAB = C::P_SLAB, NU = C::NU;
    constexpr int TOTAL4 = C::TOTAL4;
    constexpr uint32_t TMEM_COLS = C::TMEM_COLS, IDESC_S = C::IDESC_S, IDESC_O = C::IDESC_O;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = (uint8_t *)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
    uint8_t *Vs = sm, *Qs = sm + C::Q_OFF, *Ps = sm + C::P_OFF;
    float *Ob = reinterpret_cast<float *>(Vs);
    __shared__ __align__(8) uint64_t bar_q, bar_s, bar_o;
    __shared__ uint32_t tmem_base;
    __shared__ float red_m[4][HG], red_l[4][HG];
    __shared__ float m_s[HG], l_s[HG];                   // this tile's (m, l) per head, read by the cluster
    __shared__ float mt_s[NTILES][HG], lt_s[NTILES][HG];   // every tile's (m, l), gathered for the merge
    cg::cluster_group cluster = cg::this_cluster();

    const int tile = blockIdx.x, hg0 = blockIdx.y * HG, b = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int row = tid & (KT - 1), qtr = tid >> 7;     // gather: key row, quarter of its channels
    if (warp == 0) {
        tmem_alloc(&tmem_base, TMEM_COLS);
        fence_before_sync();
    }
    if (tid == 32) tma_prefetch_map(&map_q);
    if (warp == 1) {
        // An L2 hint of this tile's fifth of the group's q rows (nothing is
        // read before the wait; the copy after it sees the current data).
        const size_t row0 = (size_t)b * heads + hg0, nb = (size_t)min(HG, heads - hg0) * CSA2_LATENT * 2;
        prefetch_l2_range(q + row0 * CSA2_LATENT, nb * tile / NTILES, nb * (tile + 1) / NTILES, lane, 2);
    }
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
    if (tid == 0) {
        mbar_init(&bar_q, 1);
        mbar_init(&bar_s, 4);                                // one commit per issuing warp
        mbar_init(&bar_o, 4);                                // one commit per issuing warp
        mbar_fence_init();
    }
    // Settled inputs: the gather, and the CTA barrier that publishes it (and
    // the tensor-memory base and the mbarriers), overlap the previous kernel.
    bool live = false;                                    // any valid key in this tile
    if (early) {
        gather();
        fence_proxy_async_smem();
        live = __syncthreads_or(valid) != 0;
        fence_after_sync();
    }
    grid_dependency_wait();                               // q (and, unless settled, the rest) may be fresh
    allow_dependents();
    const int nh = min(HG, heads - hg0);
    if (tid == 0) {
        // ---- 1. q -> smem by TMA: 8 boxes of 64 dims x HG heads, 128-byte
        // swizzled (K-major operand layout); heads past `heads` read as zero.
        mbar_arrive_expect_tx(&bar_q, C::Q_BOX_BYTES);
        for (int slab = 0; slab < 8; ++slab) tma_load_3d(Qs + slab * Q_SLAB, &map_q, 64 * slab, hg0, b, &bar_q);
    }
    if (!early) {
        gather();
        fence_proxy_async_smem();
        live = __syncthreads_or(valid) != 0;
        fence_after_sync();
    }
    const uint32_t tb = tmem_base;
    const int sp = warp & 3;                              // TMEM lane group: keys / dims 32 sp ..
    const uint32_t lane_base = (uint32_t)(32 * sp) << 16;

    if (live) {
        // ---- 3. S^T = V . Q^T, split along the 512 channels over four
        // issuers (lane 0 of warps 0-3): issuer w sums channels [128w,
        // 128w + 128) into its own accumulator, columns [SN w, SN w + SN).
        if (lane == 0 && warp < 4) {
            wait_bar(&bar_q, 0, c.error);
            const uint32_t va = smem_addr(Vs), qa = smem_addr(Qs);
#pragma unroll
            for (int j = 0; j < CSA2_LATENT / 64; ++j) {
                const int kk = warp * (CSA2_LATENT / 64) + j;
                const uint32_t off = (kk >> 2), in = (kk & 3) * 32;
                mma_ss(tb + (uint32_t)(C::SN * warp), smem_desc(va + off * V_SLAB + in, 16, 1024),
                       smem_desc(qa + off * Q_SLAB + in, 16, 1024), IDESC_S, j > 0 ? 1u : 0u);
            }
            mma_commit(&bar_s);
        }
        __syncwarp();
        wait_bar(&bar_s, 0, c.error);
        fence_after_sync();
    }
    // ---- 4. softmax in the base-2 domain: x = s * scale * log2(e).  This
    // thread: key `row` (its TMEM lane), heads c0 .. c0 + CPT.
    const int c0 = (warp >> 2) * CPT;
    float p[CPT];
    if (live) {
        float x[CPT];
        {
            uint32_t r0[C::CPT_LD], r1[C::CPT_LD], r2[C::CPT_LD], r3[C::CPT_LD];   // the four channel quarters
            ld_cols(tb + lane_base + c0, r0);
            ld_cols(tb + lane_base + C::SN + c0, r1);
            ld_cols(tb + lane_base + 2 * C::SN + c0, r2);
            ld_cols(tb + lane_base + 3 * C::SN + c0, r3);
            tmem_ld_wait();
            const float sc2 = scale * LOG2E;
#pragma unroll
            for (int j = 0; j < CPT; ++j) {
                const float sv = (__uint_as_float(r0[j]) + __uint_as_float(r1[j])) +
                                 (__uint_as_float(r2[j]) + __uint_as_float(r3[j]));
                x[j] = valid ? sv * sc2 : -INFINITY;
            }
        }
        fence_before_sync();
#pragma unroll
        for (int j = 0; j < CPT; ++j) {
            const float mx = warp_max(x[j]);
            if (lane == 0) red_m[sp][c0 + j] = mx;
        }
        __syncthreads();
#pragma unroll
        for (int j = 0; j < CPT; ++j) {
            const float m = fmaxf(fmaxf(red_m[0][c0 + j], red_m[1][c0 + j]), fmaxf(red_m[2][c0 + j], red_m[3][c0 + j]));
            p[j] = exp2f_approx(x[j] - m);                 // x = -inf (invalid key) -> 0
        }
        // P^T rows c0 + j (hi) and HG + c0 + j (lo), K-major [row][key]
#pragma unroll
        for (int j = 0; j < CPT; ++j) {
            const __nv_bfloat16 ph = __float2bfloat16_rn(p[j]);
            const __nv_bfloat16 pl = __float2bfloat16_rn(p[j] - __bfloat162float(ph));
            *reinterpret_cast<__nv_bfloat16 *>(Ps + kmajor_off(c0 + j, row, P_SLAB)) = ph;
            *reinterpret_cast<__nv_bfloat16 *>(Ps + kmajor_off(HG + c0 + j, row, P_SLAB)) = pl;
        }
        fence_proxy_async_smem();
        fence_before_sync();
        __syncthreads();                                   // P complete; every S^T column read
        fence_after_sync();
    }
    // ---- 5. O^T = V^T . [P_hi | P_lo]^T, 128 dims per chunk; lane 0 of
    // warp cc issues chunk cc (four issuers, disjoint accumulators).  The
    // per-head sums of p follow, off the products' path.
    if (live) {
        if (lane == 0 && warp < 4) {
            const uint32_t va = smem_addr(Vs), pa = smem_addr(Ps);
            const int cc = warp;
#pragma unroll
            for (int kk = 0; kk < KT / 16; ++kk) {
                const uint64_t ad = smem_desc(va + (2 * cc) * V_SLAB + kk * 2048, V_SLAB, 1024);
                const uint64_t bd = smem_desc(pa + (kk >> 2) * P_SLAB + (kk & 3) * 32, 16, 1024);
                mma_ss(tb + (uint32_t)(C::O_COL * cc), ad, bd, IDESC_O, kk > 0 ? 1u : 0u);
            }
            mma_commit(&bar_o);
        }
        __syncwarp();
#pragma unroll
        for (int j = 0; j < CPT; ++j) {
            const float sm = warp_sum(p[j]);
            if (lane == 0) red_l[sp][c0 + j] = sm;
        }
        __syncthreads();
        if (tid < HG) {
            m_s[tid] = fmaxf(fmaxf(red_m[0][tid], red_m[1][tid]), fmaxf(red_m[2][tid], red_m[3][tid]));
            l_s[tid] = (red_l[0][tid] + red_l[1][tid]) + (red_l[2][tid] + red_l[3][tid]);
        }
        // ---- 6a. this tile's unnormalised partial hi + lo, staged
        // [head][dim] over the V tile (free once the product has completed)
        wait_bar(&bar_o, 0, c.error);
        fence_after_sync();
        const int cc = warp >> 2;
        uint32_t rr[2 * HG];
        ld_cols(tb + lane_base + (uint32_t)(C::O_COL * cc), rr);
        tmem_ld_wait();
        const int d = 128 * cc + 32 * sp + lane;
#pragma unroll
        for (int j = 0; j < HG; ++j) Ob[j * CSA2_LATENT + d] = __uint_as_float(rr[j]) + __uint_as_float(rr[HG + j]);
    } else {
        if (tid == 0) wait_bar(&bar_q, 0, c.error);          // no copy may be in flight at exit
        if (tid < HG) {
            m_s[tid] = -INFINITY;
            l_s[tid] = 0.0f;
        }
    }
    // ---- 6b. one cluster barrier, then one round of distributed-shared-
    // memory loads: every tile's (m, l) into shared memory beside this
    // thread's five partial float4s, issued together.  Output (head h):
    //   out = sum_r 2^(m_r - M) O_r / sum_r l_r 2^(m_r - M),  M = max_r m_r.
    cluster_sync_aligned();
    {
        const int lo4 = tile * TOTAL4 / NTILES, hi4 = (tile + 1) * TOTAL4 / NTILES;
        if (tid < 2 * NTILES * HG) {
            const int r = (tid >> 1) / HG, hh = (tid >> 1) % HG;
            const float *src = (tid & 1) ? &l_s[0] : &m_s[0];
            (tid & 1 ? lt_s : mt_s)[r][hh] = cluster.map_shared_rank(src, r)[hh];
        }
        float4 v[NU][NTILES];
#pragma unroll
        for (int u = 0; u < NU; ++u) {
            const int i = lo4 + tid + u * THREADS;
#pragma unroll
            for (int r = 0; r < NTILES; ++r)
                v[u][r] = i < hi4 ? reinterpret_cast<const float4 *>(cluster.map_shared_rank(Ob, r))[i]
                                  : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        __syncthreads();                                   // every tile's (m, l) in shared memory
        float4 acc[NU];
#pragma unroll
        for (int u = 0; u < NU; ++u) {
            const int i = lo4 + tid + u * THREADS;
            const int hh = min(i, TOTAL4 - 1) / (CSA2_LATENT / 4);
            float M = -INFINITY;
#pragma unroll
            for (int r = 0; r < NTILES; ++r) M = fmaxf(M, mt_s[r][hh]);
            float wr[NTILES], L = 0.0f;
#pragma unroll
            for (int r = 0; r < NTILES; ++r) {
                wr[r] = mt_s[r][hh] != -INFINITY ? exp2f_approx(mt_s[r][hh] - M) : 0.0f;
                L += wr[r] * lt_s[r][hh];
            }
            const bool any = M != -INFINITY && L > 0.0f;
            const float inv = any ? 1.0f / L : 0.0f;
            acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int r = 0; r < NTILES; ++r) {
                if (wr[r] == 0.0f) continue;                 // a dead tile's staging is not written
                const float f = wr[r] * inv;
                acc[u].x = fmaf(f, v[u][r].x, acc[u].x);
                acc[u].y = fmaf(f, v[u][r].y, acc[u].y);
                acc[u].z = fmaf(f, v[u][r].z, acc[u].z);
                acc[u].w = fmaf(f, v[u][r].w, acc[u].w);
            }
            if (lse && i < hi4 && (i % (CSA2_LATENT / 4)) == 0 && hh < nh)
                lse[(size_t)b * heads + hg0 + hh] = any ? (M + log2f(L)) * LN2 : -INFINITY;
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
    // No CTA leaves while another may still read its staging.
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
    return launch_pdl(attend_kernel<HG>, grid, dim3(THREADS), Cfg<HG>::SMEM_BYTES, st, map_q, c, heads, topk, q, scale,
                      out, out_is_fp32, flags, lse);
}

}  // namespace

// Head groups: 16-head CTAs halve each CTA's softmax, staging and merge work
// (the latency of a small batch) but gather every key more often.  16 heads
// while all of a launch's clusters run at once (one wave), 24 while those
// do, 32 beyond.  (Fewer, larger CTAs would let consecutive launches be
// resident together, but at a batch of 4 x 64 heads 24-head CTAs measured
// 10.2 us per launch in a chain against 10.0 for 16-head ones: their merge
// costs more than the residency saves.)  A request with at most 16 heads
// takes 16.
cudaError_t launch_attend(const CacheView &c, int heads, const uint16_t *q, const int32_t *topk, float scale,
                          void *out, int out_is_fp32, uint32_t flags, cudaStream_t st, float *lse)
{
    static DeviceOnce once;
    static int wave16[DeviceOnce::N] = {}, wave24[DeviceOnce::N] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess)
        e = once.run(dev, [&] {
            cudaError_t r = cudaFuncSetAttribute(attend_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 (int)Cfg<16>::SMEM_BYTES);
            if (r == cudaSuccess)
                r = cudaFuncSetAttribute(attend_kernel<24>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Cfg<24>::SMEM_BYTES);
            if (r == cudaSuccess)
                r = cudaFuncSetAttribute(attend_kernel<32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Cfg<32>::SMEM_BYTES);
            if (r != cudaSuccess) return r;
            auto clusters = [&](const void *fn, size_t smem) {
                cudaLaunchConfig_t cfg = {};
                cfg.gridDim = dim3(NTILES, 1, 1);
                cfg.blockDim = dim3(THREADS, 1, 1);
                cfg.dynamicSmemBytes = smem;
                cudaLaunchAttribute attr[1];
                attr[0].id = cudaLaunchAttributeClusterDimension;
                attr[0].val.clusterDim.x = NTILES;
                attr[0].val.clusterDim.y = 1;
                attr[0].val.clusterDim.z = 1;
                cfg.attrs = attr;
                cfg.numAttrs = 1;
                int n = 0;
                if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess) {
                    cudaGetLastError();
                    n = 0;
                }
                return n;
            };
            wave16[dev] = clusters((const void *)attend_kernel<16>, Cfg<16>::SMEM_BYTES);
            wave24[dev] = clusters((const void *)attend_kernel<24>, Cfg<24>::SMEM_BYTES);
            return cudaSuccess;
        });
    if (e != cudaSuccess) return e;
    const long long clusters16 = (long long)((heads + 15) / 16) * c.batch;
    const long long clusters24 = (long long)((heads + 23) / 24) * c.batch;
    int hg;
    if (heads <= 16 || clusters16 <= wave16[dev])
        hg = 16;
    else if (clusters24 <= wave24[dev])
        hg = 24;
    else
        hg = 32;
    if (hg == 16) return launch_hg<16>(c, heads, q, topk, scale, out, out_is_fp32, flags, st, lse);
    if (hg == 24) return launch_hg<24>(c, heads, q, topk, scale, out, out_is_fp32, flags, st, lse);
    return launch_hg<32>(c, heads, q, topk, scale, out, out_is_fp32, flags, st, lse);
}

}  // namespace csa2

// The indexer query as an FP8 tensor-core operand.
//
// A bf16 query head q (128 dims) is scaled by 2^s so that max|q'| lies in
// [2^14, 2^15), then split into three e5m2 parts q' = p1 + p2 + p3 with
// p1 = e5m2(q'), p2 = e5m2(q' - p1), p3 = e5m2(q' - p1 - p2).  A bf16 value
// has 8 significant bits and each e5m2 part takes 3, so the sum is exact for
// every element not below 2^-9 (e5m2 steps of 2^-16), i.e. down to 2^-24 of
// the head's largest entry.  w' = w * 2^-s undoes the scale.  Used by both
// scoring kernels (score_umma.cu, pool_select.cu).
#pragma once
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "common.cuh"

namespace csa2 {

constexpr int IQ_PARTS = 3;
constexpr int IQ_ROWS = IQ_PARTS * CSA2_IDX_HEADS;          // 96 rows: part p, head h at row 32p + h
constexpr int IQ_BYTES = IQ_ROWS * CSA2_KEY_DIM;            // 12 KB of e5m2

// An e5m2 code is the high byte of the fp16 with the same value.
__device__ __forceinline__ float iq_e5m2_to_f32(uint32_t c) { return __half2float(__ushort_as_half((uint16_t)(c << 8))); }

// x * 2^k, correctly rounded (as ldexpf) for k in [-126, 254]: a single
// multiplication by an exact power of two when 2^k is a normal float, two
// for k > 127 (both scale up, so neither rounds).
__device__ __forceinline__ float iq_scale(float x, int k)
{
    if (k <= 127) return x * __int_as_float((k + 127) << 23);
    return (x * __int_as_float(254 << 23)) * __int_as_float((k - 127 + 127) << 23);
}

// Called by 128 threads (t = 0..127): head t/4, dims 32*(t%4) .. +31 of
// request b.  Writes the 96 x 128 e5m2 operand (row n = part*32 + head,
// K-major, 128-byte swizzled) to qbuf and w' to wq[head].
__device__ __forceinline__ void iq_split(int t, const uint16_t *q_idx, const float *w, int b, uint8_t *qbuf,
                                         float *wq)
{
    const int h = t >> 2, qd = t & 3;
    const uint4 *src =
        reinterpret_cast<const uint4 *>(q_idx + ((size_t)b * CSA2_IDX_HEADS + h) * CSA2_KEY_DIM + 32 * qd);
    uint4 raw[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) raw[i] = src[i];
    const uint32_t *rw = reinterpret_cast<const uint32_t *>(raw);
    float x[32];
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        x[2 * i] = __uint_as_float(rw[i] << 16);
        x[2 * i + 1] = __uint_as_float(rw[i] & 0xffff0000u);
        amax = fmaxf(amax, fmaxf(fabsf(x[2 * i]), fabsf(x[2 * i + 1])));
    }
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    int ex = 0;
    if (amax > 0.0f) frexpf(amax, &ex);
    const int sh = (amax > 0.0f) ? 15 - ex : 0;              // amax * 2^sh in [2^14, 2^15); sh in [-114, 164]
    uint32_t part[IQ_PARTS][8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        uint32_t w0 = 0, w1 = 0, w2 = 0;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            float r = iq_scale(x[4 * i + k], sh);
            const uint8_t c0 = (uint8_t)__nv_cvt_float_to_fp8(r, __NV_SATFINITE, __NV_E5M2);
            r -= iq_e5m2_to_f32(c0);
            const uint8_t c1 = (uint8_t)__nv_cvt_float_to_fp8(r, __NV_SATFINITE, __NV_E5M2);
            r -= iq_e5m2_to_f32(c1);
            const uint8_t c2 = (uint8_t)__nv_cvt_float_to_fp8(r, __NV_SATFINITE, __NV_E5M2);
            w0 |= (uint32_t)c0 << (8 * k);
            w1 |= (uint32_t)c1 << (8 * k);
            w2 |= (uint32_t)c2 << (8 * k);
        }
        part[0][i] = w0;
        part[1][i] = w1;
        part[2][i] = w2;
    }
    // row n = part * 32 + h; bytes 32*qd .. +31 are the 16-byte chunks 2qd, 2qd+1
#pragma unroll
    for (int pp = 0; pp < IQ_PARTS; ++pp) {
        const int n = pp * CSA2_IDX_HEADS + h;
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
            const int chunk = 2 * qd + cc;
            *reinterpret_cast<uint4 *>(qbuf + n * 128 + ((chunk ^ (n & 7)) << 4)) =
                make_uint4(part[pp][4 * cc], part[pp][4 * cc + 1], part[pp][4 * cc + 2], part[pp][4 * cc + 3]);
        }
    }
    if (qd == 0) wq[h] = ldexpf(w[(size_t)b * CSA2_IDX_HEADS + h], -sh);
}

}  // namespace csa2

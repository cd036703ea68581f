// mx_block.cuh - one MXFP8 block of 32 values (OCP Microscaling v1.0 as read for
// the triangle contraction): the shared E8M0 scale 2^e with
// e = floor(log2 max|v|) - 8 clamped to [-127, 127] (an all-zero block takes
// -127), and the E4M3 elements v / 2^e rounded to nearest even and saturated at
// +-448; plus where the contraction kernel expects each block's scale byte.
#pragma once

#include <cuda_fp8.h>
#include <stdint.h>

namespace trimul {

// Quantises v[0..31] into q8 (4 E4M3 codes per word, element 0 in the low byte)
// and returns e. The input values are exact in fp32, so amax, e and the division
// by 2^e are exact; __nv_cvt_float2_to_fp8x2 rounds to nearest even and saturates.
__device__ __forceinline__ int mx_quantize32(const float (&v)[32], uint32_t (&q8)[8]) {
    float amax = 0.f;
#pragma unroll
    for (int t = 0; t < 32; ++t) amax = fmaxf(amax, fabsf(v[t]));
    int e = (int)((__float_as_uint(amax) >> 23) & 0xFF) - 127 - 8;
    if (amax == 0.f || e < -127) e = -127;
    if (e > 127) e = 127;
    const float inv = __uint_as_float((uint32_t)(127 - e) << 23);  // 2^-e, exact (e <= 119 for finite bf16)
#pragma unroll
    for (int t = 0; t < 8; ++t) {
        const __nv_fp8x2_storage_t lo =
            __nv_cvt_float2_to_fp8x2(make_float2(v[4 * t] * inv, v[4 * t + 1] * inv), __NV_SATFINITE, __NV_E4M3);
        const __nv_fp8x2_storage_t hi =
            __nv_cvt_float2_to_fp8x2(make_float2(v[4 * t + 2] * inv, v[4 * t + 3] * inv), __NV_SATFINITE, __NV_E4M3);
        q8[t] = (uint32_t)lo | ((uint32_t)hi << 16);
    }
    return e;
}

// The same for 32 bf16 values packed in pairs (w[t] holds values 2t, 2t + 1, the
// lower index in the low half). Non-negative bf16 bit patterns order like their
// values, so max|v| is an unsigned 16-bit max over the patterns with the sign
// cleared, and e comes from its exponent field; the scaling is the fp32 one.
__device__ __forceinline__ int mx_quantize32_bf16(const uint32_t (&w)[16], uint32_t (&q8)[8]) {
    uint32_t m[16];
#pragma unroll
    for (int t = 0; t < 16; ++t) m[t] = w[t] & 0x7FFF7FFFu;
#pragma unroll
    for (int h = 8; h >= 1; h >>= 1)  // pairwise tree: 4 dependent steps instead of 15
#pragma unroll
        for (int t = 0; t < h; ++t) asm("max.u16x2 %0, %0, %1;" : "+r"(m[t]) : "r"(m[t + h]));
    const uint32_t amax = (m[0] & 0xFFFFu) > (m[0] >> 16) ? (m[0] & 0xFFFFu) : (m[0] >> 16);
    int e = (int)(amax >> 7) - 127 - 8;
    if (amax == 0 || e < -127) e = -127;
    if (e > 127) e = 127;
    const float inv = __uint_as_float((uint32_t)(127 - e) << 23);
    const float2 inv2 = make_float2(inv, inv);
#pragma unroll
    for (int t = 0; t < 8; ++t) {
        const uint32_t u0 = w[2 * t], u1 = w[2 * t + 1];
        const float2 x0 = __fmul2_rn(make_float2(__uint_as_float(u0 << 16), __uint_as_float(u0 & 0xFFFF0000u)), inv2);
        const float2 x1 = __fmul2_rn(make_float2(__uint_as_float(u1 << 16), __uint_as_float(u1 & 0xFFFF0000u)), inv2);
        const __nv_fp8x2_storage_t lo = __nv_cvt_float2_to_fp8x2(x0, __NV_SATFINITE, __NV_E4M3);
        const __nv_fp8x2_storage_t hi = __nv_cvt_float2_to_fp8x2(x1, __NV_SATFINITE, __NV_E4M3);
        q8[t] = (uint32_t)lo | ((uint32_t)hi << 16);
    }
    return e;
}

// Byte offset of the scale of (operand row r, K block kb) of channel c in a scale
// array laid out per row tile of the contraction (rows_per_tile rows in
// chunks_per_tile chunks of 128 rows) and per 128-wide K chunk: within a
// 512-byte chunk, row r and block b sit at (r % 32) * 16 + ((r % 128) / 32) * 4
// + b, the order in which a 32 x 128-bit tensor-memory copy places them.
__host__ __device__ __forceinline__ size_t mx_scale_offset(int c, int r, int kb, int rows_per_tile, int row_tiles,
                                                            int kchunks, int chunks_per_tile) {
    const int rt = r / rows_per_tile, nl = r - rt * rows_per_tile;
    const size_t chunk = (((size_t)c * row_tiles + rt) * kchunks + (kb >> 2)) * chunks_per_tile + (nl >> 7);
    return chunk * 512 + (size_t)(nl & 31) * 16 + ((nl & 127) >> 5) * 4 + (kb & 3);
}

}  // namespace trimul

// tile_ops.cuh - per-tile LayerNorm and gating helpers shared by the prologue
// and epilogue kernels (packed fp32x2 arithmetic, bf16 storage).
#pragma once

#include "common.cuh"

namespace trimul {

__device__ __forceinline__ float tanh_approx(float x) {
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// bf16x2 bits -> (low, high) as float2.
__device__ __forceinline__ float2 unpack_bf16x2(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

__device__ __forceinline__ float2 ld_pair_bf16(const __nv_bfloat16 *v, int c) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(v + c));
}

// In-place LayerNorm of one 128-channel cell (row r) of a bf16 tile stored as
// two 64-channel halves (half_bytes apart) of 128-byte rows with the 128-byte
// swizzle (16-byte chunk index XOR row & 7). Two threads per cell: this thread
// takes channel half h and its partner (lane ^ 1) the other half. fp32
// statistics, bf16 result. kAffine: apply gamma/beta (bf16 vectors; a null
// one means 1 or 0).
template <bool kAffine>
__device__ __forceinline__ void ln_row_sw128(uint8_t *tile, int half_bytes, int r, int h, const __nv_bfloat16 *gw,
                                             const __nv_bfloat16 *gb, float eps) {
    uint8_t *rowp = tile + h * half_bytes + r * 128;
    float2 v[32];  // register slot q*4 + e holds logical chunk kc = (q + 4h) & 7, word e
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const int kc = (q + 4 * h) & 7;  // staggered so the two halves of a cell use different banks
        const uint4 u = *reinterpret_cast<const uint4 *>(rowp + ((kc ^ (r & 7)) << 4));
        v[q * 4 + 0] = unpack_bf16x2(u.x);
        v[q * 4 + 1] = unpack_bf16x2(u.y);
        v[q * 4 + 2] = unpack_bf16x2(u.z);
        v[q * 4 + 3] = unpack_bf16x2(u.w);
    }
    float2 a0 = make_float2(0.f, 0.f), a1 = a0, a2 = a0, a3 = a0;
#pragma unroll
    for (int k = 0; k < 32; k += 4) {
        a0 = __fadd2_rn(a0, v[k]);
        a1 = __fadd2_rn(a1, v[k + 1]);
        a2 = __fadd2_rn(a2, v[k + 2]);
        a3 = __fadd2_rn(a3, v[k + 3]);
    }
    float s = (a0.x + a0.y) + (a1.x + a1.y) + (a2.x + a2.y) + (a3.x + a3.y);
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    const float mean = s * (1.f / 128.f);
    const float2 nm = make_float2(-mean, -mean);
    a0 = a1 = a2 = a3 = make_float2(0.f, 0.f);
#pragma unroll
    for (int k = 0; k < 32; k += 4) {
        const float2 d0 = __fadd2_rn(v[k], nm), d1 = __fadd2_rn(v[k + 1], nm);
        const float2 d2 = __fadd2_rn(v[k + 2], nm), d3 = __fadd2_rn(v[k + 3], nm);
        a0 = __ffma2_rn(d0, d0, a0);
        a1 = __ffma2_rn(d1, d1, a1);
        a2 = __ffma2_rn(d2, d2, a2);
        a3 = __ffma2_rn(d3, d3, a3);
    }
    float ss = (a0.x + a0.y) + (a1.x + a1.y) + (a2.x + a2.y) + (a3.x + a3.y);
    ss += __shfl_xor_sync(0xffffffffu, ss, 1);
    const float rstd = rsqrtf(ss * (1.f / 128.f) + eps);
    const float2 sc = make_float2(rstd, rstd), sh = make_float2(-mean * rstd, -mean * rstd);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const int kc = (q + 4 * h) & 7;
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            float2 y = __ffma2_rn(v[q * 4 + e], sc, sh);
            if (kAffine) {
                const int c = h * 64 + kc * 8 + 2 * e;
                const float2 g = gw ? ld_pair_bf16(gw, c) : make_float2(1.f, 1.f);
                const float2 b = gb ? ld_pair_bf16(gb, c) : make_float2(0.f, 0.f);
                y = __ffma2_rn(y, g, b);
            }
            w[e] = pack_bf16x2(y.x, y.y);
        }
        *reinterpret_cast<uint4 *>(rowp + ((kc ^ (r & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

// The whole 128-cell tile by 256 threads (thread t: cell t / 2, half t % 2).
template <bool kAffine>
__device__ __forceinline__ void ln_tile_sw128(uint8_t *tile, int half_bytes, const __nv_bfloat16 *gw,
                                              const __nv_bfloat16 *gb, float eps) {
    ln_row_sw128<kAffine>(tile, half_bytes, (int)threadIdx.x >> 1, (int)threadIdx.x & 1, gw, gb, eps);
}

// Mean and rstd of 128 values, accumulated in fp32 around the first value
// (which keeps E[d^2] - E[d]^2 well conditioned when |mean| >> std). Each of
// two partner lanes (lane ^ 1) accumulates one channel half.
struct RowStats {
    float2 s, ss;
    float k;
};
__device__ __forceinline__ void stats_add(RowStats &st, uint32_t w) {
    const float2 d = __fadd2_rn(unpack_bf16x2(w), make_float2(-st.k, -st.k));
    st.s = __fadd2_rn(st.s, d);
    st.ss = __ffma2_rn(d, d, st.ss);
}
__device__ __forceinline__ float2 stats_finish(const RowStats &st, float eps) {
    float s = st.s.x + st.s.y, ss = st.ss.x + st.ss.y;
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    ss += __shfl_xor_sync(0xffffffffu, ss, 1);
    const float m = s * (1.f / 128.f);
    const float var = fmaxf(ss * (1.f / 128.f) - m * m, 0.f);
    return make_float2(st.k + m, rsqrtf(var + eps));
}

}  // namespace trimul

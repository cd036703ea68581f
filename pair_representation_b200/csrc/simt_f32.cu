// simt_f32.cu - the triangle multiplicative update in true fp32 on CUDA cores.
//
// The same three stages as the bf16 tensor-core path (prologue, contraction,
// epilogue) with every product and sum in fp32 FMA and no TF32 anywhere, for
// callers that need fp32 accuracy. Layouts match the bf16 path: a, b and x are
// channel-major [128][N][ld] in the workspace.
#include "kernels.h"

namespace trimul {
namespace f32 {
constexpr int CELLS = 32;     // cells per prologue / epilogue tile (one residue row segment)
constexpr int THREADS = 256;
}  // namespace f32

__device__ __forceinline__ float sigmoid_exact(float t) { return 1.f / (1.f + expf(-t)); }

// LayerNorm of `cells` rows of 128 values in shared memory, one warp per row.
static __device__ void ln_rows_f32(float (*rows)[kC], int cells, const float *gw, const float *gb, float eps) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int r = warp; r < cells; r += f32::THREADS / 32) {
        float v[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) v[e] = rows[r][lane + 32 * e];
        float s = v[0] + v[1] + v[2] + v[3];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        const float mean = s * (1.f / kC);
        float ss = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) ss = fmaf(v[e] - mean, v[e] - mean, ss);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        const float rstd = 1.f / sqrtf(ss * (1.f / kC) + eps);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int c = lane + 32 * e;
            rows[r][c] = (v[e] - mean) * rstd * (gw ? gw[c] : 1.f) + (gb ? gb[c] : 0.f);
        }
    }
}

// a, b for 32-cell tiles: thread (o, p) computes output channel o of the
// a-pair (p = 0) or b-pair (p = 1) for all 32 cells of the tile.
__global__ void __launch_bounds__(f32::THREADS) prologue_f32_kernel(const float *__restrict__ z, F32Layer L) {
    __shared__ float zh[f32::CELLS][kC];
    const int N = L.N;
    const int jt = (N + f32::CELLS - 1) / f32::CELLS;
    const int o = threadIdx.x & 127, p = threadIdx.x >> 7;
    const float *Wv = p ? L.w_b : L.w_a;
    const float *Wg = p ? L.w_bg : L.w_ag;
    const float bv = (p ? L.b_b : L.b_a) ? (p ? L.b_b : L.b_a)[o] : 0.f;
    const float bg = (p ? L.b_bg : L.b_ag) ? (p ? L.b_bg : L.b_ag)[o] : 0.f;
    float *dst = p ? L.b : L.a;
    for (long tile = blockIdx.x; tile < (long)N * jt; tile += gridDim.x) {
        const int i = (int)(tile / jt), j0 = (int)(tile % jt) * f32::CELLS;
        const int nc = min(f32::CELLS, N - j0);
        __syncthreads();
        for (int e = threadIdx.x; e < f32::CELLS * kC; e += f32::THREADS) {
            const int cl = e / kC, c = e % kC;
            zh[cl][c] = cl < nc ? z[((size_t)i * N + j0 + cl) * kC + c] : 0.f;
        }
        __syncthreads();
        ln_rows_f32(zh, f32::CELLS, L.ln_in_w, L.ln_in_b, L.eps);
        __syncthreads();
        float av[f32::CELLS], ag[f32::CELLS];
#pragma unroll
        for (int cl = 0; cl < f32::CELLS; ++cl) av[cl] = ag[cl] = 0.f;
        for (int k = 0; k < kC; k += 4) {
            const float4 wv = *reinterpret_cast<const float4 *>(Wv + (size_t)o * kC + k);
            const float4 wg = *reinterpret_cast<const float4 *>(Wg + (size_t)o * kC + k);
#pragma unroll
            for (int cl = 0; cl < f32::CELLS; ++cl) {
                const float4 zz = *reinterpret_cast<const float4 *>(&zh[cl][k]);
                av[cl] = fmaf(wv.x, zz.x, av[cl]); av[cl] = fmaf(wv.y, zz.y, av[cl]);
                av[cl] = fmaf(wv.z, zz.z, av[cl]); av[cl] = fmaf(wv.w, zz.w, av[cl]);
                ag[cl] = fmaf(wg.x, zz.x, ag[cl]); ag[cl] = fmaf(wg.y, zz.y, ag[cl]);
                ag[cl] = fmaf(wg.z, zz.z, ag[cl]); ag[cl] = fmaf(wg.w, zz.w, ag[cl]);
            }
        }
        float *row = dst + ((size_t)o * N + i) * L.ld + j0;
#pragma unroll
        for (int cl = 0; cl < f32::CELLS; ++cl) {
            if (cl < nc) {
                const float m = L.mask ? L.mask[(size_t)i * N + j0 + cl] : 1.f;
                row[cl] = m * sigmoid_exact(ag[cl] + bg) * (av[cl] + bv);
            }
        }
    }
}

// x_c = A_c B_c^T (outgoing) or A_c^T B_c (incoming); 64 x 64 tiles, 4 x 4 per thread.
__global__ void __launch_bounds__(256) contract_f32_kernel(F32Layer L, int incoming) {
    constexpr int T = 64, BK = 16;
    __shared__ float As[BK][T + 1], Bs[BK][T + 1];
    const int N = L.N;
    const size_t ld = L.ld;
    const int c = blockIdx.z;
    const int i0 = blockIdx.y * T, j0 = blockIdx.x * T;
    const float *A = L.a + (size_t)c * N * ld;
    const float *B = L.b + (size_t)c * N * ld;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < N; k0 += BK) {
        for (int e = threadIdx.x; e < BK * T; e += 256) {
            int kk, mm;
            if (!incoming) { mm = e / BK; kk = e % BK; }  // k fastest: coalesced along rows of a
            else { kk = e / T; mm = e % T; }              // i fastest: coalesced along columns
            const int k = k0 + kk;
            const int ia = i0 + mm, jb = j0 + mm;
            float va = 0.f, vb = 0.f;
            if (k < N) {
                if (!incoming) {
                    if (ia < N) va = A[(size_t)ia * ld + k];
                    if (jb < N) vb = B[(size_t)jb * ld + k];
                } else {
                    if (ia < N) va = A[(size_t)k * ld + ia];
                    if (jb < N) vb = B[(size_t)k * ld + jb];
                }
            }
            As[kk][mm] = va;
            Bs[kk][mm] = vb;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < BK; ++kk) {
            float av[4], bv[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) { av[u] = As[kk][ty + 16 * u]; bv[u] = Bs[kk][tx + 16 * u]; }
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(av[u], bv[v], acc[u][v]);
        }
        __syncthreads();
    }
    float *X = L.x + (size_t)c * N * ld;
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const int i = i0 + ty + 16 * u, j = j0 + tx + 16 * v;
            if (i < N && j < N) X[(size_t)i * ld + j] = acc[u][v];
        }
}

// out for 32-cell tiles: thread (o, half) computes output channel o for 16 cells.
__global__ void __launch_bounds__(f32::THREADS) epilogue_f32_kernel(const float *__restrict__ z,
                                                                    float *__restrict__ out, F32Layer L) {
    __shared__ float xh[f32::CELLS][kC];
    __shared__ float zh[f32::CELLS][kC];
    const int N = L.N;
    const int jt = (N + f32::CELLS - 1) / f32::CELLS;
    const int o = threadIdx.x & 127, half = threadIdx.x >> 7;
    const float bg = L.b_g ? L.b_g[o] : 0.f, bo = L.b_o ? L.b_o[o] : 0.f;
    for (long tile = blockIdx.x; tile < (long)N * jt; tile += gridDim.x) {
        const int i = (int)(tile / jt), j0 = (int)(tile % jt) * f32::CELLS;
        const int nc = min(f32::CELLS, N - j0);
        __syncthreads();
        for (int e = threadIdx.x; e < f32::CELLS * kC; e += f32::THREADS) {
            const int c = e / f32::CELLS, cl = e % f32::CELLS;  // cells fastest: x is channel-major
            xh[cl][c] = cl < nc ? L.x[((size_t)c * N + i) * L.ld + j0 + cl] : 0.f;
            const int cl2 = e / kC, c2 = e % kC;
            zh[cl2][c2] = cl2 < nc ? z[((size_t)i * N + j0 + cl2) * kC + c2] : 0.f;
        }
        __syncthreads();
        ln_rows_f32(xh, f32::CELLS, L.ln_out_w, L.ln_out_b, L.eps);
        ln_rows_f32(zh, f32::CELLS, L.ln_in_w, L.ln_in_b, L.eps);
        __syncthreads();
        constexpr int H = f32::CELLS / 2;
        float g[H], v[H];
#pragma unroll
        for (int u = 0; u < H; ++u) g[u] = v[u] = 0.f;
        for (int k = 0; k < kC; k += 4) {
            const float4 wg = *reinterpret_cast<const float4 *>(L.w_g + (size_t)o * kC + k);
            const float4 wo = *reinterpret_cast<const float4 *>(L.w_o + (size_t)o * kC + k);
#pragma unroll
            for (int u = 0; u < H; ++u) {
                const int cl = half * H + u;
                const float4 zz = *reinterpret_cast<const float4 *>(&zh[cl][k]);
                const float4 xx = *reinterpret_cast<const float4 *>(&xh[cl][k]);
                g[u] = fmaf(wg.x, zz.x, g[u]); g[u] = fmaf(wg.y, zz.y, g[u]);
                g[u] = fmaf(wg.z, zz.z, g[u]); g[u] = fmaf(wg.w, zz.w, g[u]);
                v[u] = fmaf(wo.x, xx.x, v[u]); v[u] = fmaf(wo.y, xx.y, v[u]);
                v[u] = fmaf(wo.z, xx.z, v[u]); v[u] = fmaf(wo.w, xx.w, v[u]);
            }
        }
#pragma unroll
        for (int u = 0; u < H; ++u) {
            const int cl = half * H + u;
            if (cl < nc) out[((size_t)i * N + j0 + cl) * kC + o] = sigmoid_exact(g[u] + bg) * (v[u] + bo);
        }
    }
}

cudaError_t launch_prologue_f32(const float *z, const F32Layer &L, int grid, cudaStream_t s) {
    prologue_f32_kernel<<<grid, f32::THREADS, 0, s>>>(z, L);
    return cudaGetLastError();
}

cudaError_t launch_contract_f32(const F32Layer &L, int incoming, cudaStream_t s) {
    dim3 grid((L.N + 63) / 64, (L.N + 63) / 64, kC);
    contract_f32_kernel<<<grid, 256, 0, s>>>(L, incoming);
    return cudaGetLastError();
}

cudaError_t launch_epilogue_f32(const float *z, float *out, const F32Layer &L, int grid, cudaStream_t s) {
    epilogue_f32_kernel<<<grid, f32::THREADS, 0, s>>>(z, out, L);
    return cudaGetLastError();
}

}  // namespace trimul

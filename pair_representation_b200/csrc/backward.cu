// backward.cu - the LayerNorm, output-gate and input-gate adjoints of the
// triangle multiplicative update ("Scaling biomolecular modeling with context
// parallelism in NVIDIA BioNeMo", section "Context-parallel implementation of
// triangle multiplication": the layer's forward, differentiated by hand), and
// the final reduction of the weight gradients.
//
// These are the elementwise and per-cell steps of the backward; its GEMMs run
// on the tcgen05 pair kernel (contract_tc.cu). The per-cell kernels walk 64-cell tiles with 8 warps of
// 8 cells; lane l owns channels l, l + 32, l + 64 and l + 96, so shared-memory
// tiles are read without bank conflicts. Every kernel issues all global loads
// for 4 cells (read-only path) before it computes and stores, so each warp
// keeps several cells' loads in flight. Channel-major operands ([128][N][ld])
// move as 16-byte vectors of 8 cells and are transposed through a
// [64 cells][129] fp32 shared tile. Per-channel gradient sums are kept per
// lane, reduced over the block at the end and added with one atomic per
// channel and block. Grids are one wave of resident blocks.
#include "kernels.h"

namespace trimul {
namespace {

typedef __nv_bfloat16 bf;

constexpr int kTile = 64;               // cells per tile
constexpr int kWarps = 8;
constexpr int kCellsPerWarp = kTile / kWarps;
constexpr int kU = 4;                   // cells whose loads a warp issues together
constexpr int kThreads = kWarps * 32;
constexpr int kPitch = kC + 1;          // fp32 tile row: 128 channels + 1 pad word
constexpr int kCPL = kC / 32;           // channels per lane
constexpr size_t kTileBytes = (size_t)kTile * kPitch * sizeof(float);
constexpr size_t kRedBytes = (size_t)kWarps * kC * sizeof(float);
constexpr int kVecPerTile = kC * (kTile / 8);        // 16-byte vectors of 8 cells in a bf16 tile
constexpr int kVecPerThread = kVecPerTile / kThreads;
constexpr size_t kP = (size_t)kProjBlocks * kC;      // row length of P and D

__device__ __forceinline__ float ldbf(const bf *p, size_t i, float dflt) {
    return p ? __bfloat162float(__ldg(p + i)) : dflt;
}
__device__ __forceinline__ float ld(const bf *p) { return __bfloat162float(__ldg(p)); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__device__ __forceinline__ float sigmoid(float t) { return 1.f / (1.f + __expf(-t)); }

__device__ __forceinline__ void unpack8(const uint4 &u, float f[8]) {
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const float2 p = __bfloat1622float2(h[t]);
        f[2 * t] = p.x;
        f[2 * t + 1] = p.y;
    }
}

// Tiles of kA channel-major bf16 arrays, row segment (i, j0 .. j0 + 63), into
// tile[a][cell][channel]. A vector of 8 cells that starts inside the row ends
// within the row's pitch (ld is a multiple of 8), so it never leaves the row;
// cells past N hold whatever the padding holds and are not used.
template <int kA>
__device__ __forceinline__ void load_cm(const bf *const (&src)[kA], int N, size_t ld, int i, int j0,
                                        float *const (&tile)[kA]) {
    const size_t cs = (size_t)N * ld;
    uint4 v[kA][kVecPerThread];
#pragma unroll
    for (int a = 0; a < kA; ++a)
#pragma unroll
        for (int k = 0; k < kVecPerThread; ++k) {
            const int e = threadIdx.x + k * kThreads, c = e >> 3, j = j0 + 8 * (e & 7);
            v[a][k] = j < N ? __ldg(reinterpret_cast<const uint4 *>(src[a] + c * cs + (size_t)i * ld + j))
                            : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
    for (int a = 0; a < kA; ++a)
#pragma unroll
        for (int k = 0; k < kVecPerThread; ++k) {
            const int e = threadIdx.x + k * kThreads, c = e >> 3, jj = 8 * (e & 7);
            float f[8];
            unpack8(v[a][k], f);
#pragma unroll
            for (int t = 0; t < 8; ++t) tile[a][(jj + t) * kPitch + c] = f[t];
        }
}

// tile[cell][channel] back to a channel-major bf16 row segment in vectors of 8
// cells; a vector that starts below N also writes the padding cells after N,
// which the tile holds as 0.
__device__ __forceinline__ void store_cm(bf *dst, int N, size_t ld, int i, int j0, const float *tile) {
    const size_t cs = (size_t)N * ld;
#pragma unroll
    for (int k = 0; k < kVecPerThread; ++k) {
        const int e = threadIdx.x + k * kThreads, c = e >> 3, jj = 8 * (e & 7), j = j0 + jj;
        if (j >= N) continue;
        uint4 u;
        __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&u);
#pragma unroll
        for (int t = 0; t < 4; ++t)
            h[t] = __floats2bfloat162_rn(tile[(jj + 2 * t) * kPitch + c], tile[(jj + 2 * t + 1) * kPitch + c]);
        *reinterpret_cast<uint4 *>(dst + c * cs + (size_t)i * ld + j) = u;
    }
}

// Adds the block's per-lane channel sums acc[k][r] (channel lane + 32 r) to dst[k][128].
template <int K>
__device__ void flush_sums(const float (&acc)[K][kCPL], float *const (&dst)[K], float *red) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int k = 0; k < K; ++k) {
        __syncthreads();
#pragma unroll
        for (int r = 0; r < kCPL; ++r) red[warp * kC + lane + 32 * r] = acc[k][r];
        __syncthreads();
        if (threadIdx.x < kC && dst[k]) {
            float s = 0.f;
            for (int w = 0; w < kWarps; ++w) s += red[w * kC + threadIdx.x];
            atomicAdd(dst[k] + threadIdx.x, s);
        }
    }
}

struct TileIdx {
    int i, j0;
};
__device__ __forceinline__ TileIdx tile_of(long long t, int jt) {
    TileIdx x;
    x.i = (int)(t / jt);
    x.j0 = (int)(t % jt) * kTile;
    return x;
}

// ---- LayerNorm forward (recomputed statistics and normalised operand) ----------

template <bool kCM>
__global__ void __launch_bounds__(kThreads) ln_fwd_kernel(LnFwdArgs a) {
    extern __shared__ float tile[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int jt = (a.N + kTile - 1) / kTile;
    const long long tiles = (long long)a.N * jt;
    float gm[kCPL], bt[kCPL];
#pragma unroll
    for (int r = 0; r < kCPL; ++r) {
        gm[r] = ldbf(a.gamma, lane + 32 * r, 1.f);
        bt[r] = ldbf(a.beta, lane + 32 * r, 0.f);
    }
    for (long long t = blockIdx.x; t < tiles; t += gridDim.x) {
        const TileIdx ti = tile_of(t, jt);
        if (kCM) {
            const bf *src[1] = {a.src};
            float *const tl[1] = {tile};
            __syncthreads();
            load_cm<1>(src, a.N, a.ld, ti.i, ti.j0, tl);
            __syncthreads();
        }
        for (int q0 = 0; q0 < kCellsPerWarp; q0 += kU) {
            float v[kU][kCPL];
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int jj = warp * kCellsPerWarp + q0 + u, j = min(ti.j0 + jj, a.N - 1);
                const size_t m = (size_t)ti.i * a.N + j;
#pragma unroll
                for (int r = 0; r < kCPL; ++r)
                    v[u][r] = kCM ? tile[jj * kPitch + lane + 32 * r] : ld(a.src + m * kC + lane + 32 * r);
            }
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int jj = warp * kCellsPerWarp + q0 + u, j = ti.j0 + jj;
                if (j >= a.N) continue;
                const size_t m = (size_t)ti.i * a.N + j;
                float s = 0.f;
#pragma unroll
                for (int r = 0; r < kCPL; ++r) s += v[u][r];
                const float mu = warp_sum(s) * (1.f / kC);
                float ss = 0.f;
#pragma unroll
                for (int r = 0; r < kCPL; ++r) {
                    v[u][r] -= mu;
                    ss += v[u][r] * v[u][r];
                }
                const float rs = rsqrtf(warp_sum(ss) * (1.f / kC) + a.eps);
#pragma unroll
                for (int r = 0; r < kCPL; ++r)
                    a.out[m * kC + lane + 32 * r] = __float2bfloat16_rn(v[u][r] * rs * gm[r] + bt[r]);
                if (lane == 0) a.stats[m] = make_float2(mu, rs);
            }
        }
    }
}

// ---- LayerNorm adjoint ------------------------------------------------------------

template <bool kCM>
__global__ void __launch_bounds__(kThreads) ln_bwd_kernel(LnBwdArgs a) {
    extern __shared__ float smem[];
    float *tile = smem;
    float *red = smem + (kCM ? kTile * kPitch : 0);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int jt = (a.N + kTile - 1) / kTile;
    const long long tiles = (long long)a.N * jt;
    float gm[kCPL];
    float acc[2][kCPL] = {};
#pragma unroll
    for (int r = 0; r < kCPL; ++r) gm[r] = ldbf(a.gamma, lane + 32 * r, 1.f);
    for (long long t = blockIdx.x; t < tiles; t += gridDim.x) {
        const TileIdx ti = tile_of(t, jt);
        if (kCM) {
            const bf *src[1] = {a.src};
            float *const tl[1] = {tile};
            __syncthreads();
            load_cm<1>(src, a.N, a.ld, ti.i, ti.j0, tl);
            __syncthreads();
        }
        for (int q0 = 0; q0 < kCellsPerWarp; q0 += kU) {
            float v[kU][kCPL], g[kU][kCPL];
            float2 st[kU];
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int jj = warp * kCellsPerWarp + q0 + u, j = min(ti.j0 + jj, a.N - 1);
                const size_t m = (size_t)ti.i * a.N + j;
                st[u] = __ldg(a.stats + m);
#pragma unroll
                for (int r = 0; r < kCPL; ++r) {
                    const int c = lane + 32 * r;
                    v[u][r] = kCM ? tile[jj * kPitch + c] : ld(a.src + m * kC + c);
                    g[u][r] = __ldg(a.dh + m * kC + c);
                }
            }
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int jj = warp * kCellsPerWarp + q0 + u, j = ti.j0 + jj;
                if (j >= a.N) {
                    // Padding cell, stored with its vector: zero.
                    if (kCM)
#pragma unroll
                        for (int r = 0; r < kCPL; ++r) tile[jj * kPitch + lane + 32 * r] = 0.f;
                    continue;
                }
                const size_t m = (size_t)ti.i * a.N + j;
                float n[kCPL], dn[kCPL], s1 = 0.f, s2 = 0.f;
#pragma unroll
                for (int r = 0; r < kCPL; ++r) {
                    n[r] = (v[u][r] - st[u].x) * st[u].y;
                    dn[r] = g[u][r] * gm[r];
                    s1 += dn[r];
                    s2 += dn[r] * n[r];
                    acc[0][r] += g[u][r] * n[r];
                    acc[1][r] += g[u][r];
                }
                s1 = warp_sum(s1) * (1.f / kC);
                s2 = warp_sum(s2) * (1.f / kC);
#pragma unroll
                for (int r = 0; r < kCPL; ++r) {
                    const int c = lane + 32 * r;
                    const float dv = st[u].y * (dn[r] - s1 - n[r] * s2);
                    if (kCM)
                        tile[jj * kPitch + c] = dv;  // this warp's own cell row: no other warp touches it
                    else
                        a.dsrc[m * kC + c] = __float2bfloat16_rn(dv);
                }
            }
        }
        if (kCM) {
            __syncthreads();
            store_cm(a.dsrc, a.N, a.ld, ti.i, ti.j0, tile);
        }
    }
    float *const dst[2] = {a.dgamma, a.dbeta};
    flush_sums<2>(acc, dst, red);
}

// ---- output gate adjoint -------------------------------------------------------------

__global__ void __launch_bounds__(kThreads) gate_bwd_kernel(GateBwdArgs a) {
    __shared__ float red[kWarps * kC];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float bg[kCPL], bo[kCPL];
    float acc[2][kCPL] = {};
#pragma unroll
    for (int r = 0; r < kCPL; ++r) {
        bg[r] = ldbf(a.b_g, lane + 32 * r, 0.f);
        bo[r] = ldbf(a.b_o, lane + 32 * r, 0.f);
    }
    const long long tiles = (a.cells + kTile - 1) / kTile;
    for (long long t = blockIdx.x; t < tiles; t += gridDim.x) {
        for (int q0 = 0; q0 < kCellsPerWarp; q0 += kU) {
            float pg[kU][kCPL], y[kU][kCPL], d[kU][kCPL];
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const long long m = min(t * kTile + warp * kCellsPerWarp + q0 + u, a.cells - 1);
#pragma unroll
                for (int r = 0; r < kCPL; ++r) {
                    const int c = lane + 32 * r;
                    pg[u][r] = ld(a.P + m * kP + P_G * kC + c);
                    y[u][r] = ld(a.Y + m * kC + c);
                    d[u][r] = ld(a.dout + m * kC + c);
                }
            }
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const long long m = t * kTile + warp * kCellsPerWarp + q0 + u;
                if (m >= a.cells) continue;
#pragma unroll
                for (int r = 0; r < kCPL; ++r) {
                    const int c = lane + 32 * r;
                    const float g = sigmoid(pg[u][r] + bg[r]), yy = y[u][r] + bo[r];
                    const float dy = d[u][r] * g, dpg = d[u][r] * yy * g * (1.f - g);
                    a.dy[m * kC + c] = __float2bfloat16_rn(dy);
                    a.D[m * kP + P_G * kC + c] = __float2bfloat16_rn(dpg);
                    acc[0][r] += dpg;
                    acc[1][r] += dy;
                }
            }
        }
    }
    float *const dst[2] = {a.db_g, a.db_o};
    flush_sums<2>(acc, dst, red);
}

// ---- input gates and mask adjoint --------------------------------------------------------

__global__ void __launch_bounds__(kThreads) proj_bwd_kernel(ProjBwdArgs a) {
    extern __shared__ float smem[];
    float *tA = smem, *tB = smem + kTile * kPitch, *red = smem + 2 * kTile * kPitch;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int jt = (a.N + kTile - 1) / kTile;
    const long long tiles = (long long)a.N * jt;
    float bias[4][kCPL];
    float acc[4][kCPL] = {};
    const bf *bp[4] = {a.b_a, a.b_ag, a.b_b, a.b_bg};
#pragma unroll
    for (int k = 0; k < 4; ++k)
#pragma unroll
        for (int r = 0; r < kCPL; ++r) bias[k][r] = ldbf(bp[k], lane + 32 * r, 0.f);
    for (long long t = blockIdx.x; t < tiles; t += gridDim.x) {
        const TileIdx ti = tile_of(t, jt);
        {
            const bf *src[2] = {a.dA, a.dB};
            float *const tl[2] = {tA, tB};
            __syncthreads();
            load_cm<2>(src, a.N, a.ld, ti.i, ti.j0, tl);
            __syncthreads();
        }
        for (int q0 = 0; q0 < kCellsPerWarp; q0 += kU) {
            float p[kU][4][kCPL], mk[kU];
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int jj = warp * kCellsPerWarp + q0 + u, j = min(ti.j0 + jj, a.N - 1);
                const size_t m = (size_t)ti.i * a.N + j;
                mk[u] = ldbf(a.mask, m, 1.f);
#pragma unroll
                for (int k = 0; k < 4; ++k)
#pragma unroll
                    for (int r = 0; r < kCPL; ++r) p[u][k][r] = ld(a.P + m * kP + (P_A + k) * kC + lane + 32 * r);
            }
#pragma unroll
            for (int u = 0; u < kU; ++u) {
                const int jj = warp * kCellsPerWarp + q0 + u, j = ti.j0 + jj;
                if (j >= a.N) continue;
                const size_t m = (size_t)ti.i * a.N + j;
                bf *d = a.D + m * kP;
#pragma unroll
                for (int r = 0; r < kCPL; ++r) {
                    const int c = lane + 32 * r;
                    const float da = tA[jj * kPitch + c] * mk[u], db = tB[jj * kPitch + c] * mk[u];
                    const float pa = p[u][0][r] + bias[0][r], pb = p[u][2][r] + bias[2][r];
                    const float sa = sigmoid(p[u][1][r] + bias[1][r]), sb = sigmoid(p[u][3][r] + bias[3][r]);
                    const float g0 = da * sa, g1 = da * pa * sa * (1.f - sa);
                    const float g2 = db * sb, g3 = db * pb * sb * (1.f - sb);
                    d[P_A * kC + c] = __float2bfloat16_rn(g0);
                    d[P_AG * kC + c] = __float2bfloat16_rn(g1);
                    d[P_B * kC + c] = __float2bfloat16_rn(g2);
                    d[P_BG * kC + c] = __float2bfloat16_rn(g3);
                    acc[0][r] += g0;
                    acc[1][r] += g1;
                    acc[2][r] += g2;
                    acc[3][r] += g3;
                }
            }
        }
    }
    float *const dst[4] = {a.db, a.db + kC, a.db + 2 * kC, a.db + 3 * kC};
    flush_sums<4>(acc, dst, red);
}

// ---- weight gradients: sum of the per-chunk GEMM partials, in double ---------------------

__global__ void __launch_bounds__(256) wgrad_reduce_kernel(WgradReduceArgs a) {
    constexpr int kPer = kC * kC;
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= kWgradRows * kC) return;
    double s = 0.0;
    for (int k = 0; k < a.slots; ++k) s += (double)__ldg(a.partial + (size_t)k * kWgradRows * kC + e);
    float *dst = nullptr;
#pragma unroll
    for (int k = 0; k <= kProjBlocks; ++k)
        if (e / kPer == k) dst = a.dst[k];
    if (dst) dst[e % kPer] = (float)s;
}

size_t ln_fwd_smem(bool cm) { return cm ? kTileBytes : 0; }
size_t ln_bwd_smem(bool cm) { return (cm ? kTileBytes : 0) + kRedBytes; }
constexpr size_t kProjSmem = 2 * kTileBytes + kRedBytes;

// One wave: the resident blocks of the kernel on all SMs, at most `work`.
template <typename K>
int wave(K kernel, size_t smem, int sms, long long work) {
    int per = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, kernel, kThreads, smem) != cudaSuccess || per < 1) per = 1;
    const long long g = (long long)per * sms;
    return (int)(work < g ? work : g);
}

long long tiles_of(int N) { return (long long)N * ((N + kTile - 1) / kTile); }

}  // namespace

cudaError_t backward_setup() {
    cudaError_t e = cudaFuncSetAttribute(proj_bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kProjSmem);
    if (e == cudaSuccess)
        e = cudaFuncSetAttribute(ln_bwd_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)ln_bwd_smem(true));
    return e;
}

cudaError_t launch_ln_fwd(const LnFwdArgs &a, int sms, cudaStream_t s) {
    if (a.channel_major) {
        const size_t sm = ln_fwd_smem(true);
        ln_fwd_kernel<true><<<wave(ln_fwd_kernel<true>, sm, sms, tiles_of(a.N)), kThreads, sm, s>>>(a);
    } else {
        ln_fwd_kernel<false><<<wave(ln_fwd_kernel<false>, 0, sms, tiles_of(a.N)), kThreads, 0, s>>>(a);
    }
    return cudaGetLastError();
}

cudaError_t launch_ln_bwd(const LnBwdArgs &a, int sms, cudaStream_t s) {
    if (a.channel_major) {
        const size_t sm = ln_bwd_smem(true);
        ln_bwd_kernel<true><<<wave(ln_bwd_kernel<true>, sm, sms, tiles_of(a.N)), kThreads, sm, s>>>(a);
    } else {
        const size_t sm = ln_bwd_smem(false);
        ln_bwd_kernel<false><<<wave(ln_bwd_kernel<false>, sm, sms, tiles_of(a.N)), kThreads, sm, s>>>(a);
    }
    return cudaGetLastError();
}

cudaError_t launch_gate_bwd(const GateBwdArgs &a, int sms, cudaStream_t s) {
    gate_bwd_kernel<<<wave(gate_bwd_kernel, 0, sms, (a.cells + kTile - 1) / kTile), kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_proj_bwd(const ProjBwdArgs &a, int sms, cudaStream_t s) {
    proj_bwd_kernel<<<wave(proj_bwd_kernel, kProjSmem, sms, tiles_of(a.N)), kThreads, kProjSmem, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_wgrad_reduce(const WgradReduceArgs &a, cudaStream_t s) {
    wgrad_reduce_kernel<<<(kWgradRows * kC + 255) / 256, 256, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace trimul

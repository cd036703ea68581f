// backward.cu - the LayerNorm, output-gate and input-gate adjoints of the
// triangle multiplicative update ("Scaling biomolecular modeling with context
// parallelism in NVIDIA BioNeMo", section "Context-parallel implementation of
// triangle multiplication": the layer's forward, differentiated by hand), and
// the final reduction of the weight gradients.
//
// These are the elementwise and per-cell steps of the backward; its GEMMs run
// on the tcgen05 pair kernel (contract_tc.cu). The per-cell kernels walk
// 64-cell tiles with 8 warps of 8 cells. Half a warp serves one cell: lane q
// of the half owns channels 8q .. 8q + 7 and moves them as one 16-byte vector,
// so a warp reads or writes two whole 256-byte cell rows per instruction.
// Every kernel issues all global loads of its warp's 8 cells (read-only path)
// before it computes and stores. Channel-major operands ([128][N][ld]) move as
// 16-byte vectors of 8 cells and are transposed through a [64 cells][128
// channels] bf16 shared tile whose 16-byte chunks are XOR-swizzled by the
// cell's group of eight, which keeps both the transposing accesses and the
// per-cell vector accesses free of bank conflicts. Per-channel gradient sums
// are kept per lane, reduced over the block at the end and added with one
// atomic per channel and block. Grids are one wave of resident blocks.
#include "kernels.h"
#include "tile_ops.cuh"

namespace trimul {
namespace {

typedef __nv_bfloat16 bf;

constexpr int kTile = 64;               // cells per tile
constexpr int kWarps = 8;
constexpr int kCellsPerWarp = kTile / kWarps;
constexpr int kPairs = kCellsPerWarp / 2;    // cell pairs per warp and tile (one cell per half warp)
constexpr int kThreads = kWarps * 32;
constexpr int kChunks = kC / 8;         // 16-byte chunks of a cell row = lanes per cell
constexpr size_t kTileBytes = (size_t)kTile * kC * sizeof(bf);
constexpr size_t kRedBytes = (size_t)kWarps * kC * sizeof(float);
constexpr int kVecPerTile = kC * (kTile / 8);        // 16-byte vectors of 8 cells in a channel-major tile
constexpr int kVecPerThread = kVecPerTile / kThreads;
constexpr size_t kP = (size_t)kProjBlocks * kC;      // row length of P and D

static_assert(kChunks == 16 && kCellsPerWarp == 8, "half a warp per 128-channel cell, two cells per warp step");

__device__ __forceinline__ float ld(const bf *p) { return __bfloat162float(__ldg(p)); }
__device__ __forceinline__ uint4 ldg16(const void *p) { return __ldg(reinterpret_cast<const uint4 *>(p)); }
__device__ __forceinline__ void st16(void *p, const uint4 &v) { *reinterpret_cast<uint4 *>(p) = v; }

// Eight per-channel parameters c0 .. c0 + 7 (dflt for a null pointer).
__device__ __forceinline__ void ld8(const bf *p, int c0, float dflt, float f[8]) {
#pragma unroll
    for (int t = 0; t < 8; ++t) f[t] = p ? ld(p + c0 + t) : dflt;
}

// Sum over the 16 lanes of this half warp (one cell).
__device__ __forceinline__ float half_sum(float v) {
#pragma unroll
    for (int o = 8; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// sigma(t) = (1 + tanh(t / 2)) / 2: one MUFU operation (tanh.approx, relative
// error about 2^-11, far below the bf16 rounding of every output it feeds).
__device__ __forceinline__ float sigmoid(float t) { return fmaf(0.5f, tanh_approx(0.5f * t), 0.5f); }

__device__ __forceinline__ void unpack8(const uint4 &u, float f[8]) {
    const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&u);
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        const float2 p = __bfloat1622float2(h[t]);
        f[2 * t] = p.x;
        f[2 * t + 1] = p.y;
    }
}

__device__ __forceinline__ float2 bf2f(uint32_t w) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&w));
}
__device__ __forceinline__ uint32_t f2bf(float x, float y) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(x, y);
    return *reinterpret_cast<const uint32_t *>(&h);
}

__device__ __forceinline__ uint4 pack8(const float f[8]) {
    uint4 u;
    __nv_bfloat162 *h = reinterpret_cast<__nv_bfloat162 *>(&u);
#pragma unroll
    for (int t = 0; t < 4; ++t) h[t] = __floats2bfloat162_rn(f[2 * t], f[2 * t + 1]);
    return u;
}

// Index (in 16-byte chunks) of channels 8q .. 8q + 7 of cell jj in a bf16 tile.
// The XOR with the cell's group of eight spreads a transposing access (8
// consecutive cells of one channel in a vector, 8 vectors per warp) and a
// quarter warp's per-cell access (8 chunks of one cell) over all 32 banks.
__device__ __forceinline__ int chunk_at(int jj, int q) { return jj * kChunks + (q ^ ((jj >> 3) & 7)); }

// Tiles of kA channel-major bf16 arrays, row segment (i, j0 .. j0 + 63), into
// tile[a] (bf16 [cell][channel], swizzled). A vector of 8 cells that starts
// inside the row ends within the row's pitch (ld is a multiple of 8), so it
// never leaves the row; cells past N hold whatever the padding holds and are
// not used.
template <int kA>
__device__ __forceinline__ void load_cm(const bf *const (&src)[kA], int N, size_t ld, int i, int j0,
                                        uint4 *const (&tile)[kA]) {
    const size_t cs = (size_t)N * ld;
    uint4 v[kA][kVecPerThread];
#pragma unroll
    for (int a = 0; a < kA; ++a)
#pragma unroll
        for (int k = 0; k < kVecPerThread; ++k) {
            const int e = threadIdx.x + k * kThreads, c = e >> 3, j = j0 + 8 * (e & 7);
            v[a][k] = j < N ? ldg16(src[a] + c * cs + (size_t)i * ld + j) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
    for (int a = 0; a < kA; ++a) {
        unsigned short *tb = reinterpret_cast<unsigned short *>(tile[a]);
#pragma unroll
        for (int k = 0; k < kVecPerThread; ++k) {
            const int e = threadIdx.x + k * kThreads, c = e >> 3, jj = 8 * (e & 7);
            const uint32_t w[4] = {v[a][k].x, v[a][k].y, v[a][k].z, v[a][k].w};
#pragma unroll
            for (int t = 0; t < 8; ++t)
                tb[chunk_at(jj + t, c >> 3) * 8 + (c & 7)] = (unsigned short)(w[t >> 1] >> (16 * (t & 1)));
        }
    }
}

// A bf16 tile back to a channel-major row segment in vectors of 8 cells; a
// vector that starts below N also writes the padding cells after N, which the
// tile holds as 0.
__device__ __forceinline__ void store_cm(bf *dst, int N, size_t ld, int i, int j0, const uint4 *tile) {
    const size_t cs = (size_t)N * ld;
    const unsigned short *tb = reinterpret_cast<const unsigned short *>(tile);
#pragma unroll
    for (int k = 0; k < kVecPerThread; ++k) {
        const int e = threadIdx.x + k * kThreads, c = e >> 3, jj = 8 * (e & 7), j = j0 + jj;
        if (j >= N) continue;
        uint32_t w[4];
#pragma unroll
        for (int t = 0; t < 4; ++t)
            w[t] = (uint32_t)tb[chunk_at(jj + 2 * t, c >> 3) * 8 + (c & 7)] |
                   ((uint32_t)tb[chunk_at(jj + 2 * t + 1, c >> 3) * 8 + (c & 7)] << 16);
        st16(dst + c * cs + (size_t)i * ld + j, make_uint4(w[0], w[1], w[2], w[3]));
    }
}

// Adds the block's per-lane channel sums acc[k][t] (channel 8 (lane % 16) + t)
// to dst[k][128].
template <int K>
__device__ void flush_sums(float (&acc)[K][8], float *const (&dst)[K], float *red) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll
    for (int k = 0; k < K; ++k) {
#pragma unroll
        for (int t = 0; t < 8; ++t) acc[k][t] += __shfl_xor_sync(0xffffffffu, acc[k][t], 16);
        __syncthreads();
        if (lane < kChunks)
#pragma unroll
            for (int t = 0; t < 8; ++t) red[warp * kC + 8 * lane + t] = acc[k][t];
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

// The tile cell of pair u for this half warp.
__device__ __forceinline__ int cell_of(int warp, int u) { return warp * kCellsPerWarp + 2 * u + (threadIdx.x >> 4 & 1); }

// ---- LayerNorm forward (recomputed statistics and normalised operand) ----------

template <bool kCM>
__global__ void __launch_bounds__(kThreads, 2) ln_fwd_kernel(LnFwdArgs a) {
    extern __shared__ uint4 tile[];
    const int warp = threadIdx.x >> 5, q = threadIdx.x & 15, c0 = 8 * q;
    const int jt = (a.N + kTile - 1) / kTile;
    const long long tiles = (long long)a.N * jt;
    float gm[8], bt[8];
    ld8(a.gamma, c0, 1.f, gm);
    ld8(a.beta, c0, 0.f, bt);
    for (long long t = blockIdx.x; t < tiles; t += gridDim.x) {
        const TileIdx ti = tile_of(t, jt);
        if (kCM) {
            const bf *src[1] = {a.src};
            uint4 *const tl[1] = {tile};
            __syncthreads();
            load_cm<1>(src, a.N, a.ld, ti.i, ti.j0, tl);
            __syncthreads();
        }
        uint4 raw[kPairs];
#pragma unroll
        for (int u = 0; u < kPairs; ++u) {
            const int jj = cell_of(warp, u), j = min(ti.j0 + jj, a.N - 1);
            const size_t m = (size_t)ti.i * a.N + j;
            raw[u] = kCM ? tile[chunk_at(jj, q)] : ldg16(a.src + m * kC + c0);
        }
        // Both halves take every shuffle: a cell past N computes on a clamped copy and stores nothing.
#pragma unroll
        for (int u = 0; u < kPairs; ++u) {
            const int j = ti.j0 + cell_of(warp, u);
            const size_t m = (size_t)ti.i * a.N + j;
            float v[8], s = 0.f, ss = 0.f;
            unpack8(raw[u], v);
#pragma unroll
            for (int k = 0; k < 8; ++k) s += v[k];
            const float mu = half_sum(s) * (1.f / kC);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                v[k] -= mu;
                ss += v[k] * v[k];
            }
            const float rs = rsqrtf(half_sum(ss) * (1.f / kC) + a.eps);
#pragma unroll
            for (int k = 0; k < 8; ++k) v[k] = v[k] * rs * gm[k] + bt[k];
            if (j < a.N) {
                st16(a.out + m * kC + c0, pack8(v));
                if (q == 0) a.stats[m] = make_float2(mu, rs);
            }
        }
    }
}

// ---- LayerNorm adjoint ------------------------------------------------------------

template <bool kCM>
__global__ void __launch_bounds__(kThreads, 2) ln_bwd_kernel(LnBwdArgs a) {
    extern __shared__ uint4 smem4[];
    uint4 *tile = smem4;
    float *red = reinterpret_cast<float *>(smem4 + (kCM ? kTile * kChunks : 0));
    const int warp = threadIdx.x >> 5, q = threadIdx.x & 15, c0 = 8 * q;
    const int jt = (a.N + kTile - 1) / kTile;
    const long long tiles = (long long)a.N * jt;
    float gm[8];
    float acc[2][8] = {};
    ld8(a.gamma, c0, 1.f, gm);
    for (long long t = blockIdx.x; t < tiles; t += gridDim.x) {
        const TileIdx ti = tile_of(t, jt);
        if (kCM) {
            const bf *src[1] = {a.src};
            uint4 *const tl[1] = {tile};
            __syncthreads();
            load_cm<1>(src, a.N, a.ld, ti.i, ti.j0, tl);
            __syncthreads();
        }
        uint4 raw[kPairs];
        float4 g[kPairs][2];
        float2 st[kPairs];
#pragma unroll
        for (int u = 0; u < kPairs; ++u) {
            const int jj = cell_of(warp, u), j = min(ti.j0 + jj, a.N - 1);
            const size_t m = (size_t)ti.i * a.N + j;
            st[u] = __ldg(a.stats + m);
            raw[u] = kCM ? tile[chunk_at(jj, q)] : ldg16(a.src + m * kC + c0);
            g[u][0] = __ldg(reinterpret_cast<const float4 *>(a.dh + m * kC + c0));
            g[u][1] = __ldg(reinterpret_cast<const float4 *>(a.dh + m * kC + c0 + 4));
        }
#pragma unroll
        for (int u = 0; u < kPairs; ++u) {
            const int jj = cell_of(warp, u), j = ti.j0 + jj;
            const bool valid = j < a.N;
            const size_t m = (size_t)ti.i * a.N + j;
            const float gg[8] = {g[u][0].x, g[u][0].y, g[u][0].z, g[u][0].w,
                                 g[u][1].x, g[u][1].y, g[u][1].z, g[u][1].w};
            float v[8], n[8], dn[8], s1 = 0.f, s2 = 0.f;
            unpack8(raw[u], v);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                n[k] = (v[k] - st[u].x) * st[u].y;
                dn[k] = gg[k] * gm[k];
                s1 += dn[k];
                s2 += dn[k] * n[k];
                if (valid) {
                    acc[0][k] += gg[k] * n[k];
                    acc[1][k] += gg[k];
                }
            }
            s1 = half_sum(s1) * (1.f / kC);
            s2 = half_sum(s2) * (1.f / kC);
#pragma unroll
            for (int k = 0; k < 8; ++k) v[k] = st[u].y * (dn[k] - s1 - n[k] * s2);
            if (kCM)  // this half warp's own cell row: no other thread touches it; padding cells store 0
                tile[chunk_at(jj, q)] = valid ? pack8(v) : make_uint4(0, 0, 0, 0);
            else if (valid)
                st16(a.dsrc + m * kC + c0, pack8(v));
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

__global__ void __launch_bounds__(kThreads, 2) gate_bwd_kernel(GateBwdArgs a) {
    __shared__ float red[kWarps * kC];
    const int warp = threadIdx.x >> 5, q = threadIdx.x & 15, c0 = 8 * q;
    float bg[8], bo[8];
    float acc[2][8] = {};
    ld8(a.b_g, c0, 0.f, bg);
    ld8(a.b_o, c0, 0.f, bo);
    const long long tiles = (a.cells + kTile - 1) / kTile;
    for (long long t = blockIdx.x; t < tiles; t += gridDim.x) {
        uint4 pg[kPairs], y[kPairs], d[kPairs];
#pragma unroll
        for (int u = 0; u < kPairs; ++u) {
            const long long m = min(t * kTile + cell_of(warp, u), a.cells - 1);
            pg[u] = ldg16(a.P + m * kP + P_G * kC + c0);
            y[u] = ldg16(a.Y + m * kC + c0);
            d[u] = ldg16(a.dout + m * kC + c0);
        }
#pragma unroll
        for (int u = 0; u < kPairs; ++u) {
            const long long m = t * kTile + cell_of(warp, u);
            if (m >= a.cells) continue;
            float fp[8], fy[8], fd[8], dy[8], dpg[8];
            unpack8(pg[u], fp);
            unpack8(y[u], fy);
            unpack8(d[u], fd);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const float gt = sigmoid(fp[k] + bg[k]), yy = fy[k] + bo[k];
                dy[k] = fd[k] * gt;
                dpg[k] = fd[k] * yy * gt * (1.f - gt);
                acc[0][k] += dpg[k];
                acc[1][k] += dy[k];
            }
            st16(a.dy + m * kC + c0, pack8(dy));
            st16(a.D + m * kP + P_G * kC + c0, pack8(dpg));
        }
    }
    float *const dst[2] = {a.db_g, a.db_o};
    flush_sums<2>(acc, dst, red);
}

// ---- input gates and mask adjoint --------------------------------------------------------
//
// The largest per-cell pass (about 2.5 KB per cell). Its inputs move by
// asynchronous 16-byte copies (cp.async, no registers held) into a two-stage
// shared-memory ring, one tile ahead of the compute, on 32-cell tiles: a stage
// holds P's blocks P_A .. P_BG of the tile's cells ([cell][block][channel],
// 32 KB) and the channel-major dA and dB row segments as they lie in memory
// ([array][channel][4 vectors of 8 cells], 16 KB), which are transposed into
// swizzled cell-major tiles before the compute. Two blocks of 256 threads per
// SM, so that one block computes while the other waits at its barriers.

__device__ __forceinline__ void cp_async16(void *dst, const void *src, bool valid) {
    const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(d), "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }

constexpr int kPT = 32;                                  // cells per tile of this pass
constexpr int kProjPChunks = kPT * 4 * kChunks;          // P_A .. P_BG of one tile, 16-byte chunks
constexpr int kProjRChunks = 2 * kC * (kPT / 8);         // raw dA, dB row segments
constexpr int kProjStage = kProjPChunks + kProjRChunks;  // in 16-byte chunks
constexpr int kProjT = kPT * kChunks;                    // one transposed tile, in chunks
constexpr size_t kProjSmem = (size_t)(2 * kProjStage + 2 * kProjT) * 16 + 2 * kPT * sizeof(float);
static_assert(kProjPChunks % kThreads == 0 && kProjRChunks % kThreads == 0, "copies split evenly");
static_assert(2 * kProjT * 16 >= kRedBytes, "block sums reuse the transposed tiles");
static_assert(2 * (kProjSmem + 1024) <= 228 * 1024, "two blocks per SM");

struct ProjTile {
    int i, j0;
    bool live;
};
__device__ __forceinline__ ProjTile proj_tile(long long t, long long tiles, int jt) {
    ProjTile p;
    p.live = t < tiles;
    p.i = p.live ? (int)(t / jt) : 0;
    p.j0 = p.live ? (int)(t % jt) * kPT : 0;
    return p;
}

// Issues the copies of one tile into stage `st` (none for a dead tile; the
// caller commits a group either way, so that group counting stays uniform).
// Chunks of cells past N are zero-filled without a read.
__device__ __forceinline__ void proj_issue(const ProjBwdArgs &a, const ProjTile &ti, uint4 *st) {
    if (!ti.live) return;
    const size_t cs = (size_t)a.N * a.ld;
#pragma unroll
    for (int r = 0; r < kProjPChunks / kThreads; ++r) {
        const int x = threadIdx.x + r * kThreads, jj = x >> 6, k = (x >> 4) & 3, q = x & 15;
        const bool ok = ti.j0 + jj < a.N;
        const size_t m = (size_t)ti.i * a.N + (ok ? ti.j0 + jj : 0);
        cp_async16(st + x, a.P + m * kP + (P_A + k) * kC + 8 * q, ok);
    }
#pragma unroll
    for (int r = 0; r < kProjRChunks / kThreads; ++r) {
        const int y = threadIdx.x + r * kThreads, arr = y / (kC * kPT / 8), c = (y >> 2) & (kC - 1), g = y & 3;
        const bool ok = ti.j0 + 8 * g < a.N;
        const bf *src = (arr ? a.dB : a.dA) + c * cs + (size_t)ti.i * a.ld + (ok ? ti.j0 + 8 * g : 0);
        cp_async16(st + kProjPChunks + y, src, ok);
    }
}

__global__ void __launch_bounds__(kThreads, 2) proj_bwd_kernel(ProjBwdArgs a) {
    extern __shared__ uint4 smem4[];
    uint4 *const stage0 = smem4;
    uint4 *tA = smem4 + 2 * kProjStage, *tB = tA + kProjT;
    float *msk = reinterpret_cast<float *>(tB + kProjT);  // [2][kPT] mask per stage
    float *red = reinterpret_cast<float *>(tA);           // after the last tile
    const int warp = threadIdx.x >> 5, q = threadIdx.x & 15, c0 = 8 * q;
    const int jt = (a.N + kPT - 1) / kPT;
    const long long tiles = (long long)a.N * jt;
    // The four bias vectors stay bf16 (exact), two channels to a register.
    __nv_bfloat162 bias[4][4];
    float acc[4][8] = {};
    const bf *bp[4] = {a.b_a, a.b_ag, a.b_b, a.b_bg};
#pragma unroll
    for (int k = 0; k < 4; ++k)
#pragma unroll
        for (int t = 0; t < 4; ++t)
            bias[k][t] = bp[k] ? __halves2bfloat162(bp[k][c0 + 2 * t], bp[k][c0 + 2 * t + 1])
                               : __floats2bfloat162_rn(0.f, 0.f);
    const long long t0 = blockIdx.x, dt = gridDim.x;
    auto mask_of = [&](long long t) -> float {
        const ProjTile ti = proj_tile(t, tiles, jt);
        const int j = ti.j0 + (int)threadIdx.x;
        return a.mask && ti.live && j < a.N ? ld(a.mask + (size_t)ti.i * a.N + j) : 1.f;
    };
    proj_issue(a, proj_tile(t0, tiles, jt), stage0);
    cp_async_commit();
    proj_issue(a, proj_tile(t0 + dt, tiles, jt), stage0 + kProjStage);
    cp_async_commit();
    if (threadIdx.x < kPT) msk[threadIdx.x] = mask_of(t0);
    int s = 0;
    for (long long t = t0; t < tiles; t += dt, s ^= 1) {
        const ProjTile ti = proj_tile(t, tiles, jt);
        uint4 *const st = stage0 + s * kProjStage;
        asm volatile("cp.async.wait_group 1;\n" ::: "memory");  // this thread's copies of tile t landed
        __syncthreads();  // everyone's have; tA, tB and the other mask slot are free
        const float mnext = threadIdx.x < kPT ? mask_of(t + dt) : 1.f;
        {
            // Chunk (array, channel c, vector g) holds cells 8g .. 8g + 7 of channel c.
            const uint4 *raw = st + kProjPChunks;
#pragma unroll
            for (int r = 0; r < kProjRChunks / kThreads; ++r) {
                const int y = threadIdx.x + r * kThreads, arr = y / (kC * kPT / 8), c = (y >> 2) & (kC - 1);
                const int jj = 8 * (y & 3);
                const uint4 v = raw[y];
                unsigned short *tb = reinterpret_cast<unsigned short *>(arr ? tB : tA);
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    tb[chunk_at(jj + e, c >> 3) * 8 + (c & 7)] = (unsigned short)(w[e >> 1] >> (16 * (e & 1)));
            }
        }
        __syncthreads();
#pragma unroll 1
        for (int u = 0; u < kPT / kWarps / 2; ++u) {
            const int jj = warp * (kPT / kWarps) + 2 * u + (int)(threadIdx.x >> 4 & 1), j = ti.j0 + jj;
            if (j >= a.N) continue;
            const size_t m = (size_t)ti.i * a.N + j;
            const float mk = msk[s * kPT + jj];
            // Two channels at a time: the four outputs of channels c0 + 2e, c0 + 2e + 1
            // are packed as they are made, which keeps few values live.
            const uint4 ta = tA[chunk_at(jj, q)], tb = tB[chunk_at(jj, q)];
            const uint4 p0 = st[(jj * 4 + 0) * kChunks + q], p1 = st[(jj * 4 + 1) * kChunks + q];
            const uint4 p2 = st[(jj * 4 + 2) * kChunks + q], p3 = st[(jj * 4 + 3) * kChunks + q];
            const uint32_t wa[4] = {ta.x, ta.y, ta.z, ta.w}, wb[4] = {tb.x, tb.y, tb.z, tb.w};
            const uint32_t w0[4] = {p0.x, p0.y, p0.z, p0.w}, w1[4] = {p1.x, p1.y, p1.z, p1.w};
            const uint32_t w2[4] = {p2.x, p2.y, p2.z, p2.w}, w3[4] = {p3.x, p3.y, p3.z, p3.w};
            uint32_t o[4][4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float2 da = bf2f(wa[e]), db = bf2f(wb[e]);
                const float2 b0 = __bfloat1622float2(bias[0][e]), b1 = __bfloat1622float2(bias[1][e]);
                const float2 b2 = __bfloat1622float2(bias[2][e]), b3 = __bfloat1622float2(bias[3][e]);
                const float2 pa = bf2f(w0[e]), pag = bf2f(w1[e]), pb = bf2f(w2[e]), pbg = bf2f(w3[e]);
                float g[4][2];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const float dah = (h ? da.y : da.x) * mk, dbh = (h ? db.y : db.x) * mk;
                    const float sa = sigmoid((h ? pag.y : pag.x) + (h ? b1.y : b1.x));
                    const float sb = sigmoid((h ? pbg.y : pbg.x) + (h ? b3.y : b3.x));
                    g[0][h] = dah * sa;
                    g[1][h] = dah * ((h ? pa.y : pa.x) + (h ? b0.y : b0.x)) * sa * (1.f - sa);
                    g[2][h] = dbh * sb;
                    g[3][h] = dbh * ((h ? pb.y : pb.x) + (h ? b2.y : b2.x)) * sb * (1.f - sb);
                }
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    acc[k][2 * e] += g[k][0];
                    acc[k][2 * e + 1] += g[k][1];
                    o[k][e] = f2bf(g[k][0], g[k][1]);
                }
            }
            bf *d = a.D + m * kP + c0;
#pragma unroll
            for (int k = 0; k < 4; ++k) st16(d + (P_A + k) * kC, make_uint4(o[k][0], o[k][1], o[k][2], o[k][3]));
        }
        if (threadIdx.x < kPT) msk[(s ^ 1) * kPT + threadIdx.x] = mnext;
        __syncthreads();  // stage s is read out
        proj_issue(a, proj_tile(t + 2 * dt, tiles, jt), st);
        cp_async_commit();
    }
    asm volatile("cp.async.wait_group 0;\n" ::: "memory");
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
    if (e == cudaSuccess)  // all of the unified L1 as shared memory: room for two blocks per SM
        e = cudaFuncSetAttribute(proj_bwd_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
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
    proj_bwd_kernel<<<wave(proj_bwd_kernel, kProjSmem, sms, (long long)a.N * ((a.N + kPT - 1) / kPT)), kThreads, kProjSmem, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_wgrad_reduce(const WgradReduceArgs &a, cudaStream_t s) {
    wgrad_reduce_kernel<<<(kWgradRows * kC + 255) / 256, 256, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace trimul

// backward.cu - the LayerNorm, output-gate and input-gate adjoints of the
// triangle multiplicative update ("Scaling biomolecular modeling with context
// parallelism in NVIDIA BioNeMo", section "Context-parallel implementation of
// triangle multiplication": the layer's forward, differentiated by hand), and
// the reduction of the weight-gradient partials into sums in double. Each
// kernel works on one block of rows of the N x N grid (all of it, or as many
// rows as the caller's workspace holds).
//
// These are the elementwise and per-cell steps of the backward; its GEMMs run
// on the tcgen05 pair kernel (contract_tc.cu). Half a warp serves one cell:
// lane q of the half owns channels 8q .. 8q + 7 and moves them as one 16-byte
// vector, so a warp reads or writes two whole 256-byte cell rows per
// instruction. The passes over cell-major data alone walk 64-cell tiles with
// register loads, all of a warp's 8 cells issued before the first use. The
// passes with a channel-major operand ([128][N][ld]) walk 32-cell tiles whose
// inputs are staged by cp.async in a ring of shared-memory stages, tiles ahead
// of the compute; their channel-major row segments are transposed through a
// bf16 [cell][channel] tile whose 16-byte chunks are XOR-swizzled by the
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
constexpr size_t kRedBytes = (size_t)kWarps * kC * sizeof(float);
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

// ---- asynchronous copies and the 32-cell tiles they feed -----------------------------
//
// The passes with a channel-major operand (the LayerNorm forward and adjoint of
// x, and the input-gate adjoint) run on 32-cell tiles whose inputs move by
// cp.async (global -> shared, no register held) into a ring of stages, several
// tiles ahead of the compute, with two blocks per SM so that one block computes
// while the other waits at its barriers. A channel-major row segment lands as it
// lies in memory ([channel][4 vectors of 8 cells]) and is transposed into the
// swizzled cell-major tile before the compute.

// 16 (or 8) bytes global -> shared; valid == false fills zeros and reads nothing.
__device__ __forceinline__ void cp_async16(void *dst, const void *src, bool valid) {
    const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(d), "l"(src), "r"(valid ? 16 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async8(void *dst, const void *src, bool valid) {
    const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;\n" ::"r"(d), "l"(src), "r"(valid ? 8 : 0)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
// Waits until at most n of this thread's newest copy groups are still pending.
template <int n>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(n) : "memory");
}

constexpr int kPT = 32;                      // cells per tile of the cp.async passes
constexpr int kRawChunks = kC * (kPT / 8);   // one channel-major row segment, 16-byte chunks
constexpr int kTChunks = kPT * kChunks;      // one cell-major tile
static_assert(kRawChunks % kThreads == 0 && kTChunks * 16 >= (int)kRedBytes, "tile sizes");

struct PTile {
    int li, i, j0;  // row within the block, global row (i0 + li), first cell
    bool live;      // false past the last tile: nothing is copied
};
__device__ __forceinline__ PTile ptile(long long t, long long tiles, int jt, int i0) {
    PTile p;
    p.live = t < tiles;
    p.li = p.live ? (int)(t / jt) : 0;
    p.i = i0 + p.li;
    p.j0 = p.live ? (int)(t % jt) * kPT : 0;
    return p;
}
long long ptiles_of(int rows, int N) { return (long long)rows * ((N + kPT - 1) / kPT); }

// The tile cell of pair u (0 or 1) for this half warp.
__device__ __forceinline__ int pcell_of(int warp, int u) {
    return warp * (kPT / kWarps) + 2 * u + (threadIdx.x >> 4 & 1);
}

// Copies the row segment (row i, cells j0 .. j0 + 31, all channels) of a
// channel-major [128][N][ld] array to raw[channel * 4 + vector]. A vector that
// starts inside the row ends within the row's pitch (ld is a multiple of 8);
// vectors past N are zero-filled.
__device__ __forceinline__ void issue_raw(const bf *src, int N, size_t ld, const PTile &ti, uint4 *raw) {
    if (!ti.live) return;
    const size_t cs = (size_t)N * ld;
#pragma unroll
    for (int r = 0; r < kRawChunks / kThreads; ++r) {
        const int y = threadIdx.x + r * kThreads, c = y >> 2, g = y & 3;
        const bool ok = ti.j0 + 8 * g < N;
        cp_async16(raw + y, src + c * cs + (size_t)ti.i * ld + (ok ? ti.j0 + 8 * g : 0), ok);
    }
}

// raw (issue_raw's layout) -> the swizzled cell-major tile.
__device__ __forceinline__ void transpose_raw(const uint4 *raw, uint4 *tile) {
    unsigned short *tb = reinterpret_cast<unsigned short *>(tile);
#pragma unroll
    for (int r = 0; r < kRawChunks / kThreads; ++r) {
        const int y = threadIdx.x + r * kThreads, c = y >> 2, jj = 8 * (y & 3);
        const uint4 v = raw[y];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 8; ++e)
            tb[chunk_at(jj + e, c >> 3) * 8 + (c & 7)] = (unsigned short)(w[e >> 1] >> (16 * (e & 1)));
    }
}

// A cell-major tile back to a channel-major row segment in vectors of 8 cells; a
// vector that starts below N also writes the padding cells after N, which the
// tile holds as 0.
__device__ __forceinline__ void store_cm(bf *dst, int N, size_t ld, const PTile &ti, const uint4 *tile) {
    const size_t cs = (size_t)N * ld;
    const unsigned short *tb = reinterpret_cast<const unsigned short *>(tile);
#pragma unroll
    for (int r = 0; r < kRawChunks / kThreads; ++r) {
        const int y = threadIdx.x + r * kThreads, c = y >> 2, jj = 8 * (y & 3), j = ti.j0 + jj;
        if (j >= N) continue;
        uint32_t w[4];
#pragma unroll
        for (int t = 0; t < 4; ++t)
            w[t] = (uint32_t)tb[chunk_at(jj + 2 * t, c >> 3) * 8 + (c & 7)] |
                   ((uint32_t)tb[chunk_at(jj + 2 * t + 1, c >> 3) * 8 + (c & 7)] << 16);
        st16(dst + c * cs + (size_t)ti.i * ld + j, make_uint4(w[0], w[1], w[2], w[3]));
    }
}

// ---- LayerNorm forward (recomputed statistics and normalised operand) ----------

// One cell from this lane's 8 channels; both halves of the warp take every
// shuffle (a cell past N computes on whatever its chunk holds and stores nothing).
__device__ __forceinline__ void ln_fwd_cell(const uint4 &raw, const float (&gm)[8], const float (&bt)[8], float eps,
                                            bool valid, bf *out, float2 *stat) {
    float v[8], s = 0.f, ss = 0.f;
    unpack8(raw, v);
#pragma unroll
    for (int k = 0; k < 8; ++k) s += v[k];
    const float mu = half_sum(s) * (1.f / kC);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        v[k] -= mu;
        ss += v[k] * v[k];
    }
    const float rs = rsqrtf(half_sum(ss) * (1.f / kC) + eps);
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = v[k] * rs * gm[k] + bt[k];
    if (valid) {
        st16(out, pack8(v));
        if ((threadIdx.x & 15) == 0) *stat = make_float2(mu, rs);
    }
}

// Cell-major source ([cells][128]): 64-cell tiles, register loads.
__global__ void __launch_bounds__(kThreads, 2) ln_fwd_kernel(LnFwdArgs a) {
    const int warp = threadIdx.x >> 5, q = threadIdx.x & 15, c0 = 8 * q;
    const int jt = (a.N + kTile - 1) / kTile;
    const long long tiles = (long long)a.rows * jt;
    float gm[8], bt[8];
    ld8(a.gamma, c0, 1.f, gm);
    ld8(a.beta, c0, 0.f, bt);
    for (long long t = blockIdx.x; t < tiles; t += gridDim.x) {
        const TileIdx ti = tile_of(t, jt);
        uint4 raw[kPairs];
#pragma unroll
        for (int u = 0; u < kPairs; ++u) {
            const size_t m = (size_t)ti.i * a.N + min(ti.j0 + cell_of(warp, u), a.N - 1);
            raw[u] = ldg16(a.src + m * kC + c0);
        }
#pragma unroll
        for (int u = 0; u < kPairs; ++u) {
            const int j = ti.j0 + cell_of(warp, u);
            const size_t m = (size_t)ti.i * a.N + j;
            ln_fwd_cell(raw[u], gm, bt, a.eps, j < a.N, a.out + m * kC + c0, a.stats + m);
        }
    }
}

// Channel-major source ([128][N][ld]): 32-cell tiles through a ring of kLnFwdStages.
constexpr int kLnFwdStages = 6;
constexpr size_t kLnFwdCmSmem = (size_t)(kLnFwdStages * kRawChunks + kTChunks) * 16;

__global__ void __launch_bounds__(kThreads, 2) ln_fwd_cm_kernel(LnFwdArgs a) {
    extern __shared__ uint4 smem4[];
    uint4 *tile = smem4 + kLnFwdStages * kRawChunks;
    const int warp = threadIdx.x >> 5, q = threadIdx.x & 15, c0 = 8 * q;
    const int jt = (a.N + kPT - 1) / kPT;
    const long long tiles = (long long)a.rows * jt, t0 = blockIdx.x, dt = gridDim.x;
    float gm[8], bt[8];
    ld8(a.gamma, c0, 1.f, gm);
    ld8(a.beta, c0, 0.f, bt);
#pragma unroll
    for (int p = 0; p < kLnFwdStages - 1; ++p) {
        issue_raw(a.src, a.N, a.ld, ptile(t0 + p * dt, tiles, jt, a.i0), smem4 + p * kRawChunks);
        cp_async_commit();
    }
    int s = 0;
    for (long long t = t0; t < tiles; t += dt) {
        const PTile ti = ptile(t, tiles, jt, a.i0);
        cp_async_wait<kLnFwdStages - 2>();  // this thread's copies of tile t have landed
        __syncthreads();  // everyone's have; the previous tile's stage and the cell-major tile are free
        const int sn = s == 0 ? kLnFwdStages - 1 : s - 1;
        issue_raw(a.src, a.N, a.ld, ptile(t + (kLnFwdStages - 1) * dt, tiles, jt, a.i0), smem4 + sn * kRawChunks);
        cp_async_commit();
        transpose_raw(smem4 + s * kRawChunks, tile);
        __syncthreads();
#pragma unroll
        for (int u = 0; u < kPT / kWarps / 2; ++u) {
            const int jj = pcell_of(warp, u), j = ti.j0 + jj;
            const size_t m = (size_t)ti.li * a.N + j;
            ln_fwd_cell(tile[chunk_at(jj, q)], gm, bt, a.eps, j < a.N, a.out + m * kC + c0, a.stats + m);
        }
        s = s + 1 == kLnFwdStages ? 0 : s + 1;
    }
    cp_async_wait<0>();
}

// ---- LayerNorm adjoint ------------------------------------------------------------

// One cell: dsrc's 8 channels of this lane, packed; adds the cell's dgamma and
// dbeta terms to acc when it is valid. Both halves take every shuffle.
__device__ __forceinline__ uint4 ln_bwd_cell(const uint4 &raw, const float (&gg)[8], float2 st, const float (&gm)[8],
                                             bool valid, float (&acc)[2][8]) {
    float v[8], n[8], dn[8], s1 = 0.f, s2 = 0.f;
    unpack8(raw, v);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        n[k] = (v[k] - st.x) * st.y;
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
    for (int k = 0; k < 8; ++k) v[k] = st.y * (dn[k] - s1 - n[k] * s2);
    return pack8(v);
}

// Cell-major source and result: 64-cell tiles, register loads.
__global__ void __launch_bounds__(kThreads, 2) ln_bwd_kernel(LnBwdArgs a) {
    __shared__ float red[kWarps * kC];
    const int warp = threadIdx.x >> 5, q = threadIdx.x & 15, c0 = 8 * q;
    const int jt = (a.N + kTile - 1) / kTile;
    const long long tiles = (long long)a.rows * jt;
    float gm[8];
    float acc[2][8] = {};
    ld8(a.gamma, c0, 1.f, gm);
    for (long long t = blockIdx.x; t < tiles; t += gridDim.x) {
        const TileIdx ti = tile_of(t, jt);
        uint4 raw[kPairs];
        float4 g[kPairs][2];
        float2 st[kPairs];
#pragma unroll
        for (int u = 0; u < kPairs; ++u) {
            const size_t m = (size_t)ti.i * a.N + min(ti.j0 + cell_of(warp, u), a.N - 1);
            st[u] = __ldg(a.stats + m);
            raw[u] = ldg16(a.src + m * kC + c0);
            g[u][0] = __ldg(reinterpret_cast<const float4 *>(a.dh + m * kC + c0));
            g[u][1] = __ldg(reinterpret_cast<const float4 *>(a.dh + m * kC + c0 + 4));
        }
#pragma unroll
        for (int u = 0; u < kPairs; ++u) {
            const int j = ti.j0 + cell_of(warp, u);
            const size_t m = (size_t)ti.i * a.N + j;
            const float gg[8] = {g[u][0].x, g[u][0].y, g[u][0].z, g[u][0].w,
                                 g[u][1].x, g[u][1].y, g[u][1].z, g[u][1].w};
            const uint4 dv = ln_bwd_cell(raw[u], gg, st[u], gm, j < a.N, acc);
            if (j < a.N) st16(a.dsrc + m * kC + c0, dv);
        }
    }
    float *const dst[2] = {a.dgamma, a.dbeta};
    flush_sums<2>(acc, dst, red);
}

// Channel-major source and result: 32-cell tiles through a ring of kLnBwdStages.
// A stage holds the source row segment, dh of the tile's cells ([cell][32
// chunks of 4 floats], chunk p at p ^ ((p >> 3) & 1), which keeps a quarter
// warp's two reads per lane free of bank conflicts) and the cells' statistics.
constexpr int kLnBwdStages = 3;
constexpr int kDhChunks = kPT * (kC * 4 / 16);
constexpr int kStatChunks = kPT * 8 / 16;
constexpr int kLnBwdStage = kRawChunks + kDhChunks + kStatChunks;
constexpr size_t kLnBwdCmSmem = (size_t)(kLnBwdStages * kLnBwdStage + kTChunks) * 16;
static_assert(kDhChunks % kThreads == 0 && kPT <= kThreads, "copies split evenly");

__device__ __forceinline__ int dh_pos(int p) { return p ^ ((p >> 3) & 1); }

__device__ __forceinline__ void ln_bwd_issue(const LnBwdArgs &a, const PTile &ti, uint4 *st) {
    if (!ti.live) return;
    issue_raw(a.src, a.N, a.ld, ti, st);
#pragma unroll
    for (int r = 0; r < kDhChunks / kThreads; ++r) {
        const int z = threadIdx.x + r * kThreads, jj = z >> 5, p = z & 31;
        const bool ok = ti.j0 + jj < a.N;
        const size_t m = (size_t)ti.li * a.N + (ok ? ti.j0 + jj : 0);
        cp_async16(st + kRawChunks + jj * 32 + dh_pos(p), a.dh + m * kC + 4 * p, ok);
    }
    if (threadIdx.x < kPT) {
        const bool ok = ti.j0 + (int)threadIdx.x < a.N;
        const size_t m = (size_t)ti.li * a.N + (ok ? ti.j0 + threadIdx.x : 0);
        cp_async8(reinterpret_cast<float2 *>(st + kRawChunks + kDhChunks) + threadIdx.x, a.stats + m, ok);
    }
}

__global__ void __launch_bounds__(kThreads, 2) ln_bwd_cm_kernel(LnBwdArgs a) {
    extern __shared__ uint4 smem4[];
    uint4 *tile = smem4 + kLnBwdStages * kLnBwdStage;
    float *red = reinterpret_cast<float *>(tile);  // after the last tile
    const int warp = threadIdx.x >> 5, q = threadIdx.x & 15, c0 = 8 * q;
    const int jt = (a.N + kPT - 1) / kPT;
    const long long tiles = (long long)a.rows * jt, t0 = blockIdx.x, dt = gridDim.x;
    float gm[8];
    float acc[2][8] = {};
    ld8(a.gamma, c0, 1.f, gm);
#pragma unroll
    for (int p = 0; p < kLnBwdStages - 1; ++p) {
        ln_bwd_issue(a, ptile(t0 + p * dt, tiles, jt, a.i0), smem4 + p * kLnBwdStage);
        cp_async_commit();
    }
    int s = 0;
    for (long long t = t0; t < tiles; t += dt) {
        const PTile ti = ptile(t, tiles, jt, a.i0);
        const uint4 *st = smem4 + s * kLnBwdStage;
        cp_async_wait<kLnBwdStages - 2>();  // this thread's copies of tile t have landed
        __syncthreads();  // everyone's have; the previous tile's stage and the cell-major tile are free
        const int sn = s == 0 ? kLnBwdStages - 1 : s - 1;
        ln_bwd_issue(a, ptile(t + (kLnBwdStages - 1) * dt, tiles, jt, a.i0), smem4 + sn * kLnBwdStage);
        cp_async_commit();
        transpose_raw(st, tile);
        __syncthreads();
        const float4 *dh = reinterpret_cast<const float4 *>(st + kRawChunks);
        const float2 *stats = reinterpret_cast<const float2 *>(st + kRawChunks + kDhChunks);
#pragma unroll
        for (int u = 0; u < kPT / kWarps / 2; ++u) {
            const int jj = pcell_of(warp, u);
            const bool valid = ti.j0 + jj < a.N;
            const float4 g0 = dh[jj * 32 + dh_pos(2 * q)], g1 = dh[jj * 32 + dh_pos(2 * q + 1)];
            const float gg[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
            const uint4 dv = ln_bwd_cell(tile[chunk_at(jj, q)], gg, stats[jj], gm, valid, acc);
            // This half warp's own cell row: no other thread touches it; padding cells store 0.
            tile[chunk_at(jj, q)] = valid ? dv : make_uint4(0, 0, 0, 0);
        }
        __syncthreads();
        store_cm(a.dsrc, a.N, a.ld, ti, tile);
        s = s + 1 == kLnBwdStages ? 0 : s + 1;
    }
    cp_async_wait<0>();
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
            st16(a.dg + m * a.dg_stride + c0, pack8(dpg));
        }
    }
    float *const dst[2] = {a.db_g, a.db_o};
    flush_sums<2>(acc, dst, red);
}

// ---- input gates and mask adjoint --------------------------------------------------------
//
// The largest per-cell pass (about 2.5 KB per cell), on 32-cell tiles through a
// two-stage ring: a stage holds P's blocks P_A .. P_BG of the tile's cells
// ([cell][block][channel], 32 KB) and the dA and dB row segments (8 KB each).

constexpr int kProjPChunks = kPT * 4 * kChunks;               // P_A .. P_BG of one tile
constexpr int kProjStage = kProjPChunks + 2 * kRawChunks;     // in 16-byte chunks
constexpr size_t kProjSmem = (size_t)(2 * kProjStage + 2 * kTChunks) * 16 + 2 * kPT * sizeof(float);
static_assert(kProjPChunks % kThreads == 0, "copies split evenly");
static_assert(2 * (kProjSmem + 1024) <= 228 * 1024, "two blocks per SM");

// The copies of one tile into stage st; chunks of cells past N are zero-filled.
__device__ __forceinline__ void proj_issue(const ProjBwdArgs &a, const PTile &ti, uint4 *st) {
    if (!ti.live) return;
#pragma unroll
    for (int r = 0; r < kProjPChunks / kThreads; ++r) {
        const int x = threadIdx.x + r * kThreads, jj = x >> 6, k = (x >> 4) & 3, q = x & 15;
        const bool ok = ti.j0 + jj < a.N;
        const size_t m = (size_t)ti.li * a.N + (ok ? ti.j0 + jj : 0);
        cp_async16(st + x, a.P + m * kP + (P_A + k) * kC + 8 * q, ok);
    }
    issue_raw(a.dA, a.N, a.ld, ti, st + kProjPChunks);
    issue_raw(a.dB, a.N, a.ld, ti, st + kProjPChunks + kRawChunks);
}

__global__ void __launch_bounds__(kThreads, 2) proj_bwd_kernel(ProjBwdArgs a) {
    extern __shared__ uint4 smem4[];
    uint4 *tA = smem4 + 2 * kProjStage, *tB = tA + kTChunks;
    float *msk = reinterpret_cast<float *>(tB + kTChunks);  // [2][kPT] mask per stage
    float *red = reinterpret_cast<float *>(tA);             // after the last tile
    const int warp = threadIdx.x >> 5, q = threadIdx.x & 15, c0 = 8 * q;
    const int jt = (a.N + kPT - 1) / kPT;
    const long long tiles = (long long)a.rows * jt, t0 = blockIdx.x, dt = gridDim.x;
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
    auto mask_of = [&](long long t) -> float {
        const PTile ti = ptile(t, tiles, jt, a.i0);
        const int j = ti.j0 + (int)threadIdx.x;
        return a.mask && ti.live && j < a.N ? ld(a.mask + (size_t)ti.i * a.N + j) : 1.f;
    };
    proj_issue(a, ptile(t0, tiles, jt, a.i0), smem4);
    cp_async_commit();
    proj_issue(a, ptile(t0 + dt, tiles, jt, a.i0), smem4 + kProjStage);
    cp_async_commit();
    if (threadIdx.x < kPT) msk[threadIdx.x] = mask_of(t0);
    int s = 0;
    for (long long t = t0; t < tiles; t += dt, s ^= 1) {
        const PTile ti = ptile(t, tiles, jt, a.i0);
        uint4 *const st = smem4 + s * kProjStage;
        cp_async_wait<1>();  // this thread's copies of tile t have landed
        __syncthreads();     // everyone's have; tA, tB and the other mask slot are free
        const float mnext = threadIdx.x < kPT ? mask_of(t + dt) : 1.f;
        transpose_raw(st + kProjPChunks, tA);
        transpose_raw(st + kProjPChunks + kRawChunks, tB);
        __syncthreads();
#pragma unroll 1
        for (int u = 0; u < kPT / kWarps / 2; ++u) {
            const int jj = pcell_of(warp, u), j = ti.j0 + jj;
            if (j >= a.N) continue;
            const size_t m = (size_t)ti.li * a.N + j;
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
        proj_issue(a, ptile(t + 2 * dt, tiles, jt, a.i0), st);
        cp_async_commit();
    }
    cp_async_wait<0>();
    float *const dst[4] = {a.db, a.db + kC, a.db + 2 * kC, a.db + 3 * kC};
    flush_sums<4>(acc, dst, red);
}

// ---- weight gradients: sum of the per-chunk GEMM partials, in double ---------------------

__global__ void __launch_bounds__(256) wgrad_reduce_kernel(WgradReduceArgs a) {
    constexpr int kPer = kC * kC;
    const int e = a.row0 * kC + blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= (a.row0 + a.rows) * kC) return;
    double s = a.first ? 0.0 : a.acc[e];
    for (int k = 0; k < a.slots; ++k) s += (double)__ldg(a.partial + (size_t)k * kWgradRows * kC + e);
    a.acc[e] = s;
    if (!a.last) return;
    float *dst = nullptr;
#pragma unroll
    for (int k = 0; k <= kProjBlocks; ++k)
        if (e / kPer == k) dst = a.dst[k];
    if (dst) dst[e % kPer] = (float)s;
}

// One wave: the resident blocks of the kernel on all SMs, at most `work`.
template <typename K>
int wave(K kernel, size_t smem, int sms, long long work) {
    int per = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, kernel, kThreads, smem) != cudaSuccess || per < 1) per = 1;
    const long long g = (long long)per * sms;
    return (int)(work < g ? work : g);
}

long long tiles_of(int rows, int N) { return (long long)rows * ((N + kTile - 1) / kTile); }

}  // namespace

cudaError_t backward_setup() {
    // All of the unified L1 as shared memory: room for two blocks per SM of the cp.async passes.
    const void *k[3] = {(const void *)proj_bwd_kernel, (const void *)ln_fwd_cm_kernel, (const void *)ln_bwd_cm_kernel};
    const size_t sm[3] = {kProjSmem, kLnFwdCmSmem, kLnBwdCmSmem};
    cudaError_t e = cudaSuccess;
    for (int i = 0; i < 3 && e == cudaSuccess; ++i) {
        e = cudaFuncSetAttribute(k[i], cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm[i]);
        if (e == cudaSuccess) e = cudaFuncSetAttribute(k[i], cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    }
    return e;
}

cudaError_t launch_ln_fwd(const LnFwdArgs &a, int sms, cudaStream_t s) {
    if (a.channel_major)
        ln_fwd_cm_kernel<<<wave(ln_fwd_cm_kernel, kLnFwdCmSmem, sms, ptiles_of(a.rows, a.N)), kThreads, kLnFwdCmSmem, s>>>(a);
    else
        ln_fwd_kernel<<<wave(ln_fwd_kernel, 0, sms, tiles_of(a.rows, a.N)), kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_ln_bwd(const LnBwdArgs &a, int sms, cudaStream_t s) {
    if (a.channel_major)
        ln_bwd_cm_kernel<<<wave(ln_bwd_cm_kernel, kLnBwdCmSmem, sms, ptiles_of(a.rows, a.N)), kThreads, kLnBwdCmSmem, s>>>(a);
    else
        ln_bwd_kernel<<<wave(ln_bwd_kernel, 0, sms, tiles_of(a.rows, a.N)), kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_gate_bwd(const GateBwdArgs &a, int sms, cudaStream_t s) {
    gate_bwd_kernel<<<wave(gate_bwd_kernel, 0, sms, (a.cells + kTile - 1) / kTile), kThreads, 0, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_proj_bwd(const ProjBwdArgs &a, int sms, cudaStream_t s) {
    proj_bwd_kernel<<<wave(proj_bwd_kernel, kProjSmem, sms, ptiles_of(a.rows, a.N)), kThreads, kProjSmem, s>>>(a);
    return cudaGetLastError();
}

cudaError_t launch_wgrad_reduce(const WgradReduceArgs &a, cudaStream_t s) {
    wgrad_reduce_kernel<<<(a.rows * kC + 255) / 256, 256, 0, s>>>(a);
    return cudaGetLastError();
}

}  // namespace trimul

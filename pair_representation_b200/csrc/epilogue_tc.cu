// epilogue_tc.cu - output LayerNorm, gate and output projection, fused, on
// tcgen05 tensor cores.
//
// Per cell (i, j):  out_ij = sigmoid(W_g LN_in(z_ij) + b_g) * (W_o LN_out(x_ij) + b_o)
// (the output half of TriangleMultiplicationOutgoing, "Scaling biomolecular
// modeling with context parallelism in NVIDIA BioNeMo", section
// "Context-parallel implementation of triangle multiplication").
//
// The gate is recomputed from z rather than stored by the prologue: reading z
// again costs 256 B per cell against 512 B per cell to write and re-read g.
//
// Tiles are 128 consecutive cells of one residue row. Per tile:
//   TMA  x tile  [128 ch][128 cells] (channel-major, as the contraction wrote it)
//   TMA  z tile  [128 cells][128 ch] (128-byte swizzle)
//   LN   z in place; LN of x read down its columns and written back in place
//        transposed to the swizzled cell-major layout the MMA reads
//   MMA  G = zh * W_g^T and O = xh * W_o^T (N = 128 each) into a
//        double-buffered 256-column TMEM accumulator
//   out  TMEM -> registers -> sigmoid(G + b_g) * (O + b_o) -> bf16 ->
//        swizzled smem -> TMA store into out[i][j0 .. j0+127][:]
// Loads for tile t+2 are issued as soon as the MMAs of tile t have read their
// buffers, so they are in flight for a whole iteration.
#include "kernels.h"

namespace trimul {
namespace epi {
constexpr int TILE = 128;
constexpr int THREADS = 256;
constexpr int W_HALF = 128 * 128;        // one 64-channel K half of a 128 x 128 weight: 16 KB
constexpr int W_BYTES = 2 * W_HALF;      // 32 KB per weight
constexpr int T_HALF = TILE * 128;       // 16 KB
constexpr int T_BYTES = 2 * T_HALF;      // 32 KB per tile buffer (x or z)
constexpr int ST_BYTES = TILE * 64 * 2;  // 16 KB output staging [128 cells][64 ch]
constexpr int NUM_ST = 2;
constexpr int RED_BYTES = 2 * TILE * 4;  // cross-warp LayerNorm partials
constexpr int BAR_BYTES = 128;
constexpr size_t SMEM = 1024 + 2 * (size_t)W_BYTES + 2 * 2 * (size_t)T_BYTES + NUM_ST * ST_BYTES + RED_BYTES +
                        BAR_BYTES;
static_assert(SMEM <= 232448, "shared memory budget");
}  // namespace epi

// In-place LayerNorm of a swizzled z tile (same layout as the prologue's).
__device__ __forceinline__ void epi_layer_norm_z(uint8_t *zt, const __nv_bfloat16 *gw, const __nv_bfloat16 *gb,
                                                 float eps) {
    const int t = threadIdx.x;
    const int r = t >> 1, h = t & 1;
    uint8_t *rowp = zt + h * epi::T_HALF + r * 128;
    float v[64];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const int kc = (q + 4 * h) & 7;
        uint4 u = *reinterpret_cast<const uint4 *>(rowp + ((kc ^ (r & 7)) << 4));
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            v[kc * 8 + 2 * e] = __uint_as_float(w[e] << 16);
            v[kc * 8 + 2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
        }
    }
    float s = 0.f;
#pragma unroll
    for (int k = 0; k < 64; ++k) s += v[k];
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    const float mean = s * (1.f / 128.f);
    float ss = 0.f;
#pragma unroll
    for (int k = 0; k < 64; ++k) {
        const float d = v[k] - mean;
        ss = fmaf(d, d, ss);
    }
    ss += __shfl_xor_sync(0xffffffffu, ss, 1);
    const float rstd = rsqrtf(ss * (1.f / 128.f) + eps);
#pragma unroll
    for (int kc = 0; kc < 8; ++kc) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int c0 = h * 64 + kc * 8 + 2 * e;
            const float g0 = gw ? __bfloat162float(gw[c0]) : 1.f, g1 = gw ? __bfloat162float(gw[c0 + 1]) : 1.f;
            const float b0 = gb ? __bfloat162float(gb[c0]) : 0.f, b1 = gb ? __bfloat162float(gb[c0 + 1]) : 0.f;
            w[e] = pack_bf16x2(fmaf((v[kc * 8 + 2 * e] - mean) * rstd, g0, b0),
                               fmaf((v[kc * 8 + 2 * e + 1] - mean) * rstd, g1, b1));
        }
        *reinterpret_cast<uint4 *>(rowp + ((kc ^ (r & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

// LayerNorm of a channel-major x tile [128 ch][128 cells], written back in
// place as the swizzled cell-major [2 halves][128 cells][64 ch] MMA operand.
// Thread t owns cell t & 127 and channel half t >> 7 (warp-uniform), so reads
// of one channel across a warp are 64 contiguous bytes; the two halves of a
// cell meet through `red`.
__device__ __forceinline__ void epi_layer_norm_x(uint8_t *xt, float *red, const __nv_bfloat16 *gw,
                                                 const __nv_bfloat16 *gb, float eps) {
    const int t = threadIdx.x;
    const int r = t & 127, h = t >> 7;
    const uint16_t *col = reinterpret_cast<const uint16_t *>(xt) + h * 64 * epi::TILE + r;
    float v[64];
#pragma unroll
    for (int k = 0; k < 64; ++k) v[k] = bf16_bits_to_float(col[k * epi::TILE]);
    float s = 0.f;
#pragma unroll
    for (int k = 0; k < 64; ++k) s += v[k];
    red[h * epi::TILE + r] = s;
    __syncthreads();
    const float mean = (red[r] + red[epi::TILE + r]) * (1.f / 128.f);
    __syncthreads();
    float ss = 0.f;
#pragma unroll
    for (int k = 0; k < 64; ++k) {
        const float d = v[k] - mean;
        ss = fmaf(d, d, ss);
    }
    red[h * epi::TILE + r] = ss;
    __syncthreads();  // also: every thread has read its x column before anyone overwrites the tile
    const float rstd = rsqrtf((red[r] + red[epi::TILE + r]) * (1.f / 128.f) + eps);
    uint8_t *rowp = xt + h * epi::T_HALF + r * 128;
#pragma unroll
    for (int kc = 0; kc < 8; ++kc) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int c0 = h * 64 + kc * 8 + 2 * e;
            const float g0 = gw ? __bfloat162float(gw[c0]) : 1.f, g1 = gw ? __bfloat162float(gw[c0 + 1]) : 1.f;
            const float b0 = gb ? __bfloat162float(gb[c0]) : 0.f, b1 = gb ? __bfloat162float(gb[c0 + 1]) : 0.f;
            w[e] = pack_bf16x2(fmaf((v[kc * 8 + 2 * e] - mean) * rstd, g0, b0),
                               fmaf((v[kc * 8 + 2 * e + 1] - mean) * rstd, g1, b1));
        }
        *reinterpret_cast<uint4 *>(rowp + ((kc ^ (r & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

__global__ void __launch_bounds__(epi::THREADS, 1)
    epilogue_tc_kernel(const __grid_constant__ CUtensorMap tmWg, const __grid_constant__ CUtensorMap tmWo,
                       const __grid_constant__ CUtensorMap tmZ, const __grid_constant__ CUtensorMap tmX,
                       const __grid_constant__ CUtensorMap tmOut, const EpilogueArgs args) {
    using namespace epi;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *wg = smem;
    uint8_t *wo = wg + W_BYTES;
    uint8_t *xs = wo + W_BYTES;        // [2] x tiles
    uint8_t *zs = xs + 2 * T_BYTES;    // [2] z tiles
    uint8_t *st = zs + 2 * T_BYTES;    // [2] output staging
    float *red = reinterpret_cast<float *>(st + NUM_ST * ST_BYTES);
    uint64_t *bars = reinterpret_cast<uint64_t *>(reinterpret_cast<uint8_t *>(red) + RED_BYTES);
    uint64_t *wbar = bars;       // weights landed
    uint64_t *full = bars + 1;   // [2] x and z tile landed
    uint64_t *mma = bars + 3;    // [2] MMAs of the tile in buffer b done
    uint64_t *drain = bars + 5;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 6);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const KernelCtl &ctl = args.ctl;
    const int n_local = (blockIdx.x < (unsigned)args.total_tiles)
                            ? (args.total_tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1
                            : 0;

    if (threadIdx.x == 0) {
        mbar_init(wbar, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&full[b], 1);
            mbar_init(&mma[b], 1);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0) {
        __syncwarp();  // thread 0 ran the set-up above alone; the allocation is warp-wide
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    auto tile_coords = [&](int lt, int &i, int &j0) {
        const int tile = (int)blockIdx.x + lt * (int)gridDim.x;
        i = tile / args.jt_tiles;
        j0 = (tile - i * args.jt_tiles) * TILE;
    };
    int last_load[2] = {-1, -1};
    auto load_tile = [&](int lt) {
        int i, j0;
        tile_coords(lt, i, j0);
        const int b = lt & 1;
        last_load[b] = lt;
        mbar_arrive_expect_tx(&full[b], 2 * T_BYTES);
        tma_load_3d(xs + b * T_BYTES, &tmX, &full[b], j0, i, 0);
        tma_load_3d(zs + b * T_BYTES, &tmZ, &full[b], 0, j0, i);
        tma_load_3d(zs + b * T_BYTES + T_HALF, &tmZ, &full[b], 64, j0, i);
    };
    // G = zh W_g^T into columns [0,128), O = xh W_o^T into [128,256) of accumulator b.
    auto issue_mma = [&](int b) {
        const uint32_t idesc = idesc_bf16(128, 128, 0, 0);
        const uint32_t za = smem_u32(zs + b * T_BYTES), xa = smem_u32(xs + b * T_BYTES);
        const uint32_t gb = smem_u32(wg), ob = smem_u32(wo);
        const uint32_t d = tmem_base + (uint32_t)(b * 256);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (uint32_t)((kk >> 2) * T_HALF + (kk & 3) * 32);
            const uint32_t woff = (uint32_t)((kk >> 2) * W_HALF + (kk & 3) * 32);
            mma_bf16(d, sdesc_sw128(za + off, 16, 1024), sdesc_sw128(gb + woff, 16, 1024), idesc, kk ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (uint32_t)((kk >> 2) * T_HALF + (kk & 3) * 32);
            const uint32_t woff = (uint32_t)((kk >> 2) * W_HALF + (kk & 3) * 32);
            mma_bf16(d + 128, sdesc_sw128(xa + off, 16, 1024), sdesc_sw128(ob + woff, 16, 1024), idesc,
                     kk ? 1u : 0u);
        }
    };
    auto prepare = [&](int b) {
        epi_layer_norm_z(zs + b * T_BYTES, args.ln_in_w, args.ln_in_b, args.eps);
        epi_layer_norm_x(xs + b * T_BYTES, red, args.ln_out_w, args.ln_out_b, args.eps);
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (threadIdx.x == 0) {
            tc_fence_after();
            issue_mma(b);
            mma_commit(&mma[b]);
        }
    };

    if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(wbar, 2 * W_BYTES);
#pragma unroll
        for (int kh = 0; kh < 2; ++kh) {
            tma_load_2d(wg + kh * W_HALF, &tmWg, wbar, kh * 64, 0);
            tma_load_2d(wo + kh * W_HALF, &tmWo, wbar, kh * 64, 0);
        }
        if (n_local > 0) load_tile(0);
        if (n_local > 1) load_tile(1);
    }

    bool ok = __syncthreads_and(wait_bounded(wbar, 0, abort_flag, ctl, SITE_EPI | 1, 0));
    if (ok && n_local > 0) {
        ok = __syncthreads_and(wait_bounded(&full[0], 0, abort_flag, ctl, SITE_EPI | 2, 0));
        if (ok) prepare(0);
    }

    int st_round = 0;
    for (int lt = 0; ok && lt < n_local; ++lt) {
        const int cur = lt & 1, nxt = cur ^ 1;
        int i, j0;
        tile_coords(lt, i, j0);

        // MMAs of tile lt done: accumulator `cur` is ready, buffers `cur` are free.
        ok = __syncthreads_and(wait_bounded(&mma[cur], (uint32_t)(lt >> 1) & 1u, abort_flag, ctl, SITE_EPI | 3, lt));
        if (!ok) break;
        tc_fence_after();
        if (threadIdx.x == 0 && lt + 2 < n_local) load_tile(lt + 2);

        // Normalise tile lt+1 and start its MMAs into the other accumulator.
        if (lt + 1 < n_local) {
            ok = __syncthreads_and(
                wait_bounded(&full[nxt], (uint32_t)((lt + 1) >> 1) & 1u, abort_flag, ctl, SITE_EPI | 4, lt));
            if (!ok) break;
            prepare(nxt);
        }

        // Gate * projection for tile lt, two 64-channel slabs.
        const int q = warp & 3, sub = warp >> 2;
        const int r = q * 32 + lane;
        const uint32_t lane_base = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(cur * 256);
#pragma unroll 1
        for (int hh = 0; hh < 2; ++hh) {
            const int ch0 = hh * 64 + sub * 32;
            uint32_t G[32], O[32];
            __syncwarp();  // tcgen05.ld is warp-wide; thread 0 may have just issued a store alone
            tmem_ld32(lane_base + (uint32_t)ch0, G);
            tmem_ld32(lane_base + 128u + (uint32_t)ch0, O);
            tmem_ld_wait();
            uint32_t p[16];
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                const int c = ch0 + 2 * k;
                const float y0 = sigmoid_fast(__uint_as_float(G[2 * k]) + ld_vec_bf16(args.b_g, c, 0.f)) *
                                 (__uint_as_float(O[2 * k]) + ld_vec_bf16(args.b_o, c, 0.f));
                const float y1 = sigmoid_fast(__uint_as_float(G[2 * k + 1]) + ld_vec_bf16(args.b_g, c + 1, 0.f)) *
                                 (__uint_as_float(O[2 * k + 1]) + ld_vec_bf16(args.b_o, c + 1, 0.f));
                p[k] = pack_bf16x2(y0, y1);
            }
            uint8_t *sb = st + (st_round & 1) * ST_BYTES;
            ++st_round;
            if (threadIdx.x == 0) tma_store_wait_read<1>();
            __syncthreads();
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int kc = sub * 4 + k;  // 16-byte chunk within the 128-byte row
                *reinterpret_cast<uint4 *>(sb + r * 128 + ((kc ^ (r & 7)) << 4)) =
                    make_uint4(p[4 * k], p[4 * k + 1], p[4 * k + 2], p[4 * k + 3]);
            }
            fence_proxy_async_smem();
            __syncthreads();
            if (threadIdx.x == 0) {
                tma_store_3d(&tmOut, sb, hh * 64, j0, i);
                tma_store_commit();
            }
        }
        tc_fence_before();
    }

    if (threadIdx.x == 0) {
        tma_store_wait_all<0>();
        if (!ok) {
            wait_drain(wbar, 0, ctl.timeout_ns);
            for (int b = 0; b < 2; ++b)
                if (last_load[b] >= 0) wait_drain(&full[b], (uint32_t)(last_load[b] >> 1) & 1u, ctl.timeout_ns);
        }
        mma_commit(drain);
        wait_drain(drain, 0, ctl.timeout_ns);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem_base, 512);
}

size_t epilogue_tc_smem() { return epi::SMEM; }

cudaError_t epilogue_tc_setup() {
    return cudaFuncSetAttribute(epilogue_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)epi::SMEM);
}

cudaError_t launch_epilogue_tc(const EpilogueMaps &m, const EpilogueArgs &a, int grid, cudaStream_t s) {
    epilogue_tc_kernel<<<grid, epi::THREADS, epi::SMEM, s>>>(m.wg, m.wo, m.z, m.x, m.out, a);
    return cudaGetLastError();
}

}  // namespace trimul

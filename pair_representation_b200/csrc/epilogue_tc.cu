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
// Tiles are 128 consecutive cells of one residue row. Roles (288 threads):
//   warp 8 (control): TMA loads of the x tile ([128 ch][128 cells], as the
//     contraction wrote it) and the z tile (128-byte swizzle), two tiles ahead;
//     per tile two MMAs, G = zh W_g^T and O = xh W_o^T (M = 128 cells,
//     N = 128, K = 128), into a double-buffered 256-column TMEM accumulator.
//   warps 0-7 (workers):
//     * LayerNorm of z in place (16 cells per warp) and of x, read down its
//       columns and written back in place, transposed, as the swizzled
//       cell-major MMA operand (32 cells x 64 channels per warp, the
//       workers meeting at a 256-thread named barrier);
//     * out = sigmoid(G + b_g) * (O + b_o) for 32 cells x 32 channels per
//       warp in packed fp32x2, bf16, into a 64-byte-swizzled 2 KB buffer of
//       the warp and out by that warp's own TMA store.
// The next tile's LayerNorms run before this tile's gating, so its MMAs
// overlap the gating; the only barrier in the tile loop is the workers' x LayerNorm.
#include "kernels.h"
#include "tile_ops.cuh"

namespace trimul {
namespace epi {
constexpr int TILE = 128;
constexpr int WORKERS = 8;
constexpr int THREADS = 32 * (WORKERS + 1);
constexpr int W_HALF = 128 * 128;        // one 64-channel K half of a 128 x 128 weight: 16 KB
constexpr int W_BYTES = 2 * W_HALF;      // 32 KB per weight
constexpr int T_HALF = TILE * 128;       // 16 KB
constexpr int T_BYTES = 2 * T_HALF;      // 32 KB per tile buffer (x or z)
constexpr int ST_BYTES = 32 * 32 * 2;    // 2 KB per warp buffer: [32 cells][32 ch], 64-byte swizzle
constexpr int ST_PER_WARP = 2;
constexpr int RED_BYTES = 2 * TILE * 4;  // x LayerNorm partials of the two channel halves
constexpr int BAR_BYTES = 128;
constexpr size_t SMEM = 1024 + 2 * (size_t)W_BYTES + 2 * 2 * (size_t)T_BYTES +
                        (size_t)WORKERS * ST_PER_WARP * ST_BYTES + RED_BYTES + BAR_BYTES;
static_assert(SMEM <= 232448, "shared memory budget");
}  // namespace epi

// LayerNorm of a channel-major x tile [128 ch][128 cells], written back in
// place as the swizzled cell-major [2 halves][128 cells][64 ch] MMA operand.
// Worker warp w owns cells 32(w & 3) .. +31 and channel half w >> 2; the two
// halves of a cell meet through `red`. The in-place transposition needs every
// worker to finish reading before any writes, so the steps are separated by
// named barrier 1 over the 256 worker threads.
template <bool kAffine>
__device__ __forceinline__ void epi_layer_norm_x(uint8_t *xt, float *red, const __nv_bfloat16 *gw,
                                                 const __nv_bfloat16 *gb, float eps) {
    const int t = threadIdx.x;
    const int r = t & 127, h = t >> 7;
    const uint16_t *col = reinterpret_cast<const uint16_t *>(xt) + h * 64 * epi::TILE + r;
    float2 v[32];
#pragma unroll
    for (int k = 0; k < 32; ++k)
        v[k] = make_float2(bf16_bits_to_float(col[(2 * k) * epi::TILE]), bf16_bits_to_float(col[(2 * k + 1) * epi::TILE]));
    float2 a0 = make_float2(0.f, 0.f), a1 = a0, a2 = a0, a3 = a0;
#pragma unroll
    for (int k = 0; k < 32; k += 4) {
        a0 = __fadd2_rn(a0, v[k]);
        a1 = __fadd2_rn(a1, v[k + 1]);
        a2 = __fadd2_rn(a2, v[k + 2]);
        a3 = __fadd2_rn(a3, v[k + 3]);
    }
    red[h * epi::TILE + r] = (a0.x + a0.y) + (a1.x + a1.y) + (a2.x + a2.y) + (a3.x + a3.y);
    named_bar_sync(1, 256);
    const float mean = (red[r] + red[epi::TILE + r]) * (1.f / 128.f);
    named_bar_sync(1, 256);
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
    red[h * epi::TILE + r] = (a0.x + a0.y) + (a1.x + a1.y) + (a2.x + a2.y) + (a3.x + a3.y);
    named_bar_sync(1, 256);  // also: every worker has read its x columns before any overwrites them
    const float rstd = rsqrtf((red[r] + red[epi::TILE + r]) * (1.f / 128.f) + eps);
    const float2 sc = make_float2(rstd, rstd), sh = make_float2(-mean * rstd, -mean * rstd);
    uint8_t *rowp = xt + h * epi::T_HALF + r * 128;
#pragma unroll
    for (int kc = 0; kc < 8; ++kc) {
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            float2 y = __ffma2_rn(v[kc * 4 + e], sc, sh);
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

// kVec: some LayerNorm affine or output bias is present (general path).
template <bool kVec>
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
    uint8_t *st = zs + 2 * T_BYTES;    // [8 warps][2] output staging
    float *red = reinterpret_cast<float *>(st + WORKERS * ST_PER_WARP * ST_BYTES);
    uint64_t *bars = reinterpret_cast<uint64_t *>(reinterpret_cast<uint8_t *>(red) + RED_BYTES);
    uint64_t *wbar = bars;          // weights landed
    uint64_t *full = bars + 1;      // [2] x and z tile landed
    uint64_t *mma = bars + 3;       // [2] MMAs of the tile in buffer b done
    uint64_t *ln_done = bars + 5;   // workers: tile normalised (8 arrivals)
    uint64_t *acc_free = bars + 6;  // [2] workers: accumulator b read (8 arrivals)
    uint64_t *drain = bars + 8;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 9);
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
            mbar_init(&acc_free[b], WORKERS);
        }
        mbar_init(ln_done, WORKERS);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == WORKERS) {
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

    if (warp == WORKERS) {
        // ------------------------------ control warp ------------------------------
        if (lane == 0) {
            int last_load0 = -1, last_load1 = -1;
            auto load_tile = [&](int lt) {
                int i, j0;
                tile_coords(lt, i, j0);
                const int b = lt & 1;
                if (b) last_load1 = lt; else last_load0 = lt;
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
                    mma_bf16(d, sdesc_sw128(za + off, 16, 1024), sdesc_sw128(gb + woff, 16, 1024), idesc,
                             kk ? 1u : 0u);
                }
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (uint32_t)((kk >> 2) * T_HALF + (kk & 3) * 32);
                    const uint32_t woff = (uint32_t)((kk >> 2) * W_HALF + (kk & 3) * 32);
                    mma_bf16(d + 128, sdesc_sw128(xa + off, 16, 1024), sdesc_sw128(ob + woff, 16, 1024), idesc,
                             kk ? 1u : 0u);
                }
            };
            mbar_arrive_expect_tx(wbar, 2 * W_BYTES);
#pragma unroll
            for (int kh = 0; kh < 2; ++kh) {
                tma_load_2d(wg + kh * W_HALF, &tmWg, wbar, kh * 64, 0);
                tma_load_2d(wo + kh * W_HALF, &tmWo, wbar, kh * 64, 0);
            }
            if (n_local > 0) load_tile(0);
            if (n_local > 1) load_tile(1);
            bool ok = wait_bounded(wbar, 0, abort_flag, ctl, SITE_EPI | 1, 0);
            for (int lt = 0; ok && lt < n_local; ++lt) {
                const int b = lt & 1;
                if (!wait_bounded(ln_done, (uint32_t)lt & 1u, abort_flag, ctl, SITE_EPI | 2, lt) ||
                    (lt >= 2 && !wait_bounded(&acc_free[b], (uint32_t)((lt - 2) >> 1) & 1u, abort_flag, ctl,
                                              SITE_EPI | 3, lt))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                issue_mma(b);
                mma_commit(&mma[b]);
                if (lt + 2 < n_local) {
                    // Buffers b are free once the MMAs of tile lt have read them.
                    if (!wait_bounded(&mma[b], (uint32_t)(lt >> 1) & 1u, abort_flag, ctl, SITE_EPI | 4, lt)) {
                        ok = false;
                        break;
                    }
                    load_tile(lt + 2);
                }
            }
            if (!ok) {
                *abort_flag = 1;
                wait_drain(wbar, 0, ctl.timeout_ns);
                if (last_load0 >= 0) wait_drain(&full[0], (uint32_t)(last_load0 >> 1) & 1u, ctl.timeout_ns);
                if (last_load1 >= 0) wait_drain(&full[1], (uint32_t)(last_load1 >> 1) & 1u, ctl.timeout_ns);
            }
            mma_commit(drain);
            wait_drain(drain, 0, ctl.timeout_ns);
        }
    } else {
        // ------------------------------ worker warps ------------------------------
        const int q = warp & 3, sub = warp >> 2;
        uint8_t *stw = st + warp * ST_PER_WARP * ST_BYTES;
        int st_round = 0;
        auto normalise = [&](int b) {
            ln_tile_sw128<kVec>(zs + b * T_BYTES, T_HALF, args.ln_in_w, args.ln_in_b, args.eps);
            epi_layer_norm_x<kVec>(xs + b * T_BYTES, red, args.ln_out_w, args.ln_out_b, args.eps);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(ln_done);
        };

        // Every worker takes the LayerNorm barriers: before each normalisation the
        // workers agree (bar.red.and) on whether to go on, so none can be left
        // waiting at a barrier after another has stopped.
        bool ok = warp_wait(&full[0], 0, abort_flag, ctl, SITE_EPI | 5, 0);
        ok = bar_red_and(1, 32 * WORKERS, ok);
        if (ok) normalise(0);
        for (int lt = 0; ok && lt < n_local; ++lt) {
            const int cur = lt & 1;
            int i, j0;
            tile_coords(lt, i, j0);
            // Normalise tile lt+1 first, so its MMAs run while this tile is gated.
            if (lt + 1 < n_local) {
                bool got = warp_wait(&full[cur ^ 1], (uint32_t)((lt + 1) >> 1) & 1u, abort_flag, ctl, SITE_EPI | 6, lt);
                if (!(ok = bar_red_and(1, 32 * WORKERS, got))) break;
                normalise(cur ^ 1);
            }
            if (!warp_wait(&mma[cur], (uint32_t)(lt >> 1) & 1u, abort_flag, ctl, SITE_EPI | 7, lt)) {
                // Leave the gating out but stay in step with the other workers' barriers.
                ok = false;
                if (lane == 0) *abort_flag = 1;
                tc_fence_before();
                if (lane == 0) mbar_arrive(&acc_free[cur]);
                // Join the agreement the others take at the start of iteration lt + 1
                // (there is one only if that iteration normalises tile lt + 2).
                if (lt + 2 < n_local) bar_red_and(1, 32 * WORKERS, false);
                break;
            }
            tc_fence_after();
            const bool live = j0 + 32 * q < args.N;
            const uint32_t lane_base = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(cur * 256);
#pragma unroll 1
            for (int hh = 0; live && hh < 2; ++hh) {
                const int ch0 = hh * 64 + sub * 32;
                uint32_t G[32], O[32];
                tmem_ld32(lane_base + (uint32_t)ch0, G);
                tmem_ld32(lane_base + 128u + (uint32_t)ch0, O);
                tmem_ld_wait();
                // out = sigmoid(G + b_g) * (O + b_o) = (tanh((G + b_g) / 2) / 2 + 1/2) * (O + b_o)
                uint32_t p[16];
                const float2 half = make_float2(0.5f, 0.5f);
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    float2 g = make_float2(__uint_as_float(G[2 * k]), __uint_as_float(G[2 * k + 1]));
                    float2 o = make_float2(__uint_as_float(O[2 * k]), __uint_as_float(O[2 * k + 1]));
                    if (kVec) {
                        if (args.b_g) g = __fadd2_rn(g, ld_pair_bf16(args.b_g, ch0 + 2 * k));
                        if (args.b_o) o = __fadd2_rn(o, ld_pair_bf16(args.b_o, ch0 + 2 * k));
                    }
                    const float2 hg = __fmul2_rn(g, half);
                    const float2 th = make_float2(tanh_approx(hg.x), tanh_approx(hg.y));
                    const float2 y = __fmul2_rn(__ffma2_rn(th, half, half), o);
                    p[k] = pack_bf16x2(y.x, y.y);
                }
                uint8_t *sb = stw + (st_round & 1) * ST_BYTES;
                ++st_round;
                if (lane == 0) tma_store_wait_read<1>();
                __syncwarp();
                // [32 cells][32 ch]: 64-byte rows, 16-byte chunk c at c ^ ((cell >> 1) & 3).
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    *reinterpret_cast<uint4 *>(sb + lane * 64 + ((c ^ ((lane >> 1) & 3)) << 4)) =
                        make_uint4(p[4 * c], p[4 * c + 1], p[4 * c + 2], p[4 * c + 3]);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_3d(&tmOut, sb, ch0, j0 + 32 * q, i);
                    tma_store_commit();
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_free[cur]);
        }
        if (!ok && lane == 0) *abort_flag = 1;
        if (lane == 0) tma_store_wait_all<0>();
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == WORKERS) tmem_dealloc(tmem_base, 512);
}

size_t epilogue_tc_smem() { return epi::SMEM; }

cudaError_t epilogue_tc_setup() {
    cudaError_t e = cudaFuncSetAttribute(epilogue_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)epi::SMEM);
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(epilogue_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)epi::SMEM);
}

cudaError_t launch_epilogue_tc(const EpilogueMaps &m, const EpilogueArgs &a, int grid, cudaStream_t s) {
    const bool vec = a.ln_in_w || a.ln_in_b || a.ln_out_w || a.ln_out_b || a.b_g || a.b_o;
    if (vec)
        epilogue_tc_kernel<true><<<grid, epi::THREADS, epi::SMEM, s>>>(m.wg, m.wo, m.z, m.x, m.out, a);
    else
        epilogue_tc_kernel<false><<<grid, epi::THREADS, epi::SMEM, s>>>(m.wg, m.wo, m.z, m.x, m.out, a);
    return cudaGetLastError();
}

}  // namespace trimul

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
// Both LayerNorms are folded into their projections. With per-cell mean mu and
// rstd r, and W' = W diag(gamma):
//   W LN(v) + bias = r (W' v - mu s) + t,   s[n] = sum_k W'[n][k],
//                                            t[n] = sum_k W[n][k] beta[k] + bias[n].
// The MMAs therefore run on the raw tiles exactly as TMA lands them: z as the
// K-major operand and x, which the contraction wrote channel-major, as the
// MN-major operand. No warp rewrites a tile and the tensor work never waits
// for a LayerNorm. s is summed from the same bf16 W' the MMA reads, so the
// mean term cancels as it would in exact arithmetic.
//
// Tiles are 128 consecutive cells of one residue row. Roles (544 threads):
//   all, once: W' = W gamma in shared memory, s and t per output channel.
//   warp 16 (control): TMA loads of the x and z tiles two tiles ahead; per tile
//     G = z W_g'^T and O = x W_o'^T (M = 128 cells, N = 128, K = 128) into a
//     double-buffered 256-column TMEM accumulator.
//   warps 8-15 (statistics): mean and rstd of z and of x for each cell of a
//     landed tile, into a two-slot table: z by two threads per cell (one per
//     channel half), x by four threads per pair of adjacent cells (one per
//     channel quarter, 4-byte loads).
//   warps 0-7 (gaters): warp w reads TMEM lanes 32(w % 4).. (its 32 cells) and
//     channels 64(w / 4)..+63 of G and O, forms
//     sigmoid(r_z (G - mu_z s_g) + t_g) * (r_x (O - mu_x s_o) + t_o) in packed
//     fp32x2, and writes the bf16 result into a 64-byte-swizzled 2 KB buffer of
//     the warp, stored by that warp's own TMA store.
#include "kernels.h"
#include "tile_ops.cuh"

namespace trimul {
namespace epi {
constexpr int TILE = 128;
constexpr int GATERS = 8;
constexpr int STATS = 8;
constexpr int CTRL_WARP = GATERS + STATS;
constexpr int THREADS = 32 * (CTRL_WARP + 1);
constexpr int W_HALF = 128 * 128;          // one 64-channel K half of a 128 x 128 weight: 16 KB
constexpr int W_BYTES = 2 * W_HALF;        // 32 KB per weight
constexpr int T_HALF = TILE * 128;         // 16 KB
constexpr int T_BYTES = 2 * T_HALF;        // 32 KB per tile buffer (x or z)
constexpr int ST_BYTES = 32 * 32 * 2;      // 2 KB per warp buffer: [32 cells][32 ch], 64-byte swizzle
constexpr int CST_BYTES = 4 * 128 * 4;     // per channel pair: (s_g, s_g, s_o, s_o), (t_g, t_g, t_o, t_o) / 2
constexpr int STAT_BYTES = 2 * TILE * 16;  // two slots of (-mu_z, r_z / 2) and (-mu_x, r_x / 2) per cell
constexpr int BAR_BYTES = 128;
constexpr size_t SMEM = 1024 + 2 * (size_t)W_BYTES + 2 * 2 * (size_t)T_BYTES + (size_t)GATERS * ST_BYTES +
                        CST_BYTES + STAT_BYTES + BAR_BYTES;
static_assert(SMEM <= 232448, "shared memory budget");
}  // namespace epi

// Row n of a 128 x 128 bf16 weight held as two 64-column halves of 128-byte
// rows with the 128-byte swizzle: 16-byte chunk kc of half h sits at chunk
// kc ^ (n & 7).
__device__ __forceinline__ uint4 *w_chunk(uint8_t *w, int n, int h, int kc) {
    return reinterpret_cast<uint4 *>(w + h * epi::W_HALF + n * 128 + ((kc ^ (n & 7)) << 4));
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
    uint8_t *xs = wo + W_BYTES;        // [2] x tiles: [2 cell blocks][128 ch][64 cells]
    uint8_t *zs = xs + 2 * T_BYTES;    // [2] z tiles: [2 ch halves][128 cells][64 ch]
    uint8_t *st = zs + 2 * T_BYTES;    // [8 warps] output staging
    // cs4[p] = (s_g[2p], s_g[2p+1], s_o[2p], s_o[2p+1]); ct4[p] = (t_g[2p], t_g[2p+1], t_o[2p], t_o[2p+1]) / 2
    float4 *cs4 = reinterpret_cast<float4 *>(st + GATERS * ST_BYTES);
    float4 *ct4 = cs4 + 64;
    float2 *statz = reinterpret_cast<float2 *>(cs4 + 128);  // [2][128] (-mu_z, r_z / 2)
    float2 *statx = statz + 2 * TILE;                        // [2][128] (-mu_x, r_x / 2)
    uint64_t *bars = reinterpret_cast<uint64_t *>(statx + 2 * TILE);
    uint64_t *wbar = bars;             // weights landed
    uint64_t *full = bars + 1;         // [2] x and z tile landed
    uint64_t *mma = bars + 3;          // [2] MMAs into accumulator b done
    uint64_t *xzdone = bars + 5;       // [2] MMAs have read tile buffer b
    uint64_t *stat_done = bars + 7;    // [2] statistics of the tile in buffer b written (8 arrivals)
    uint64_t *stat_free = bars + 9;    // [2] gaters have read statistics slot b (8 arrivals)
    uint64_t *acc_free = bars + 11;    // [2] gaters have read accumulator b (8 arrivals)
    uint64_t *drain = bars + 13;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 14);
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
            mbar_init(&xzdone[b], 1);
            mbar_init(&stat_done[b], STATS);
            mbar_init(&stat_free[b], GATERS);
            mbar_init(&acc_free[b], GATERS);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == CTRL_WARP) {
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

    int last_load0 = -1, last_load1 = -1;  // control lane: latest tile loaded into each buffer
    auto load_tile = [&](int lt) {
        int i, j0;
        tile_coords(lt, i, j0);
        const int b = lt & 1;
        if (b) last_load1 = lt; else last_load0 = lt;
        mbar_arrive_expect_tx(&full[b], 2 * T_BYTES);
        tma_load_3d(xs + b * T_BYTES, &tmX, &full[b], j0, i, 0);
        tma_load_3d(xs + b * T_BYTES + T_HALF, &tmX, &full[b], j0 + 64, i, 0);
        tma_load_3d(zs + b * T_BYTES, &tmZ, &full[b], 0, j0, i);
        tma_load_3d(zs + b * T_BYTES + T_HALF, &tmZ, &full[b], 64, j0, i);
    };
    if (warp == CTRL_WARP && lane == 0) {
        mbar_arrive_expect_tx(wbar, 2 * W_BYTES);
#pragma unroll
        for (int kh = 0; kh < 2; ++kh) {
            tma_load_2d(wg + kh * W_HALF, &tmWg, wbar, kh * 64, 0);
            tma_load_2d(wo + kh * W_HALF, &tmWo, wbar, kh * 64, 0);
        }
        if (n_local > 0) load_tile(0);
        if (n_local > 1) load_tile(1);
    }

    // ---- weights: W' = W gamma in place, s = row sums of W', t = W beta + bias --------------
    // Thread t < 256 owns row t % 128 of weight t / 128 (W_g, then W_o).
    bool ok = warp_wait(wbar, 0, abort_flag, ctl, SITE_EPI | 1, 0);
    if (ok && threadIdx.x < 256) {
        const int w = threadIdx.x >> 7, n = threadIdx.x & 127;
        uint8_t *W = w ? wo : wg;
        const __nv_bfloat16 *gamma = w ? args.ln_out_w : args.ln_in_w;
        const __nv_bfloat16 *beta = w ? args.ln_out_b : args.ln_in_b;
        const __nv_bfloat16 *bias = w ? args.b_o : args.b_g;
        float t = 0.f;
        float2 s2 = make_float2(0.f, 0.f);
#pragma unroll 1
        for (int h = 0; h < 2; ++h)
#pragma unroll 1
            for (int kc = 0; kc < 8; ++kc) {
                uint4 *cp = w_chunk(W, n, h, kc);
                const uint4 u = *cp;
                uint32_t wd[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int k = h * 64 + kc * 8 + 2 * e;
                    float2 v = unpack_bf16x2(wd[e]);
                    if (kVec) {
                        if (beta) t = fmaf(v.x, __bfloat162float(beta[k]), fmaf(v.y, __bfloat162float(beta[k + 1]), t));
                        if (gamma) {
                            v = __fmul2_rn(v, make_float2(__bfloat162float(gamma[k]), __bfloat162float(gamma[k + 1])));
                            wd[e] = pack_bf16x2(v.x, v.y);
                            v = unpack_bf16x2(wd[e]);  // the rounded W' the MMA reads
                        }
                    }
                    s2 = __fadd2_rn(s2, v);
                }
                if (kVec && gamma) *cp = make_uint4(wd[0], wd[1], wd[2], wd[3]);
            }
        if (kVec && bias) t += __bfloat162float(bias[n]);
        reinterpret_cast<float *>(cs4)[(n >> 1) * 4 + 2 * w + (n & 1)] = s2.x + s2.y;
        reinterpret_cast<float *>(ct4)[(n >> 1) * 4 + 2 * w + (n & 1)] = 0.5f * t;
    }
    fence_proxy_async_smem();  // W' written by threads is read by the tensor core
    __syncthreads();
    ok = ok && !*abort_flag;

    if (warp == CTRL_WARP) {
        // ------------------------------ control warp ------------------------------
        if (lane == 0) {
            // Accumulator b: G in columns [0, 128), O in [128, 256).
            auto issue_mma = [&](int b) {
                const uint32_t zb = smem_u32(zs + b * T_BYTES), xb = smem_u32(xs + b * T_BYTES);
                const uint32_t gb = smem_u32(wg), ob = smem_u32(wo);
                const uint32_t d = tmem_base + (uint32_t)(b * 256);
                const uint32_t idesc_g = idesc_bf16(128, 128, 0, 0), idesc_o = idesc_bf16(128, 128, 1, 0);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t off = (uint32_t)((kk >> 2) * T_HALF + (kk & 3) * 32);
                    const uint32_t woff = (uint32_t)((kk >> 2) * W_HALF + (kk & 3) * 32);
                    mma_bf16(d, sdesc_sw128(zb + off, 16, 1024), sdesc_sw128(gb + woff, 16, 1024), idesc_g,
                             kk ? 1u : 0u);
                }
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    // x is MN-major: 16 channel rows of 128 B per K step, cell blocks T_HALF apart.
                    const uint32_t woff = (uint32_t)((kk >> 2) * W_HALF + (kk & 3) * 32);
                    mma_bf16(d + 128, sdesc_sw128(xb + (uint32_t)(kk * 2048), T_HALF, 1024),
                             sdesc_sw128(ob + woff, 16, 1024), idesc_o, kk ? 1u : 0u);
                }
            };
            for (int lt = 0; ok && lt < n_local; ++lt) {
                const int b = lt & 1;
                const uint32_t par = (uint32_t)(lt >> 1) & 1u;
                if (!wait_bounded(&full[b], par, abort_flag, ctl, SITE_EPI | 2, lt) ||
                    (lt >= 2 && !wait_bounded(&acc_free[b], par ^ 1u, abort_flag, ctl, SITE_EPI | 3, lt))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                issue_mma(b);
                mma_commit(&mma[b]);
                mma_commit(&xzdone[b]);
                if (lt + 2 < n_local) {
                    // Buffers b are free once the MMAs and the statistics of tile lt have read them.
                    if (!wait_bounded(&xzdone[b], par, abort_flag, ctl, SITE_EPI | 4, lt) ||
                        !wait_bounded(&stat_done[b], par, abort_flag, ctl, SITE_EPI | 5, lt)) {
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
    } else if (warp >= GATERS) {
        // ------------------------------ statistics ------------------------------
        // z: thread (cell, h) reads channel half h of its cell's row. x: thread (pair, quarter)
        // reads channels 32 quarter .. + 31 of the two adjacent cells 2 pair, 2 pair + 1 with
        // 4-byte loads; the four quarters of a pair are lanes 4k .. 4k + 3, visiting their
        // channels in an order staggered by 2 per quarter so that one warp load touches 8
        // distinct 16-byte chunks (no bank conflicts).
        const int t = (warp - GATERS) * 32 + lane;
        const int zcell = t >> 1, zh = t & 1;
        const int pr = t >> 2, quarter = t & 3;
        const int xcell = 2 * pr, mb = xcell >> 6, m = xcell & 63;
        for (int lt = 0; ok && lt < n_local; ++lt) {
            const int b = lt & 1;
            const uint32_t par = (uint32_t)(lt >> 1) & 1u;
            if (!(ok = warp_wait(&full[b], par, abort_flag, ctl, SITE_EPI | 6, lt))) break;
            if (lt >= 2 && !(ok = warp_wait(&stat_free[b], par ^ 1u, abort_flag, ctl, SITE_EPI | 7, lt))) break;
            const uint8_t *zr = zs + b * T_BYTES + zcell * 128;
            RowStats sz;
            sz.s = sz.ss = make_float2(0.f, 0.f);
            sz.k = bf16_bits_to_float(*reinterpret_cast<const uint16_t *>(zr + ((zcell & 7) << 4)));
#pragma unroll
            for (int kc = 0; kc < 8; ++kc) {
                const uint4 u = *reinterpret_cast<const uint4 *>(zr + zh * T_HALF + ((kc ^ (zcell & 7)) << 4));
                stats_add(sz, u.x);
                stats_add(sz, u.y);
                stats_add(sz, u.z);
                stats_add(sz, u.w);
            }
            const uint8_t *xc = xs + b * T_BYTES + mb * T_HALF + (m & 7) * 2;
            const float2 kx = unpack_bf16x2(*reinterpret_cast<const uint32_t *>(xc + ((m >> 3) << 4)));
            float2 xs1 = make_float2(0.f, 0.f), xs2 = xs1;  // per cell: sum of d, sum of d^2
#pragma unroll 8
            for (int it = 0; it < 32; ++it) {
                const int c = 32 * quarter + ((it + 2 * quarter) & 31);
                const uint32_t w2 = *reinterpret_cast<const uint32_t *>(xc + c * 128 + (((m >> 3) ^ (c & 7)) << 4));
                const float2 d = __fadd2_rn(unpack_bf16x2(w2), make_float2(-kx.x, -kx.y));
                xs1 = __fadd2_rn(xs1, d);
                xs2 = __ffma2_rn(d, d, xs2);
            }
#pragma unroll
            for (int o = 1; o <= 2; o <<= 1) {
                xs1.x += __shfl_xor_sync(0xffffffffu, xs1.x, o);
                xs1.y += __shfl_xor_sync(0xffffffffu, xs1.y, o);
                xs2.x += __shfl_xor_sync(0xffffffffu, xs2.x, o);
                xs2.y += __shfl_xor_sync(0xffffffffu, xs2.y, o);
            }
            const float2 fz = stats_finish(sz, args.eps);
            if (zh == 0) statz[b * TILE + zcell] = make_float2(-fz.x, 0.5f * fz.y);
            if (quarter == 0) {
                const float2 mx = __fmul2_rn(xs1, make_float2(1.f / 128.f, 1.f / 128.f));
                const float2 vx = __ffma2_rn(xs2, make_float2(1.f / 128.f, 1.f / 128.f), __fmul2_rn(mx, make_float2(-mx.x, -mx.y)));
                statx[b * TILE + xcell] = make_float2(-(kx.x + mx.x), 0.5f * rsqrtf(fmaxf(vx.x, 0.f) + args.eps));
                statx[b * TILE + xcell + 1] = make_float2(-(kx.y + mx.y), 0.5f * rsqrtf(fmaxf(vx.y, 0.f) + args.eps));
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&stat_done[b]);
        }
        if (!ok && lane == 0) *abort_flag = 1;
    } else {
        // ------------------------------ gaters ------------------------------
        const int q = warp & 3, sub = warp >> 2;
        uint8_t *sb = st + warp * ST_BYTES;
        for (int lt = 0; ok && lt < n_local; ++lt) {
            const int b = lt & 1;
            const uint32_t par = (uint32_t)(lt >> 1) & 1u;
            int i, j0;
            tile_coords(lt, i, j0);
            if (!(ok = warp_wait(&stat_done[b], par, abort_flag, ctl, SITE_EPI | 8, lt))) break;
            // (-mu_z, r_z / 2) and (-mu_x, r_x / 2) of this thread's cell
            const float2 cz = statz[b * TILE + 32 * q + lane], cx = statx[b * TILE + 32 * q + lane];
            __syncwarp();
            if (lane == 0) mbar_arrive(&stat_free[b]);
            if (!(ok = warp_wait(&mma[b], par, abort_flag, ctl, SITE_EPI | 9, lt))) break;
            tc_fence_after();
            const bool live = j0 + 32 * q < args.N;
            const uint32_t lane_base = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * 256);
            const float2 nmz = make_float2(cz.x, cz.x), hrz = make_float2(cz.y, cz.y);
            const float2 nmx = make_float2(cx.x, cx.x), hrx = make_float2(cx.y, cx.y);
#pragma unroll 1
            for (int hh = 0; live && hh < 2; ++hh) {
                const int ch0 = sub * 64 + hh * 32;
                // out = sigmoid(2 hg) * 2 ho = (tanh(hg) + 1) * ho with
                // hg = r_z / 2 (G - mu_z s_g) + t_g / 2 and ho = r_x / 2 (O - mu_x s_o) + t_o / 2.
                uint32_t p[16];
#pragma unroll
                for (int hc = 0; hc < 2; ++hc) {
                    uint32_t G[16], O[16];
                    tmem_ld16(lane_base + (uint32_t)(ch0 + 16 * hc), G);
                    tmem_ld16(lane_base + 128u + (uint32_t)(ch0 + 16 * hc), O);
                    tmem_ld_wait();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const int k = 8 * hc + kk, n = ch0 + 2 * k;
                        const float4 s4 = cs4[n >> 1];
                        const float2 sg = make_float2(s4.x, s4.y), so = make_float2(s4.z, s4.w);
                        const float2 g = make_float2(__uint_as_float(G[2 * kk]), __uint_as_float(G[2 * kk + 1]));
                        const float2 o = make_float2(__uint_as_float(O[2 * kk]), __uint_as_float(O[2 * kk + 1]));
                        float2 hg, ho;
                        if (kVec) {
                            const float4 t4 = ct4[n >> 1];
                            hg = __ffma2_rn(__ffma2_rn(nmz, sg, g), hrz, make_float2(t4.x, t4.y));
                            ho = __ffma2_rn(__ffma2_rn(nmx, so, o), hrx, make_float2(t4.z, t4.w));
                        } else {
                            hg = __fmul2_rn(__ffma2_rn(nmz, sg, g), hrz);
                            ho = __fmul2_rn(__ffma2_rn(nmx, so, o), hrx);
                        }
                        const float2 th = make_float2(tanh_approx(hg.x), tanh_approx(hg.y));
                        const float2 y = __ffma2_rn(th, ho, ho);
                        p[k] = pack_bf16x2(y.x, y.y);
                    }
                }
                if (lane == 0) tma_store_wait_read<0>();  // the previous store has read the buffer
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
            if (lane == 0) mbar_arrive(&acc_free[b]);
        }
        if (!ok && lane == 0) *abort_flag = 1;
        if (lane == 0) tma_store_wait_all<0>();
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == CTRL_WARP) tmem_dealloc(tmem_base, 512);
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

// prologue_tc.cu - input LayerNorm, the four gated projections and the mask,
// fused, on tcgen05 tensor cores.
//
// Per cell (r, s):  zh = LayerNorm_in(z_rs);
//   a_rs = mask_rs * sigmoid(W_ag zh + b_ag) * (W_a zh + b_a)
//   b_rs = mask_rs * sigmoid(W_bg zh + b_bg) * (W_b zh + b_b)
// (the projection half of the layer the pages call
// TriangleMultiplicationOutgoing, "Scaling biomolecular modeling with context
// parallelism in NVIDIA BioNeMo", section "Context-parallel implementation of
// triangle multiplication"), written straight into the channel-major
// [128][N][ld] bf16 layout the contraction's TMA reads.
//
// The LayerNorm is folded into the projections. With the cell's mean mu and
// rstd r, and W' = W diag(gamma):
//   W LN(z) + bias = r (W' z - mu s) + t,   s[c] = sum_k W'[c][k],
//                                            t[c] = sum_k W[c][k] beta[k] + bias[c],
// so the MMAs read the raw z tile exactly as TMA lands it and no warp ever
// writes to it. s is summed from the bf16 W' the MMA reads, so the mean term
// cancels as it would in exact arithmetic.
//
// The projection is computed transposed, D[c][cell] = W'[c][:] . z[cell][:]:
// the four weights live in tensor memory as the MMA's A operand (lane = output
// channel c, 64 columns of packed bf16 pairs each), z is the K-major B operand
// in shared memory, and the accumulator has one channel per TMEM lane and one
// cell per column - already the channel-major order of a and b. The gate
// weights are halved when they are put in tensor memory (exact in bf16), so the
// gate accumulator holds g / 2 and sigmoid(g) = (1 + tanh(g / 2)) / 2.
//
// Tiles are 64 consecutive cells of one residue row, z[i][j0 .. j0+63][:], one
// contiguous 16 KB block. Tensor memory: weights in columns 0..255, the
// accumulators of one tile in 256..511 (a values, a gates, b values, b gates,
// 64 columns each). Shared memory holds no weights, which leaves room for a
// ring of 8 z tiles: 128 KB of loads in flight per SM. Roles (448 threads),
// coupled only through mbarriers:
//   warp 12 (producer): TMA loads of z and of the tile's mask row segment, up
//     to 8 tiles ahead.
//   warp 13 (MMA): per tile the a-half (D_av, D_ag) and the b-half (D_bv, D_bg),
//     M = 128 channels, N = 64 cells, K = 128, each half issued as soon as its
//     accumulator columns are free.
//   warps 8-11 (statistics): mean and rstd of each cell of a landed tile (two
//     threads per cell, fp32 around the cell's first value) into a per-slot
//     table.
//   warps 0-7 (gaters): warp w reads TMEM lanes 32 (w % 4) .. (32 channels) and
//     columns of cells 32 (w / 4) .. + 31, forms
//       mask * (1 + tanh(r D_g - mu r s_g + t_g)) / 2 * (r D_v - mu r s_v + t_v)
//     in packed fp32x2 and writes each channel's 32 results (64 bytes) into a
//     [32 ch][64 cells] staging buffer shared by the two warps of its lane
//     quadrant, which one of them stores with TMA: 128-byte rows of a or b.
#include "kernels.h"
#include "tile_ops.cuh"

namespace trimul {
namespace pro {
constexpr int TILE = 64;                        // cells per tile
constexpr int SLOTS = 8;                        // z ring depth
constexpr int GATERS = 8;
constexpr int STATW = 4;
constexpr int PROD_WARP = GATERS + STATW;       // 12
constexpr int MMA_WARP = PROD_WARP + 1;         // 13
constexpr int THREADS = 32 * (MMA_WARP + 1);    // 448
constexpr int Z_HALF = TILE * 128;              // 8 KB: 64 cells x 64 channels
constexpr int Z_BYTES = 2 * Z_HALF;             // 16 KB
constexpr int MASK_BYTES = TILE * 2;            // one bf16 mask row segment per tile
constexpr int STG_BYTES = 32 * TILE * 2;        // 4 KB: [32 ch][64 cells] bf16, 128-byte rows, 128-byte swizzle
constexpr int NUM_STG = 8;                      // [lane quadrant][a | b]
constexpr int STAT_BYTES = TILE * 8;            // per slot: (r, r, -mu r, -mu r) per cell pair
constexpr int CST_FLOATS = 8 * 128;             // (s, t) of a values, a gates, b values, b gates per channel
constexpr int BAR_BYTES = 256;
constexpr uint32_t COL_W = 0;                   // W_a', W_ag'/2, W_b', W_bg'/2: 64 columns each
constexpr uint32_t COL_D = 256;                 // D_av, D_ag, D_bv, D_bg: 64 columns each
constexpr size_t SMEM = 1024 + (size_t)SLOTS * Z_BYTES + (size_t)NUM_STG * STG_BYTES + SLOTS * MASK_BYTES +
                        SLOTS * STAT_BYTES + CST_FLOATS * 4 + BAR_BYTES;
static_assert(SMEM <= 232448, "shared memory budget");
}  // namespace pro

__global__ void __launch_bounds__(pro::THREADS, 1)
    prologue_tc_kernel(const __grid_constant__ CUtensorMap tmZ, const __grid_constant__ CUtensorMap tmMask,
                       const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                       const PrologueArgs args) {
    using namespace pro;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *zsm = smem;                                     // [SLOTS] z tiles: [2 ch halves][64 cells][64 ch]
    uint8_t *stg = zsm + SLOTS * Z_BYTES;                    // [4 quadrants][a | b] staging
    uint8_t *msm = stg + NUM_STG * STG_BYTES;                // [SLOTS] mask rows (bf16)
    float4 *stats = reinterpret_cast<float4 *>(msm + SLOTS * MASK_BYTES);  // [SLOTS][32 cell pairs]
    float *cst = reinterpret_cast<float *>(stats + SLOTS * (TILE / 2));    // [8][128]
    uint64_t *bars = reinterpret_cast<uint64_t *>(cst + CST_FLOATS);
    uint64_t *zfull = bars;                   // [SLOTS] z tile (and mask row) landed
    uint64_t *stat_done = bars + SLOTS;       // [SLOTS] statistics written (4 arrivals)
    uint64_t *tile_done = bars + 2 * SLOTS;   // [SLOTS] gaters done with the slot's z, mask and statistics (8)
    uint64_t *mma_h = bars + 3 * SLOTS;       // [2] a-half / b-half MMAs done
    uint64_t *free_h = mma_h + 2;             // [2] gaters have read the a-half / b-half accumulators (8)
    uint64_t *wready = free_h + 2;            // weights are in tensor memory (8)
    uint64_t *drain = wready + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const KernelCtl &ctl = args.ctl;
    const int n_local = (blockIdx.x < (unsigned)args.total_tiles)
                            ? (args.total_tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1
                            : 0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < SLOTS; ++s) {
            mbar_init(&zfull[s], 1);
            mbar_init(&stat_done[s], STATW);
            mbar_init(&tile_done[s], GATERS);
        }
        for (int h = 0; h < 2; ++h) {
            mbar_init(&mma_h[h], 1);
            mbar_init(&free_h[h], GATERS);
        }
        mbar_init(wready, GATERS);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == MMA_WARP) {
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

    if (warp == PROD_WARP) {
        // ------------------------------ producer ------------------------------
        if (lane == 0) {
            tma_prefetch_desc(&tmZ);
            if (args.has_mask) tma_prefetch_desc(&tmMask);
            const uint32_t bytes = Z_BYTES + (args.has_mask ? MASK_BYTES : 0);
            bool ok = true;
            int lt = 0;
            for (; lt < n_local; ++lt) {
                const int s = lt % SLOTS;
                // Slot s last held tile lt - SLOTS: its gating (hence its MMAs and statistics) is done.
                if (lt >= SLOTS &&
                    !wait_bounded(&tile_done[s], (uint32_t)(lt / SLOTS - 1) & 1u, abort_flag, ctl, SITE_PRO | 1, lt)) {
                    ok = false;
                    break;
                }
                int i, j0;
                tile_coords(lt, i, j0);
                uint8_t *dst = zsm + s * Z_BYTES;
                mbar_arrive_expect_tx(&zfull[s], bytes);
                tma_load_3d(dst, &tmZ, &zfull[s], 0, j0, i);
                tma_load_3d(dst + Z_HALF, &tmZ, &zfull[s], 64, j0, i);
                if (args.has_mask) tma_load_2d(msm + s * MASK_BYTES, &tmMask, &zfull[s], j0, i);
            }
            if (!ok) *abort_flag = 1;
            // Let the last load into each slot land before shared memory is released (the
            // consumers may have stopped early).
            for (int t = lt - 1; t >= 0 && t >= lt - SLOTS; --t)
                wait_drain(&zfull[t % SLOTS], (uint32_t)(t / SLOTS) & 1u, ctl.timeout_ns);
        }
    } else if (warp == MMA_WARP) {
        // ------------------------------ MMA issuer ------------------------------
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(128, TILE, 0, 0);
            // Accumulators of half h (a or b): values at COL_D + 128 h, gates 64 columns on.
            auto issue_half = [&](int h, int s) {
                const uint32_t zb = smem_u32(zsm + s * Z_BYTES);
#pragma unroll
                for (int p = 0; p < 2; ++p) {
                    const uint32_t d = tmem_base + COL_D + (uint32_t)(h * 128 + p * 64);
                    const uint32_t wa = tmem_base + COL_W + (uint32_t)((2 * h + p) * 64);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t koff = (uint32_t)((kk >> 2) * Z_HALF + (kk & 3) * 32);
                        mma_bf16_ts(d, wa + (uint32_t)(kk * 8), sdesc_sw128(zb + koff, 16, 1024), idesc,
                                    kk ? 1u : 0u);
                    }
                }
            };
            bool ok = wait_bounded(wready, 0, abort_flag, ctl, SITE_PRO | 2, 0);
            for (int lt = 0; ok && lt < n_local; ++lt) {
                const int s = lt % SLOTS;
                const uint32_t ppar = (uint32_t)(lt - 1) & 1u;
                if (!wait_bounded(&zfull[s], (uint32_t)(lt / SLOTS) & 1u, abort_flag, ctl, SITE_PRO | 3, lt) ||
                    (lt > 0 && !wait_bounded(&free_h[0], ppar, abort_flag, ctl, SITE_PRO | 4, lt))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                issue_half(0, s);
                mma_commit(&mma_h[0]);
                if (lt > 0 && !wait_bounded(&free_h[1], ppar, abort_flag, ctl, SITE_PRO | 5, lt)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                issue_half(1, s);
                mma_commit(&mma_h[1]);
            }
            if (!ok) *abort_flag = 1;
            mma_commit(drain);
            wait_drain(drain, 0, ctl.timeout_ns);
        }
    } else if (warp >= GATERS) {
        // ------------------------------ statistics ------------------------------
        // Thread t: cell t / 2 of the tile, channel half t % 2 (its partner is lane ^ 1).
        const int t = (warp - GATERS) * 32 + lane;
        const int cell = t >> 1, hh = t & 1;
        bool ok = true;
        for (int lt = 0; lt < n_local; ++lt) {
            const int s = lt % SLOTS;
            if (!(ok = warp_wait(&zfull[s], (uint32_t)(lt / SLOTS) & 1u, abort_flag, ctl, SITE_PRO | 6, lt))) break;
            const uint8_t *zr = zsm + s * Z_BYTES + cell * 128;
            RowStats st;
            st.s = st.ss = make_float2(0.f, 0.f);
            st.k = bf16_bits_to_float(*reinterpret_cast<const uint16_t *>(zr + ((cell & 7) << 4)));
#pragma unroll
            for (int kc = 0; kc < 8; ++kc) {
                const uint4 u = *reinterpret_cast<const uint4 *>(zr + hh * Z_HALF + ((kc ^ (cell & 7)) << 4));
                stats_add(st, u.x);
                stats_add(st, u.y);
                stats_add(st, u.z);
                stats_add(st, u.w);
            }
            const float2 f = stats_finish(st, args.eps);  // (mu, r)
            if (hh == 0) {
                float *sp = reinterpret_cast<float *>(&stats[s * (TILE / 2) + (cell >> 1)]);
                sp[cell & 1] = f.y;
                sp[2 + (cell & 1)] = -f.x * f.y;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&stat_done[s]);
        }
        if (!ok && lane == 0) *abort_flag = 1;
    } else {
        // ------------------------------ gaters ------------------------------
        const int q = warp & 3, h = warp >> 2;  // lane quadrant (channels 32q ..), cell half (cells 32h ..)
        const int c = 32 * q + lane;            // this thread's output channel
        const uint32_t lane_base = tmem_base + ((uint32_t)(32 * q) << 16);

        // Weights into tensor memory: warp half h writes W_a, W_ag (h = 0) or W_b, W_bg (h = 1),
        // row c of each, as W' = W gamma rounded to bf16 (the gate weight also halved), and
        // the per-channel constants s (row sum of the rounded W') and t (W beta + bias; halved
        // for the gate) into the shared table.
        {
            const __nv_bfloat16 *wsrc[2] = {h ? args.w_b : args.w_a, h ? args.w_bg : args.w_ag};
            const __nv_bfloat16 *bsrc[2] = {h ? args.b_b : args.b_a, h ? args.b_bg : args.b_ag};
#pragma unroll 1
            for (int p = 0; p < 2; ++p) {
                const float scale = p ? 0.5f : 1.f;
                const uint4 *row = reinterpret_cast<const uint4 *>(wsrc[p] + (size_t)c * 128);
                uint32_t packed[64];
                float sum = 0.f, tb = 0.f;
#pragma unroll
                for (int k8 = 0; k8 < 16; ++k8) {
                    const uint4 u = __ldg(row + k8);
                    const uint32_t wd[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int k = 8 * k8 + 2 * e;
                        float2 w = unpack_bf16x2(wd[e]);
                        if (args.ln_b) tb = fmaf(w.x, __bfloat162float(args.ln_b[k]),
                                                 fmaf(w.y, __bfloat162float(args.ln_b[k + 1]), tb));
                        if (args.ln_w) w = __fmul2_rn(w, ld_pair_bf16(args.ln_w, k));
                        w = __fmul2_rn(w, make_float2(scale, scale));
                        packed[4 * k8 + e] = pack_bf16x2(w.x, w.y);
                        const float2 wr = unpack_bf16x2(packed[4 * k8 + e]);  // the rounded W' the MMA reads
                        sum += wr.x + wr.y;
                    }
                }
                tmem_st64(lane_base + COL_W + (uint32_t)((2 * h + p) * 64), packed);
                if (bsrc[p]) tb += __bfloat162float(bsrc[p][c]);
                cst[(2 * (2 * h + p)) * 128 + c] = sum;
                cst[(2 * (2 * h + p) + 1) * 128 + c] = scale * tb;
            }
            tmem_st_wait();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(wready);
        }
        named_bar_sync(5, 32 * GATERS);  // the constant table is complete
        // (s, t) per channel: a values, a gates, b values, b gates.
        float2 S2[4], T2[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            const float sv = cst[(2 * m) * 128 + c], tv = cst[(2 * m + 1) * 128 + c];
            S2[m] = make_float2(sv, sv);
            T2[m] = make_float2(tv, tv);
        }

        bool ok = true;
        for (int lt = 0; ok && lt < n_local; ++lt) {
            const int s = lt % SLOTS;
            int i, j0;
            tile_coords(lt, i, j0);
            // The two warps of a lane quadrant share staging buffers and named barriers, so
            // after every wait they agree (bar.red) on whether to go on.
            ok = warp_wait(&stat_done[s], (uint32_t)(lt / SLOTS) & 1u, abort_flag, ctl, SITE_PRO | 7, lt);
            if (!(ok = bar_red_and(6 + q, 64, ok))) break;
            const float4 *st4 = stats + s * (TILE / 2) + 16 * h;  // this warp's 16 cell pairs
            const uint32_t *m2 = reinterpret_cast<const uint32_t *>(msm + s * MASK_BYTES) + 16 * h;
#pragma unroll 1
            for (int o = 0; o < 2; ++o) {  // a, then b
                ok = warp_wait(&mma_h[o], (uint32_t)lt & 1u, abort_flag, ctl, SITE_PRO | (8 + o), lt);
                if (!(ok = bar_red_and(6 + q, 64, ok))) break;
                tc_fence_after();
                uint32_t V[32], G[32];
                const uint32_t ta = lane_base + COL_D + (uint32_t)(o * 128 + 32 * h);
                tmem_ld32(ta, V);
                tmem_ld32(ta + 64, G);
                tmem_ld_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&free_h[o]);
                const float2 Sv = S2[2 * o], Tv = T2[2 * o], Sg = S2[2 * o + 1], Tg = T2[2 * o + 1];
                uint32_t P[16];
#pragma unroll
                for (int pp = 0; pp < 16; ++pp) {
                    const float4 sr = st4[pp];  // (r0, r1, -mu0 r0, -mu1 r1)
                    const float2 R = make_float2(sr.x, sr.y), NMR = make_float2(sr.z, sr.w);
                    float2 hm;
                    if (args.has_mask) {
                        hm = __fmul2_rn(unpack_bf16x2(m2[pp]), make_float2(0.5f, 0.5f));
                    } else {
                        const int jc = j0 + 32 * h + 2 * pp;
                        hm = make_float2(jc < args.N ? 0.5f : 0.f, jc + 1 < args.N ? 0.5f : 0.f);
                    }
                    const float2 v = __ffma2_rn(R, make_float2(__uint_as_float(V[2 * pp]), __uint_as_float(V[2 * pp + 1])),
                                                __ffma2_rn(NMR, Sv, Tv));
                    const float2 g = __ffma2_rn(R, make_float2(__uint_as_float(G[2 * pp]), __uint_as_float(G[2 * pp + 1])),
                                                __ffma2_rn(NMR, Sg, Tg));
                    const float2 th = make_float2(tanh_approx(g.x), tanh_approx(g.y));
                    const float2 y = __fmul2_rn(__ffma2_rn(th, hm, hm), v);
                    P[pp] = pack_bf16x2(y.x, y.y);
                }
                if (o == 1) {
                    // Statistics and mask row of slot s are no longer needed.
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&tile_done[s]);
                }
                // Stage [32 ch][64 cells] (row = lane, 16-byte chunk k at k ^ (row & 7)), then one
                // TMA store of 32 rows of 128 bytes by warp h = 0 of the quadrant.
                uint8_t *buf = stg + (2 * q + o) * STG_BYTES;
                const bool issuer = h == 0 && lane == 0;
                if (issuer) tma_store_wait_read<1>();  // the store that last used buf (one tile ago) has read it
                named_bar_sync(1 + q, 64);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    *reinterpret_cast<uint4 *>(buf + lane * 128 + (((4 * h + kk) ^ (lane & 7)) << 4)) =
                        make_uint4(P[4 * kk], P[4 * kk + 1], P[4 * kk + 2], P[4 * kk + 3]);
                fence_proxy_async_smem();
                named_bar_sync(1 + q, 64);
                if (issuer) {
                    tma_store_3d(o ? &tmB : &tmA, buf, j0, i, 32 * q);
                    tma_store_commit();
                }
            }
        }
        if (!ok && lane == 0) *abort_flag = 1;
        if (h == 0 && lane == 0) tma_store_wait_all<0>();
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == MMA_WARP) tmem_dealloc(tmem_base, 512);
}

size_t prologue_tc_smem() { return pro::SMEM; }

cudaError_t prologue_tc_setup() {
    return cudaFuncSetAttribute(prologue_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pro::SMEM);
}

cudaError_t launch_prologue_tc(const PrologueMaps &m, const PrologueArgs &a, int grid, cudaStream_t s) {
    prologue_tc_kernel<<<grid, pro::THREADS, pro::SMEM, s>>>(m.z, m.mask, m.a, m.b, a);
    return cudaGetLastError();
}

__global__ void mask_pad_kernel(const __nv_bfloat16 *__restrict__ mask, __nv_bfloat16 *__restrict__ dst, int N,
                                int ld) {
    const size_t i = blockIdx.x;
    for (int j = threadIdx.x; j < ld; j += blockDim.x) dst[i * ld + j] = j < N ? mask[i * N + j] : __float2bfloat16(0.f);
}

cudaError_t launch_mask_pad(const __nv_bfloat16 *mask, __nv_bfloat16 *dst, int N, int rows, int ld, cudaStream_t s) {
    mask_pad_kernel<<<rows, 128, 0, s>>>(mask, dst, N, ld);
    return cudaGetLastError();
}

}  // namespace trimul

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
// Tiles are 128 consecutive cells of one residue row (z[i][j0 .. j0+127][:],
// one contiguous 32 KB block). Per tile:
//   TMA  z tile -> smem (128-byte swizzle, two 64-channel halves)
//   LN   in place, fp32 statistics, bf16 result (the MMA's A operand)
//   MMA  D[128 cells][512] = zh * [W_a; W_ag; W_b; W_bg]^T as two N = 256
//        halves (a-half, b-half) into all 512 TMEM columns
//   gate TMEM -> registers -> sigmoid, mask -> [64 ch][128 cells] smem
//   TMA  store of each 64-channel slab to a or b (4 slabs per tile)
// The four weight matrices (128 KB bf16) stay resident in shared memory for
// the whole persistent CTA. The loop is software-pipelined so that the MMA of
// the next tile runs while this tile is gated and stored, and the z load of
// tile t+2 is in flight for a whole iteration.
#include "kernels.h"

namespace trimul {
namespace pro {
constexpr int TILE = 128;
constexpr int THREADS = 256;
constexpr int W_HALF = 512 * 128;     // one 64-channel K half of the 4 stacked weights: 64 KB
constexpr int W_BYTES = 2 * W_HALF;   // 128 KB
constexpr int Z_HALF = TILE * 128;    // 16 KB
constexpr int Z_BYTES = 2 * Z_HALF;   // 32 KB
constexpr int ST_BYTES = 64 * TILE * 2;  // 16 KB staging slab [64 ch][128 cells]
constexpr int NUM_ST = 2;
constexpr int BAR_BYTES = 128;
constexpr size_t SMEM = 1024 + (size_t)W_BYTES + 2 * Z_BYTES + NUM_ST * ST_BYTES + BAR_BYTES;
static_assert(SMEM <= 232448, "shared memory budget");
}  // namespace pro

// In-place LayerNorm of one swizzled z tile: 2 threads per cell (one per
// 64-channel half), statistics in fp32, partner exchange by shuffle.
__device__ __forceinline__ void layer_norm_tile_sw128(uint8_t *zt, const __nv_bfloat16 *gw, const __nv_bfloat16 *gb,
                                                      float eps) {
    const int t = threadIdx.x;
    const int r = t >> 1, h = t & 1;
    uint8_t *rowp = zt + h * pro::Z_HALF + r * 128;
    float v[64];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const int kc = (q + 4 * h) & 7;  // staggered so the two halves hit different banks
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

__global__ void __launch_bounds__(pro::THREADS, 1)
    prologue_tc_kernel(const __grid_constant__ CUtensorMap tmWa, const __grid_constant__ CUtensorMap tmWag,
                       const __grid_constant__ CUtensorMap tmWb, const __grid_constant__ CUtensorMap tmWbg,
                       const __grid_constant__ CUtensorMap tmZ, const __grid_constant__ CUtensorMap tmA,
                       const __grid_constant__ CUtensorMap tmB, const PrologueArgs args) {
    using namespace pro;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *wsm = smem;
    uint8_t *zsm = smem + W_BYTES;               // [2] z tiles
    uint8_t *stsm = zsm + 2 * Z_BYTES;           // [2] staging slabs
    uint64_t *bars = reinterpret_cast<uint64_t *>(stsm + NUM_ST * ST_BYTES);
    uint64_t *wbar = bars;       // weights landed
    uint64_t *zfull = bars + 1;  // [2] z tile landed
    uint64_t *mma_a = bars + 3;  // a-half projections done
    uint64_t *mma_b = bars + 4;  // b-half projections done
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
        mbar_init(&zfull[0], 1);
        mbar_init(&zfull[1], 1);
        mbar_init(mma_a, 1);
        mbar_init(mma_b, 1);
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
    int last_load[2] = {-1, -1};  // thread 0: last tile loaded into each z buffer
    auto load_z = [&](int lt) {
        int i, j0;
        tile_coords(lt, i, j0);
        last_load[lt & 1] = lt;
        uint8_t *dst = zsm + (lt & 1) * Z_BYTES;
        mbar_arrive_expect_tx(&zfull[lt & 1], Z_BYTES);
        tma_load_3d(dst, &tmZ, &zfull[lt & 1], 0, j0, i);
        tma_load_3d(dst + Z_HALF, &tmZ, &zfull[lt & 1], 64, j0, i);
    };
    // One projection half: D[:, half*256 .. +255] = zh * W[half*256 .. +255]^T (K = 128).
    auto issue_half = [&](int half, int buf) {
        const uint32_t idesc = idesc_bf16(128, 256, 0, 0);
        const uint32_t za = smem_u32(zsm + buf * Z_BYTES);
        const uint32_t wb = smem_u32(wsm) + (uint32_t)(half * 256 * 128);
        const uint32_t d = tmem_base + (uint32_t)(half * 256);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const uint32_t koff = (uint32_t)((kk >> 2) * Z_HALF + (kk & 3) * 32);
            const uint32_t woff = (uint32_t)((kk >> 2) * W_HALF + (kk & 3) * 32);
            mma_bf16(d, sdesc_sw128(za + koff, 16, 1024), sdesc_sw128(wb + woff, 16, 1024), idesc, kk ? 1u : 0u);
        }
    };

    if (threadIdx.x == 0) {
        mbar_arrive_expect_tx(wbar, W_BYTES);
        const CUtensorMap *wm[4] = {&tmWa, &tmWag, &tmWb, &tmWbg};
#pragma unroll
        for (int w = 0; w < 4; ++w)
#pragma unroll
            for (int kh = 0; kh < 2; ++kh) tma_load_2d(wsm + kh * W_HALF + w * 128 * 128, wm[w], wbar, kh * 64, 0);
        if (n_local > 0) load_z(0);
        if (n_local > 1) load_z(1);
    }

    int st_round = 0;  // staging slabs used so far (alternating buffers)
    // Gate, mask and store one 64-channel slab of a (which = 0) or b (which = 1).
    auto slab = [&](int which, int hh, float m, int i, int j0) {
        const int q = warp & 3, sub = warp >> 2;
        const int r = q * 32 + lane;
        const int ch0 = hh * 64 + sub * 32;
        uint32_t V[32], G[32];
        __syncwarp();  // tcgen05.ld is warp-wide; thread 0 may have just issued a store alone
        const uint32_t lane_base = tmem_base + ((uint32_t)(q * 32) << 16);
        tmem_ld32(lane_base + (uint32_t)(which * 256 + ch0), V);
        tmem_ld32(lane_base + (uint32_t)(which * 256 + 128 + ch0), G);
        tmem_ld_wait();
        uint8_t *st = stsm + (st_round & 1) * ST_BYTES;
        ++st_round;
        if (threadIdx.x == 0) tma_store_wait_read<1>();
        __syncthreads();
        const __nv_bfloat16 *bv = which ? args.b_b : args.b_a;
        const __nv_bfloat16 *bg = which ? args.b_bg : args.b_ag;
        __nv_bfloat16 *stv = reinterpret_cast<__nv_bfloat16 *>(st);
#pragma unroll
        for (int k = 0; k < 32; ++k) {
            const int c = ch0 + k;
            const float pv = __uint_as_float(V[k]) + ld_vec_bf16(bv, c, 0.f);
            const float pg = __uint_as_float(G[k]) + ld_vec_bf16(bg, c, 0.f);
            stv[(sub * 32 + k) * TILE + r] = __float2bfloat16_rn(m * sigmoid_fast(pg) * pv);
        }
        fence_proxy_async_smem();
        __syncthreads();
        if (threadIdx.x == 0) {
            tma_store_3d(which ? &tmB : &tmA, st, j0, i, hh * 64);
            tma_store_commit();
        }
    };

    bool ok = __syncthreads_and(wait_bounded(wbar, 0, abort_flag, ctl, SITE_PRO | 1, 0));
    if (ok && n_local > 0) {
        ok = __syncthreads_and(wait_bounded(&zfull[0], 0, abort_flag, ctl, SITE_PRO | 2, 0));
        if (ok) {
            layer_norm_tile_sw128(zsm, args.ln_w, args.ln_b, args.eps);
            fence_proxy_async_smem();
            __syncthreads();
            if (threadIdx.x == 0) {
                tc_fence_after();
                issue_half(0, 0);
                mma_commit(mma_a);
                issue_half(1, 0);
                mma_commit(mma_b);
            }
        }
    }

    for (int lt = 0; ok && lt < n_local; ++lt) {
        const int cur = lt & 1, nxt = cur ^ 1;
        int i, j0;
        tile_coords(lt, i, j0);
        const int rr = (warp & 3) * 32 + lane;  // the cell this thread gates
        const int jj = j0 + rr;
        float m = 0.f;
        if (jj < args.N) m = args.mask ? __bfloat162float(args.mask[(size_t)i * args.N + jj]) : 1.f;

        // a-half of tile lt
        ok = __syncthreads_and(wait_bounded(mma_a, (uint32_t)lt & 1u, abort_flag, ctl, SITE_PRO | 3, lt));
        if (!ok) break;
        tc_fence_after();
        slab(0, 0, m, i, j0);
        slab(0, 1, m, i, j0);

        // LayerNorm of tile lt+1, then its a-half MMA into the columns just drained
        if (lt + 1 < n_local) {
            ok = __syncthreads_and(
                wait_bounded(&zfull[nxt], (uint32_t)((lt + 1) >> 1) & 1u, abort_flag, ctl, SITE_PRO | 4, lt));
            if (!ok) break;
            layer_norm_tile_sw128(zsm + nxt * Z_BYTES, args.ln_w, args.ln_b, args.eps);
            fence_proxy_async_smem();
            tc_fence_before();
            __syncthreads();
            if (threadIdx.x == 0) {
                tc_fence_after();
                issue_half(0, nxt);
                mma_commit(mma_a);
            }
        }

        // b-half of tile lt; its completion also frees z buffer `cur`
        ok = __syncthreads_and(wait_bounded(mma_b, (uint32_t)lt & 1u, abort_flag, ctl, SITE_PRO | 5, lt));
        if (!ok) break;
        tc_fence_after();
        if (threadIdx.x == 0 && lt + 2 < n_local) load_z(lt + 2);
        slab(1, 0, m, i, j0);
        slab(1, 1, m, i, j0);
        tc_fence_before();
        __syncthreads();
        if (threadIdx.x == 0 && lt + 1 < n_local) {
            tc_fence_after();
            issue_half(1, nxt);
            mma_commit(mma_b);
        }
    }

    // Teardown: stores drained, loads landed, MMAs finished, TMEM released.
    if (threadIdx.x == 0) {
        tma_store_wait_all<0>();
        if (!ok) {
            // Copies that may still be in flight after an abort.
            wait_drain(wbar, 0, ctl.timeout_ns);
            for (int b = 0; b < 2; ++b)
                if (last_load[b] >= 0) wait_drain(&zfull[b], (uint32_t)(last_load[b] >> 1) & 1u, ctl.timeout_ns);
        }
        mma_commit(drain);
        wait_drain(drain, 0, ctl.timeout_ns);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem_base, 512);
}

size_t prologue_tc_smem() { return pro::SMEM; }

cudaError_t prologue_tc_setup() {
    return cudaFuncSetAttribute(prologue_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)pro::SMEM);
}

cudaError_t launch_prologue_tc(const PrologueMaps &m, const PrologueArgs &a, int grid, cudaStream_t s) {
    prologue_tc_kernel<<<grid, pro::THREADS, pro::SMEM, s>>>(m.w[0], m.w[1], m.w[2], m.w[3], m.z, m.a, m.b, a);
    return cudaGetLastError();
}

}  // namespace trimul

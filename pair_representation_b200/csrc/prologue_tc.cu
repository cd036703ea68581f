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
// one contiguous 32 KB block). The four weight matrices (128 KB bf16) stay in
// shared memory for the whole persistent CTA. Roles (416 threads), coupled
// only through mbarriers:
//   warp 12 (control): TMA loads of z (two tiles ahead), the two projection
//     MMAs per tile (a-half D[:, 0:256] = zh [W_a; W_ag]^T, b-half
//     D[:, 256:512] = zh [W_b; W_bg]^T, M = 128 cells, N = 256, K = 128, all
//     512 TMEM columns).
//   warps 8-11 (normalisers): LayerNorm of each landed tile in place (fp32
//     statistics, two threads per cell), ahead of its MMAs.
//   warps 0-7 (workers): gating of 32 cells x 32 channels of a and of b: TMEM
//     is read in the 16-lane fragment layout, m * sigmoid(g) * v is formed in
//     packed fp32x2, the bf16 results are written channel-major with
//     stmatrix.trans into a 64-byte-swizzled 2 KB buffer of the warp and
//     stored by that warp's own TMA store, so no warp waits on global writes.
// The control warp issues the next tile's a-half MMAs as soon as that tile is
// normalised and the workers have read the a-half columns, and the b-half as
// soon as they have read the b-half columns: tensor work, gating,
// normalisation and the z loads of two tiles ahead overlap. Every wait sleeps
// in mbarrier.try_wait rather than spinning, which keeps issue slots and the
// shared-memory pipe free for the warps doing work.
//
// MXFP8 modes write a and b directly as the E4M3 operands of the block-scaled
// contraction (OCP Microscaling v1.0: blocks of 32 along the contracted index,
// one E8M0 scale each), so no separate pass reads the bf16 values back. A gating
// warp's 32 cells x 32 channels are 32 whole blocks when its 32 cells run along
// the contracted index: in PRO_MX_ROWS (outgoing, K = the column k of a_ik) the
// usual row tiles already do; in PRO_MX_COLS (incoming, K = the row k of a_ki) a
// tile is 32 rows x 4 columns, loaded column by column, so warp q holds column q.
// The warp rounds its values to bf16 exactly as the bf16 mode stores them, then
// each lane quantises one channel's block from the staging buffer and writes its
// 32 codes back in place for the warp's TMA store; the lane stores the scale byte.
#include "kernels.h"
#include "mx_block.cuh"
#include "tile_ops.cuh"

namespace trimul {
namespace pro {
constexpr int TILE = 128;
constexpr int WORKERS = 8;
constexpr int NORMS = 4;
constexpr int CTRL_WARP = WORKERS + NORMS;
constexpr int THREADS = 32 * (CTRL_WARP + 1);
constexpr int W_HALF = 512 * 128;       // one 64-channel K half of the 4 stacked weights: 64 KB
constexpr int W_BYTES = 2 * W_HALF;     // 128 KB
constexpr int Z_HALF = TILE * 128;      // 16 KB
constexpr int Z_BYTES = 2 * Z_HALF;     // 32 KB
constexpr int ST_BYTES = 32 * 32 * 2;   // 2 KB per warp buffer: [32 ch][32 cells], 64-byte swizzle
constexpr int ST_PER_WARP = 2;
constexpr int MASK_SLOTS = 3;           // mask rows of tiles lt .. lt + 2 (indexed lt % 3)
constexpr int MASK_BYTES = TILE * 2;     // one bf16 mask row segment per tile
constexpr int PB_BYTES = 4 * 128 * 2;    // folded projection biases, bf16 [a, ag / 2, b, bg / 2][128]
constexpr int BAR_BYTES = 128;
constexpr size_t SMEM = 1024 + (size_t)W_BYTES + 2 * Z_BYTES + (size_t)WORKERS * ST_PER_WARP * ST_BYTES +
                        MASK_SLOTS * MASK_BYTES + PB_BYTES + BAR_BYTES;
static_assert(SMEM <= 232448, "shared memory budget");
}  // namespace pro

// kVec: some LayerNorm affine or projection bias is present (general path). The
// LayerNorm affine is folded into the projections once per CTA (W' = W diag(gamma) in
// shared memory, b' = b + W beta), so the normalisers always run the plain
// LayerNorm and the gating adds b' from shared memory; without them the kernel
// skips every per-channel vector access. kMode: PRO_BF16,
// PRO_MX_ROWS or PRO_MX_COLS.
template <bool kVec, int kMode>
__global__ void __launch_bounds__(pro::THREADS, 1)
    prologue_tc_kernel(const __grid_constant__ CUtensorMap tmWa, const __grid_constant__ CUtensorMap tmWag,
                       const __grid_constant__ CUtensorMap tmWb, const __grid_constant__ CUtensorMap tmWbg,
                       const __grid_constant__ CUtensorMap tmZ, const __grid_constant__ CUtensorMap tmMask,
                       const __grid_constant__ CUtensorMap tmA,
                       const __grid_constant__ CUtensorMap tmB, const PrologueArgs args) {
    using namespace pro;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *wsm = smem;
    uint8_t *zsm = smem + W_BYTES;                 // [2] z tiles
    uint8_t *stsm = zsm + 2 * Z_BYTES;             // [8 warps][2] staging buffers
    uint8_t *msm = stsm + WORKERS * ST_PER_WARP * ST_BYTES;  // [3] mask rows (bf16)
    __nv_bfloat16 *pbias = reinterpret_cast<__nv_bfloat16 *>(msm + MASK_SLOTS * MASK_BYTES);  // kVec: b'
    uint64_t *bars = reinterpret_cast<uint64_t *>(msm + MASK_SLOTS * MASK_BYTES + PB_BYTES);
    uint64_t *wbar = bars;        // weights landed
    uint64_t *zfull = bars + 1;   // [2] z tile landed
    uint64_t *mma_a = bars + 3;   // a-half projections done
    uint64_t *mma_b = bars + 4;   // b-half projections done
    uint64_t *a_free = bars + 5;  // workers: a-half TMEM columns read (8 arrivals)
    uint64_t *b_free = bars + 6;  // workers: b-half TMEM columns read (8 arrivals)
    uint64_t *drain = bars + 7;
    uint64_t *ln_done = bars + 8; // [2] normalisers: tile in z buffer b normalised (4 arrivals)
    uint64_t *wprep = bars + 10;  // workers: gate weights halved (8 arrivals)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 11);
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
        mbar_init(&ln_done[0], NORMS);
        mbar_init(&ln_done[1], NORMS);
        mbar_init(a_free, WORKERS);
        mbar_init(b_free, WORKERS);
        mbar_init(drain, 1);
        mbar_init(wprep, WORKERS);
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
    if (args.clear_status && blockIdx.x == 0 && threadIdx.x == 0) *ctl.status = DeviceStatus{0, 0, 0, 0};

    // Tile lt of this CTA: z row i, columns j0 .. j0+127; PRO_MX_COLS: rows i .. i+31,
    // columns j0 .. j0+3.
    auto tile_coords = [&](int lt, int &i, int &j0) {
        const int tile = (int)blockIdx.x + lt * (int)gridDim.x;
        const int r = tile / args.jt_tiles;
        if (kMode == PRO_MX_COLS) {
            i = 32 * r;
            j0 = 4 * (tile - r * args.jt_tiles);
        } else {
            i = r;
            j0 = (tile - r * args.jt_tiles) * TILE;
        }
    };

    if (warp == CTRL_WARP) {
        // ------------------------------ control warp ------------------------------
        if (lane == 0) {
            int last_load0 = -1, last_load1 = -1;
            auto load_z = [&](int lt) {
                int i, j0;
                tile_coords(lt, i, j0);
                if (lt & 1) last_load1 = lt; else last_load0 = lt;
                uint8_t *dst = zsm + (lt & 1) * Z_BYTES;
                mbar_arrive_expect_tx(&zfull[lt & 1], Z_BYTES + (args.has_mask ? MASK_BYTES : 0));
                if (kMode == PRO_MX_COLS) {
                    // Rows i .. i+31 of column j0 + c land as cells 32c .. 32c+31.
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        tma_load_3d(dst + c * 4096, &tmZ, &zfull[lt & 1], 0, j0 + c, i);
                        tma_load_3d(dst + Z_HALF + c * 4096, &tmZ, &zfull[lt & 1], 64, j0 + c, i);
                    }
                } else {
                    tma_load_3d(dst, &tmZ, &zfull[lt & 1], 0, j0, i);
                    tma_load_3d(dst + Z_HALF, &tmZ, &zfull[lt & 1], 64, j0, i);
                }
                // Mask slot lt % 3 last served tile lt - 3, whose gating (which reads its mask
                // first) ended before the b-half MMA of tile lt - 2, which this load waited for.
                // PRO_MX_COLS reads the
                // transposed mask: [4 columns][32 rows], the same cell order as z.
                if (args.has_mask) {
                    if (kMode == PRO_MX_COLS)
                        tma_load_2d(msm + (lt % MASK_SLOTS) * MASK_BYTES, &tmMask, &zfull[lt & 1], i, j0);
                    else
                        tma_load_2d(msm + (lt % MASK_SLOTS) * MASK_BYTES, &tmMask, &zfull[lt & 1], j0, i);
                }
            };
            // D[:, half*256 .. +255] = zh * W[half*256 .. +255]^T over K = 128.
            auto issue_half = [&](int half, int buf) {
                const uint32_t idesc = idesc_bf16(128, 256, 0, 0);
                const uint32_t za = smem_u32(zsm + buf * Z_BYTES);
                const uint32_t wb = smem_u32(wsm) + (uint32_t)(half * 256 * 128);
                const uint32_t d = tmem_base + (uint32_t)(half * 256);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t koff = (uint32_t)((kk >> 2) * Z_HALF + (kk & 3) * 32);
                    const uint32_t woff = (uint32_t)((kk >> 2) * W_HALF + (kk & 3) * 32);
                    mma_bf16(d, sdesc_sw128(za + koff, 16, 1024), sdesc_sw128(wb + woff, 16, 1024), idesc,
                             kk ? 1u : 0u);
                }
            };
            mbar_arrive_expect_tx(wbar, W_BYTES);
            const CUtensorMap *wm[4] = {&tmWa, &tmWag, &tmWb, &tmWbg};
#pragma unroll
            for (int w = 0; w < 4; ++w)
#pragma unroll
                for (int kh = 0; kh < 2; ++kh) tma_load_2d(wsm + kh * W_HALF + w * 128 * 128, wm[w], wbar, kh * 64, 0);
            if (n_local > 0) load_z(0);
            if (n_local > 1) load_z(1);
            bool ok = wait_bounded(wbar, 0, abort_flag, ctl, SITE_PRO | 1, 0) &&
                      wait_bounded(wprep, 0, abort_flag, ctl, SITE_PRO | 10, 0);
            for (int lt = 0; ok && lt < n_local; ++lt) {
                const uint32_t par = (uint32_t)lt & 1u, ppar = (uint32_t)(lt - 1) & 1u;
                if (!wait_bounded(&ln_done[lt & 1], (uint32_t)(lt >> 1) & 1u, abort_flag, ctl, SITE_PRO | 2, lt) ||
                    (lt > 0 && !wait_bounded(a_free, ppar, abort_flag, ctl, SITE_PRO | 3, lt))) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                issue_half(0, lt & 1);
                mma_commit(mma_a);
                if (lt > 0 && !wait_bounded(b_free, ppar, abort_flag, ctl, SITE_PRO | 4, lt)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                issue_half(1, lt & 1);
                mma_commit(mma_b);
                if (lt + 2 < n_local) {
                    // z buffer lt & 1 is free once both projection halves of tile lt have read it.
                    if (!wait_bounded(mma_b, par, abort_flag, ctl, SITE_PRO | 5, lt)) {
                        ok = false;
                        break;
                    }
                    load_z(lt + 2);
                }
            }
            if (!ok) {
                *abort_flag = 1;
                // Copies that may still be in flight after an abort.
                wait_drain(wbar, 0, ctl.timeout_ns);
                if (last_load0 >= 0) wait_drain(&zfull[0], (uint32_t)(last_load0 >> 1) & 1u, ctl.timeout_ns);
                if (last_load1 >= 0) wait_drain(&zfull[1], (uint32_t)(last_load1 >> 1) & 1u, ctl.timeout_ns);
            }
            mma_commit(drain);
            wait_drain(drain, 0, ctl.timeout_ns);
        }
    } else if (warp >= WORKERS) {
        // ------------------------------ normalisers ------------------------------
        const int t = (warp - WORKERS) * 32 + lane;  // 0..127: cells t/2 and 64 + t/2, channel half t % 2
        bool ok = true;
        for (int lt = 0; lt < n_local; ++lt) {
            const int b = lt & 1;
            if (!(ok = warp_wait(&zfull[b], (uint32_t)(lt >> 1) & 1u, abort_flag, ctl, SITE_PRO | 6, lt))) break;
            uint8_t *tile = zsm + b * Z_BYTES;
            // The affine part is folded into the projections (kVec): plain LayerNorm here.
            ln_row_sw128<false>(tile, Z_HALF, t >> 1, t & 1, nullptr, nullptr, args.eps);
            ln_row_sw128<false>(tile, Z_HALF, 64 + (t >> 1), t & 1, nullptr, nullptr, args.eps);
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&ln_done[b]);
        }
        if (!ok && lane == 0) *abort_flag = 1;
    } else {
        // ------------------------------ worker warps ------------------------------
        const int q = warp & 3, sub = warp >> 2;  // TMEM lane quadrant (cells 32q..32q+31), channel half
        uint8_t *stw = stsm + warp * ST_PER_WARP * ST_BYTES;
        int st_round = 0;
        // MXFP8 modes: bytes between the scale arrays of consecutive channels (the scale
        // offset is linear in the channel; the arrays stay far below 4 GB).
        auto sf_cstride = [&](int o) {
            return (uint32_t)args.sf_row_tiles[o] * (uint32_t)args.kchunks * (uint32_t)args.sf_chunks[o] * 512u;
        };

        // One gated slab waits in its staging buffer while the next slab is gated: the
        // next slab's tensor-memory loads, its gating and (MXFP8 modes) the pending
        // slab's quantisation form one straight-line stretch the compiler can
        // interleave; then the pending slab is stored.
        struct Pending {
            uint8_t *buf;
            int which, ch0, ox, orow;
            uint32_t sfo;  // scale offset of channel 0 (MXFP8 modes)
            bool on;
        } pend;
        pend.buf = stw;
        pend.on = false;
        // Lane l's channel ch0 + l of the pending slab: its 32 bf16 values are buffer row l
        // (logical 16-byte chunk c at c ^ ((l >> 1) & 3)).
        auto pending_row = [&](uint32_t (&w)[16]) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const uint4 u = *reinterpret_cast<const uint4 *>(pend.buf + lane * 64 + ((c ^ ((lane >> 1) & 3)) << 4));
                w[4 * c] = u.x;
                w[4 * c + 1] = u.y;
                w[4 * c + 2] = u.z;
                w[4 * c + 3] = u.w;
            }
        };
        // Store the pending slab; MXFP8 modes first write the quantised codes back in place
        // (lane l's 32 codes at bytes 32 l .., a dense [32 ch][32 B] box) and the scale byte.
        // Every lane must have read its row before.
        auto store_pending = [&](const uint32_t (&q8)[8], int e) {
            if (kMode != PRO_BF16) {
                __syncwarp();
                uint4 *dst = reinterpret_cast<uint4 *>(pend.buf + lane * 32);
                dst[0] = make_uint4(q8[0], q8[1], q8[2], q8[3]);
                dst[1] = make_uint4(q8[4], q8[5], q8[6], q8[7]);
                args.sf[pend.which][pend.sfo + (uint32_t)(pend.ch0 + lane) * sf_cstride(pend.which)] = (uint8_t)(e + 127);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
                tma_store_3d(pend.which ? &tmB : &tmA, pend.buf, pend.ox, pend.orow, pend.ch0);
                tma_store_commit();
            }
            pend.on = false;
        };
        auto flush = [&]() {
            if (!pend.on) return;
            uint32_t q8[8];
            int e = 0;
            if (kMode != PRO_BF16) {
                uint32_t w[16];
                __syncwarp();
                pending_row(w);
                e = mx_quantize32_bf16(w, q8);
            }
            store_pending(q8, e);
        };

        // Gate 32 cells x 32 channels of a (which = 0) or b (which = 1), channels hh*64 + sub*32 ..,
        // for the outputs at (x = ox .. ox+31, row orow). `release` (if set) is signalled
        // right after the slab's tensor-memory reads, so the next tile's MMAs into these
        // columns overlap the gating and the stores.
        auto slab = [&](int which, int hh, const float (&hm)[4], int ox, int orow, uint32_t sfo, uint64_t *release) {
            const int ch0 = hh * 64 + sub * 32;
            uint32_t V[2][16], G[2][16];
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const uint32_t ta = tmem_base + ((uint32_t)(q * 32 + 16 * hf) << 16) + (uint32_t)(which * 256 + ch0);
                tmem_ld16x256_x4(ta, V[hf]);
                tmem_ld16x256_x4(ta + 128, G[hf]);
            }
            // The pending slab's row is read (and quantised below) whether or not a slab is
            // pending: pend.buf always points into this warp's staging buffers.
            uint32_t w[16];
            if (kMode != PRO_BF16) {
                __syncwarp();
                pending_row(w);
            }
            tmem_ld_wait();
            if (release) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(release);
            }
            uint32_t P[16];  // packed bf16 pairs: [hf][k][e] -> P[hf * 8 + k * 2 + e]
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
#pragma unroll
                for (int k = 0; k < 4; ++k) {
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        float2 g = make_float2(__uint_as_float(G[hf][4 * k + 2 * e]),
                                               __uint_as_float(G[hf][4 * k + 2 * e + 1]));
                        float2 v = make_float2(__uint_as_float(V[hf][4 * k + 2 * e]),
                                               __uint_as_float(V[hf][4 * k + 2 * e + 1]));
                        // g holds (W_g zh) / 2: the gate weights were halved in shared memory.
                        if (kVec) {
                            const int c = ch0 + 8 * k + 2 * (lane & 3);
                            g = __fadd2_rn(g, ld_pair_bf16(pbias + (2 * which + 1) * 128, c));
                            v = __fadd2_rn(v, ld_pair_bf16(pbias + 2 * which * 128, c));
                        }
                        const float h2 = hm[hf * 2 + e];
                        const float2 hh2 = make_float2(h2, h2);
                        const float2 th = make_float2(tanh_approx(g.x), tanh_approx(g.y));
                        const float2 y = __fmul2_rn(__ffma2_rn(th, hh2, hh2), v);
                        P[hf * 8 + k * 2 + e] = pack_bf16x2(y.x, y.y);
                    }
                }
            }
            uint32_t q8[8];
            int qe = 0;
            if (kMode != PRO_BF16) qe = mx_quantize32_bf16(w, q8);
            if (pend.on) store_pending(q8, qe);
            uint8_t *buf = stw + (st_round & 1) * ST_BYTES;
            ++st_round;
            if (lane == 0) tma_store_wait_read<1>();  // the store that last used `buf` has read it
            __syncwarp();
            // Matrix mi of a stmatrix covers channels 8k.. and cells 16hf + 8e..; thread 8mi + j
            // addresses stored row j = channel 8k + j, whose 8 cells sit in 16-byte chunk 2hf + e
            // (64-byte swizzle: chunk ^ ((channel >> 1) & 3)).
            const int mi = lane >> 3, j = lane & 7;
#pragma unroll
            for (int hf = 0; hf < 2; ++hf)
#pragma unroll
                for (int kp = 0; kp < 4; kp += 2) {
                    const int k = kp + (mi >> 1), e = mi & 1;
                    const int ch = 8 * k + j, chunk = 2 * hf + e;
                    const uint32_t addr = smem_u32(buf) + (uint32_t)(ch * 64 + ((chunk ^ ((ch >> 1) & 3)) << 4));
                    stmatrix_x4_trans(addr, P[hf * 8 + kp * 2 + 0], P[hf * 8 + kp * 2 + 1], P[hf * 8 + kp * 2 + 2],
                                      P[hf * 8 + kp * 2 + 3]);
                }
            pend.buf = buf;
            pend.which = which;
            pend.ch0 = ch0;
            pend.ox = ox;
            pend.orow = orow;
            pend.sfo = sfo;
            pend.on = true;
        };

        // hm = mask / 2 for the four cells this thread gates in tile lt: 32q + 16hf + 8e + lane/4,
        // from the mask that landed with the tile (zero past N). The first cell of the
        // warp's run of 32 along its row (PRO_MX_COLS: along its column) is `first`.
        auto read_hm = [&](int lt, int first, float (&hm)[4]) {
            const uint16_t *mrow = reinterpret_cast<const uint16_t *>(msm + (lt % MASK_SLOTS) * MASK_BYTES);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int jc = 32 * q + 16 * (c >> 1) + 8 * (c & 1) + (lane >> 2);
                if (args.has_mask)
                    hm[c] = 0.5f * bf16_bits_to_float(mrow[jc]);
                else
                    hm[c] = first + (jc - 32 * q) < args.N ? 0.5f : 0.f;
            }
        };

        // Halve W_ag and W_bg in place (exact in bf16): the MMAs then yield g / 2 for the tanh.
        bool ok = warp_wait(wbar, 0, abort_flag, ctl, SITE_PRO | 11, 0);
        if (ok && kVec) {
            // Fold the input LayerNorm's affine into the projections, once per CTA:
            // W'[n][k] = W[n][k] gamma[k] (bf16, in place; the gate rows also halved) and
            // b'[n] = b[n] + sum_k W[n][k] beta[k] (halved for the gate rows) into pbias.
            // Thread T owns stacked rows T and T + 256 (weight w = row / 128); it visits the 16
            // chunks of a row starting at chunk (lane + j) & 7, so the lanes of a quarter
            // warp touch different banks.
#pragma unroll 1
            for (int rr = 0; rr < 2; ++rr) {
                const int R = warp * 32 + lane + 256 * rr, w = R >> 7, n = R & 127;
                const float gscale = (w & 1) ? 0.5f : 1.f;
                float acc = 0.f;
#pragma unroll 1
                for (int kh = 0; kh < 2; ++kh) {
                    uint8_t *rowp = wsm + kh * W_HALF + w * 128 * 128 + n * 128;
#pragma unroll 1
                    for (int j = 0; j < 8; ++j) {
                        const int pch = (j + lane) & 7, k0 = kh * 64 + 8 * (pch ^ (n & 7));
                        uint4 *w4 = reinterpret_cast<uint4 *>(rowp + pch * 16);
                        uint4 u = *w4;
                        uint32_t *pw = reinterpret_cast<uint32_t *>(&u);
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float2 wv = unpack_bf16x2(pw[e]);
                            const int k = k0 + 2 * e;
                            const float2 gm = args.ln_w ? ld_pair_bf16(args.ln_w, k) : make_float2(1.f, 1.f);
                            const float2 bt = args.ln_b ? ld_pair_bf16(args.ln_b, k) : make_float2(0.f, 0.f);
                            acc = fmaf(wv.x, bt.x, fmaf(wv.y, bt.y, acc));
                            pw[e] = pack_bf16x2(wv.x * gm.x * gscale, wv.y * gm.y * gscale);
                        }
                        *w4 = u;
                    }
                }
                const __nv_bfloat16 *bsrc = w == 0 ? args.b_a : w == 1 ? args.b_ag : w == 2 ? args.b_b : args.b_bg;
                const float bb = (bsrc ? __bfloat162float(bsrc[n]) : 0.f) + acc;
                pbias[R] = __float2bfloat16_rn(bb * gscale);
            }
            fence_proxy_async_smem();  // read by the tensor core
        } else if (ok) {
#pragma unroll 1
            for (int k = warp * 32 + lane; k < 4 * 1024; k += WORKERS * 32) {  // 4 regions x 1024 uint4
                const int region = k >> 10;  // (K half, weight) = (0, ag), (0, bg), (1, ag), (1, bg)
                uint4 *w4 = reinterpret_cast<uint4 *>(wsm + (region >> 1) * W_HALF + (1 + 2 * (region & 1)) * 128 * 128) +
                            (k & 1023);
                uint4 u = *w4;
                const __nv_bfloat162 h = __float2bfloat162_rn(0.5f);
                uint32_t *pw = reinterpret_cast<uint32_t *>(&u);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    __nv_bfloat162 x = *reinterpret_cast<__nv_bfloat162 *>(&pw[e]);
                    x = __hmul2(x, h);
                    pw[e] = *reinterpret_cast<uint32_t *>(&x);
                }
                *w4 = u;
            }
            fence_proxy_async_smem();  // read by the tensor core
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(wprep);
        // Every worker's b' (kVec) is written before its arrival; the gating reads all of it.
        if (kVec) ok = ok && warp_wait(wprep, 0, abort_flag, ctl, SITE_PRO | 14, 0);
        for (int lt = 0; ok && lt < n_local; ++lt) {
            int i, j0;
            tile_coords(lt, i, j0);
            // The warp's 32 cells go to (x = ox .. ox+31, row orow) of the outputs; they
            // start inside the layer when `live`.
            const int ox = kMode == PRO_MX_COLS ? i : j0 + 32 * q;
            const int orow = kMode == PRO_MX_COLS ? j0 + q : i;
            const bool live = (kMode == PRO_MX_COLS ? orow : ox) < args.N;
            uint32_t sfo[2] = {0, 0};
            if (kMode != PRO_BF16 && live) {
#pragma unroll
                for (int o = 0; o < 2; ++o)
                    sfo[o] = (uint32_t)mx_scale_offset(0, orow, ox >> 5, args.sf_rows[o], args.sf_row_tiles[o],
                                                       args.kchunks, args.sf_chunks[o]);
            }
            if (!live) flush();
            // a-half of tile lt
            if (!(ok = warp_wait(mma_a, (uint32_t)lt & 1u, abort_flag, ctl, SITE_PRO | 7, lt))) break;
            tc_fence_after();
            float hm[4];  // tile lt landed (its a-half MMAs ran after it was normalised)
            read_hm(lt, ox, hm);
            if (live) {
                slab(0, 0, hm, ox, orow, sfo[0], nullptr);
                slab(0, 1, hm, ox, orow, sfo[0], a_free);
            } else {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(a_free);
            }
            // b-half of tile lt
            if (!(ok = warp_wait(mma_b, (uint32_t)lt & 1u, abort_flag, ctl, SITE_PRO | 9, lt))) break;
            tc_fence_after();
            if (live) {
                slab(1, 0, hm, ox, orow, sfo[1], nullptr);
                slab(1, 1, hm, ox, orow, sfo[1], b_free);
            } else {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(b_free);
            }
        }
        if (ok) flush();
        if (!ok && lane == 0) *abort_flag = 1;
        if (lane == 0) tma_store_wait_all<0>();
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == CTRL_WARP) tmem_dealloc(tmem_base, 512);
}

size_t prologue_tc_smem() { return pro::SMEM; }

template <bool kVec, int kMode>
static cudaError_t set_smem() {
    return cudaFuncSetAttribute(prologue_tc_kernel<kVec, kMode>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)pro::SMEM);
}

cudaError_t prologue_tc_setup() {
    cudaError_t e;
    if ((e = set_smem<false, PRO_BF16>()) != cudaSuccess || (e = set_smem<true, PRO_BF16>()) != cudaSuccess ||
        (e = set_smem<false, PRO_MX_ROWS>()) != cudaSuccess || (e = set_smem<true, PRO_MX_ROWS>()) != cudaSuccess ||
        (e = set_smem<false, PRO_MX_COLS>()) != cudaSuccess || (e = set_smem<true, PRO_MX_COLS>()) != cudaSuccess)
        return e;
    return cudaSuccess;
}

template <bool kVec, int kMode>
static cudaError_t launch_as(const PrologueMaps &m, const PrologueArgs &a, int grid, cudaStream_t s) {
    prologue_tc_kernel<kVec, kMode><<<grid, pro::THREADS, pro::SMEM, s>>>(m.w[0], m.w[1], m.w[2], m.w[3], m.z,
                                                                          m.mask, m.a, m.b, a);
    return cudaGetLastError();
}

cudaError_t launch_prologue_tc(const PrologueMaps &m, const PrologueArgs &a, int mode, int grid, cudaStream_t s) {
    const bool vec = a.ln_w || a.ln_b || a.b_a || a.b_ag || a.b_b || a.b_bg;
    switch (mode) {
        case PRO_BF16: return vec ? launch_as<true, PRO_BF16>(m, a, grid, s) : launch_as<false, PRO_BF16>(m, a, grid, s);
        case PRO_MX_ROWS:
            return vec ? launch_as<true, PRO_MX_ROWS>(m, a, grid, s) : launch_as<false, PRO_MX_ROWS>(m, a, grid, s);
        case PRO_MX_COLS:
            return vec ? launch_as<true, PRO_MX_COLS>(m, a, grid, s) : launch_as<false, PRO_MX_COLS>(m, a, grid, s);
        default: return cudaErrorInvalidValue;
    }
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

// 32 x 32 tiles through shared memory: reads along mask rows, writes along dst rows.
__global__ void mask_transpose_kernel(const __nv_bfloat16 *__restrict__ mask, __nv_bfloat16 *__restrict__ dst, int N,
                                      int ld) {
    __shared__ __nv_bfloat16 t[32][33];
    const int k0 = blockIdx.x * 32, i0 = blockIdx.y * 32;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 256 threads: 8 rows per pass
    for (int r = ty; r < 32; r += 8) {
        const int k = k0 + r, i = i0 + tx;
        t[r][tx] = (k < N && i < N) ? mask[(size_t)k * N + i] : __float2bfloat16(0.f);
    }
    __syncthreads();
    for (int r = ty; r < 32; r += 8) {
        const int i = i0 + r, k = k0 + tx;
        if (i < N && k < ld) dst[(size_t)i * ld + k] = t[tx][r];
    }
}

cudaError_t launch_mask_transpose(const __nv_bfloat16 *mask, __nv_bfloat16 *dst, int N, int ld, cudaStream_t s) {
    mask_transpose_kernel<<<dim3((ld + 31) / 32, (N + 31) / 32), 256, 0, s>>>(mask, dst, N, ld);
    return cudaGetLastError();
}

}  // namespace trimul

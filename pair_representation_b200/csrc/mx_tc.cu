// mx_tc.cu - the triangle contraction in MXFP8 on tcgen05 block-scaled MMAs.
//
// The pages list MXFP8 among the Blackwell training precisions of the BioNeMo
// recipes ("Scaling biomolecular modeling with context parallelism in NVIDIA
// BioNeMo", the precision list); the format is the OCP Microscaling (MX) v1.0
// one: blocks of 32 values along the contracted index k share an E8M0 scale
// X = 2^e with e = floor(log2 max|v|) - 8, and each value is stored as E4M3
// (round to nearest even, saturated at +-448). For the triangle contraction
// X_c[m][n] = sum_k A_c(m, k) B_c(n, k) the blocks run along k: along a row
// of a and b for the outgoing product, down a column for the incoming one.
//
// Two kernels:
//   mx_quant_kernel  reads a or b (bf16, channel-major [128][N][ld]) and writes
//     the E4M3 elements K-major, Q[c][m][k] (row m, k contiguous, pitch ldq),
//     transposing on the way for the incoming direction, and the scales in the
//     order the contraction copies them into tensor memory (below).
//   contract_mx_kernel  CTA pairs share a 256 x 192 output tile through
//     tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale (M = 256, N = 192,
//     K = 32 per instruction); K blocks of 128 (one 128-byte row per operand
//     row) in a 6-stage TMA ring; per stage the MMA thread copies the stage's
//     scales from shared into tensor memory (tcgen05.cp) and issues 4 MMAs,
//     the i-th reading byte i of every scale word (the scale-factor ids of the
//     instruction descriptor). Accumulators: 2 x 192 columns of fp32,
//     double-buffered; scales: 12 columns per stage after them.
//
// Scale layout in tensor memory (per MMA, 4 K blocks per 32-bit word): the
// scale of operand row r and K block kb sits in lane r % 32 (repeated in all
// four lane quadrants by the .warpx4 copy), column r / 32, byte kb % 4. A is
// scaled per CTA (its 128 rows: 4 columns); each CTA of a pair holds the scales
// of all N = 192 rows of B (two 128-row chunks: 8 columns). In memory one
// 128-row x 4-block chunk is 512 bytes: row r, block b at
// (r % 32) * 16 + (r / 32) * 4 + b, so that the 32 x 128-bit copy puts lane
// r % 32's 16 bytes in columns 0..3. The quantizer writes each operand's scales
// per row tile of the contraction (A: 128 rows, one chunk; B: 192 rows, two
// chunks of which the second is half used) and per 128-wide K chunk, so one
// TMA box brings a stage's scales.
#include "kernels.h"
#include "mx_block.cuh"

namespace trimul {

// ---------------------------------------------------------------------------
// Quantizer
// ---------------------------------------------------------------------------

// One thread per block of 32 values: 64 rows x 4 blocks (one 128-wide K chunk)
// of one channel per CTA. Rows >= N and columns >= N are zeros (scale byte 0);
// every scale slot of the padded row tiles is written.
template <bool kTransposed>
__global__ void __launch_bounds__(256) mx_quant_kernel(MxQuantArgs p) {
    __shared__ __align__(16) __nv_bfloat16 tile[kTransposed ? 128 * 72 : 1];  // [128 k][64 m + 8 pad]
    const int c = blockIdx.z;
    const int m0 = blockIdx.y * 64, k0 = blockIdx.x * 128;
    const __nv_bfloat16 *src = p.src + (size_t)c * p.N * p.ld;
    int ml, b;
    if (kTransposed) {
        // Source element (m, k) is src[k][m]: stage the 128 x 64 tile through shared memory.
        for (int e = threadIdx.x; e < 128 * 8; e += 256) {
            const int kr = e >> 3, ch = e & 7;  // row k0 + kr, 16-byte chunk ch (8 values of m)
            const int k = k0 + kr, m = m0 + ch * 8;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (k < p.N && m < p.N) v = *reinterpret_cast<const uint4 *>(src + (size_t)k * p.ld + m);
            *reinterpret_cast<uint4 *>(&tile[kr * 72 + ch * 8]) = v;
        }
        __syncthreads();
        ml = threadIdx.x & 63;
        b = threadIdx.x >> 6;
    } else {
        ml = threadIdx.x >> 2;
        b = threadIdx.x & 3;
    }
    const int m = m0 + ml, kb0 = k0 + 32 * b;
    float v[32];
    if (kTransposed) {
#pragma unroll
        for (int t = 0; t < 32; ++t) v[t] = m < p.N ? __bfloat162float(tile[(32 * b + t) * 72 + ml]) : 0.f;
        // Rows k >= N were loaded as zeros; columns m >= N (row padding) are excluded above.
    } else {
        const __nv_bfloat16 *row = src + (size_t)m * p.ld;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            uint4 u = make_uint4(0u, 0u, 0u, 0u);
            const int k = kb0 + 8 * q;
            if (m < p.N && k < p.N) u = *reinterpret_cast<const uint4 *>(row + k);  // ld is a multiple of 8
            const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                v[8 * q + 2 * e] = __uint_as_float(w[e] << 16);
                v[8 * q + 2 * e + 1] = __uint_as_float(w[e] & 0xFFFF0000u);
            }
        }
        // Within a row, ld >= N: values at k >= N inside the last 8-chunk are padding.
#pragma unroll
        for (int t = 0; t < 32; ++t)
            if (kb0 + t >= p.N) v[t] = 0.f;
    }
    uint32_t q8[8];
    const int e = mx_quantize32(v, q8);
    if (m < p.N) {
        if (kb0 < p.ldq) {
            uint8_t *dst = p.q + ((size_t)c * p.N + m) * p.ldq + kb0;  // ldq is a multiple of 16
            *reinterpret_cast<uint4 *>(dst) = make_uint4(q8[0], q8[1], q8[2], q8[3]);
            if (kb0 + 16 < p.ldq) *reinterpret_cast<uint4 *>(dst + 16) = make_uint4(q8[4], q8[5], q8[6], q8[7]);
        }
    }
    if (m < p.row_tiles * p.rows_per_tile)
        p.sf[mx_scale_offset(c, m, kb0 >> 5, p.rows_per_tile, p.row_tiles, p.kchunks, p.chunks_per_tile)] =
            (uint8_t)(e + 127);
}

cudaError_t launch_mx_quant(const MxQuantArgs &a, int transposed, cudaStream_t s) {
    const int mrows = a.row_tiles * a.rows_per_tile;
    dim3 grid(a.kchunks, (mrows + 63) / 64, 128);
    if (transposed)
        mx_quant_kernel<true><<<grid, 256, 0, s>>>(a);
    else
        mx_quant_kernel<false><<<grid, 256, 0, s>>>(a);
    return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Block-scaled contraction
// ---------------------------------------------------------------------------
namespace cmx {
constexpr int BM = 256, BN = 192, BK = 128, STAGES = 6;
constexpr int HALF_M = 128, HALF_N = 96;
constexpr int A_BYTES = HALF_M * BK;            // 16 KB
constexpr int B_BYTES = HALF_N * BK;            // 12 KB
constexpr int SFA_BYTES = 512;                  // 128 rows x 4 blocks
constexpr int SFB_BYTES = 1024;                 // 2 x 128 rows x 4 blocks
constexpr int STAGE_TX = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
constexpr int OUT_COLS = 64;
constexpr int WBUF_BYTES = 32 * 128;            // 4 KB: a drain warp's 32 rows x 64 bf16
constexpr int OUT_BYTES = 4 * WBUF_BYTES;       // 16 KB: one such buffer per drain warp
constexpr int THREADS = 192;
constexpr int TMEM_COLS = 512;
constexpr uint32_t COL_SF = 2 * BN;             // 384: scales of stage s at 384 + 12 s
constexpr int BAR_BYTES = 256;
constexpr size_t SMEM = 1024 + (size_t)STAGES * (A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES) + 2 * OUT_BYTES +
                        BAR_BYTES;
static_assert(SMEM <= 232448, "shared memory budget");
static_assert(COL_SF + 12 * STAGES <= TMEM_COLS, "tensor memory budget");
}  // namespace cmx

// Instruction descriptor of kind::mxf8f6f4.block_scale: E4M3 A and B (K-major),
// fp32 D, E8M0 scales, scale byte `sf` of A's and B's scale words, K = 32.
__host__ __device__ constexpr uint32_t idesc_mxf8(int M, int N, uint32_t sf) {
    return (sf << 4)                              // B scale factor id
           | (0u << 7) | (0u << 10)               // A, B format: E4M3
           | ((uint32_t)(N >> 3) << 17)           // N / 8
           | (1u << 23)                           // scale format: E8M0
           | ((uint32_t)(M >> 4) << 24)           // M / 16
           | (sf << 29);                          // A scale factor id
}

// Shared-memory descriptor of 32 rows x 16 bytes, rows 16 bytes apart (no
// swizzle): the source of a 32x128b tensor-memory copy.
__device__ __forceinline__ uint64_t sdesc_rows16(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)(128u >> 4) << 32;  // 8-row groups 128 bytes apart
    d |= (uint64_t)1u << 46;           // descriptor version for sm_100
    return d;
}

__device__ __forceinline__ void tmem_cp_32x128_pair(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

__device__ __forceinline__ void mma_mxf8_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                              uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %6, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%4], [%5], p;\n\t}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa_tmem), "r"(sfb_tmem), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void tma_load_2d_pair(void *dst, const CUtensorMap *map, uint32_t bar_cluster, int c0,
                                                 int c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(map), "r"(bar_cluster), "r"(c0), "r"(c1)
        : "memory");
}

// Same protocol as contract_tc_kernel (full / empty / tfull / tempty, abort
// and drain), with fp8 operands, scale boxes and a 192-wide tile.
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(cmx::THREADS, 1)
    contract_mx_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                       const __grid_constant__ CUtensorMap tmSA, const __grid_constant__ CUtensorMap tmSB,
                       const __grid_constant__ CUtensorMap tmX, const ContractMxArgs args) {
    using namespace cmx;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *sA = smem;                                 // [STAGES][16 KB]
    uint8_t *sB = sA + STAGES * A_BYTES;                // [STAGES][12 KB]
    uint8_t *sSA = sB + STAGES * B_BYTES;               // [STAGES][512]
    uint8_t *sSB = sSA + STAGES * SFA_BYTES;            // [STAGES][1024]
    uint8_t *outbuf = sSB + STAGES * SFB_BYTES;         // [2][16 KB]
    uint64_t *bars = reinterpret_cast<uint64_t *>(outbuf + 2 * OUT_BYTES);
    uint64_t *full = bars;
    uint64_t *empty = bars + STAGES;
    uint64_t *tfull = bars + 2 * STAGES;
    uint64_t *tempty = tfull + 2;
    uint64_t *drain = tempty + 2;
    uint64_t *peer_done = drain + 1;
    uint32_t *peer_phases = reinterpret_cast<uint32_t *>(peer_done + 1);
    uint32_t *tmem_slot = peer_phases + STAGES;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const int pair = (int)blockIdx.x >> 1, npairs = (int)gridDim.x >> 1;
    const KernelCtl &ctl = args.ctl;
    const int tiles_per_c = args.ti_tiles * args.tj_tiles;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            peer_phases[s] = 0;
        }
        mbar_init(peer_done, 1);
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 8);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        tma_prefetch_desc(&tmSA);
        tma_prefetch_desc(&tmSB);
        tma_prefetch_desc(&tmX);
    }
    if (warp == 1) {
        __syncwarp();
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    __syncwarp();
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const uint32_t peer_abort = map_to_rank((const void *)abort_flag, rank ^ 1u);
    auto raise_abort = [&]() {
        *abort_flag = 1;
        st_remote_u32(peer_abort, 1u);
    };

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer (both CTAs) ----------------
            const uint32_t full0 = map_to_rank(full, 0);
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued = 0;
            auto phases_of = [&](int s) -> uint32_t {
                return issued / STAGES + ((uint32_t)s < issued % STAGES ? 1u : 0u);
            };
            bool ok = true;
            for (int tile = pair; ok && tile < args.total_tiles; tile += npairs) {
                const int c = tile / tiles_per_c;
                const int r = tile - c * tiles_per_c;
                const int ti = r / args.tj_tiles, tj = r - ti * args.tj_tiles;
                const int i0 = ti * BM + (int)rank * HALF_M;
                const int j0 = tj * BN + (int)rank * HALF_N;
                const int sa_row0 = ((c * args.a_row_tiles + 2 * ti + (int)rank) * args.kchunks) * 32;
                const int sb_row0 = ((c * args.b_row_tiles + tj) * args.kchunks) * 64;
                for (int kb = 0; kb < args.kchunks; ++kb) {
                    if (!wait_bounded(&empty[stage], phase ^ 1u, abort_flag, ctl, SITE_CON | 1, tile)) {
                        ok = false;
                        break;
                    }
                    const uint32_t bar = full0 + (uint32_t)(stage * 8);
                    if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * STAGE_TX);
                    const int k0 = kb * BK;
                    tma_load_3d_pair(sA + stage * A_BYTES, &tmA, bar, k0, i0, c);
                    tma_load_3d_pair(sB + stage * B_BYTES, &tmB, bar, k0, j0, c);
                    tma_load_2d_pair(sSA + stage * SFA_BYTES, &tmSA, bar, 0, sa_row0 + kb * 32);
                    tma_load_2d_pair(sSB + stage * SFB_BYTES, &tmSB, bar, 0, sb_row0 + kb * 64);
                    ++issued;
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) raise_abort();
            if (rank == 1) {
#pragma unroll
                for (int s = 0; s < STAGES; ++s) st_remote_u32(map_to_rank(&peer_phases[s], 0), phases_of(s));
                fence_acq_rel_cluster();
                mbar_arrive_remote(map_to_rank(peer_done, 0));
            } else {
                const bool peer_ok = wait_drain(peer_done, 0, ctl.timeout_ns);
                fence_acq_rel_cluster();
#pragma unroll
                for (int s = 0; s < STAGES; ++s) {
                    const uint32_t n0 = phases_of(s);
                    const uint32_t n1 = peer_ok ? peer_phases[s] : n0;
                    if (n1 > n0) mbar_arrive_expect_tx(&full[s], STAGE_TX);
                    if (n0 > n1) mbar_complete_tx(&full[s], STAGE_TX);
                    const uint32_t n = n0 > n1 ? n0 : n1;
                    if (n > 0) wait_drain(&full[s], (n - 1) & 1u, ctl.timeout_ns);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            // ---------------- MMA issuer (CTA 0) ----------------
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            int lt = 0;
            for (int tile = pair; ok && tile < args.total_tiles; tile += npairs, ++lt) {
                const int acc = lt & 1;
                const uint32_t acc_par = (uint32_t)(lt >> 1) & 1u;
                if (!wait_bounded(&tempty[acc], acc_par ^ 1u, abort_flag, ctl, SITE_CON | 2, tile)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem_base + (uint32_t)(acc * BN);
                for (int kb = 0; kb < args.kchunks; ++kb) {
                    if (!wait_bounded(&full[stage], phase, abort_flag, ctl, SITE_CON | 3, tile)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    // The stage's scales into tensor memory (both CTAs, same offsets), then 4 MMAs.
                    const uint32_t tsa = tmem_base + COL_SF + (uint32_t)(12 * stage), tsb = tsa + 4;
                    tmem_cp_32x128_pair(tsa, sdesc_rows16(smem_u32(sSA + stage * SFA_BYTES)));
                    tmem_cp_32x128_pair(tsb, sdesc_rows16(smem_u32(sSB + stage * SFB_BYTES)));
                    tmem_cp_32x128_pair(tsb + 4, sdesc_rows16(smem_u32(sSB + stage * SFB_BYTES + 512)));
                    const uint32_t sa = smem_u32(sA + stage * A_BYTES), sb = smem_u32(sB + stage * B_BYTES);
#pragma unroll
                    for (int kk = 0; kk < BK / 32; ++kk) {
                        mma_mxf8_pair(d, sdesc_sw128(sa + kk * 32, 16, 1024), sdesc_sw128(sb + kk * 32, 16, 1024),
                                      idesc_mxf8(BM, BN, (uint32_t)kk), tsa, tsb, (kb | kk) != 0 ? 1u : 0u);
                    }
                    mma_commit_pair(&empty[stage]);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                mma_commit_pair(&tfull[acc]);
            }
            if (!ok) raise_abort();
            mma_commit_local2(drain);
            wait_drain(drain, 0, ctl.timeout_ns);
        }
    } else {
        // ---------------- epilogue warps 2..5 (both CTAs) ----------------
        // Warp q drains TMEM lanes 32q .. 32q + 31 (accumulator rows r0 ..) and stores them
        // itself: per chunk a [32 rows][128 bytes] block through its own two 4 KB buffers and
        // its own TMA store, so the four warps never wait on one another.
        const int q = warp & 3;
        const uint32_t tempty0 = map_to_rank(&tempty[0], 0);
        const uint32_t tempty1 = map_to_rank(&tempty[1], 0);
        uint8_t *wbuf = outbuf + q * 2 * WBUF_BYTES;
        // Stores issued so far by this warp, over all its tiles: store n stages through
        // buffer n & 1, and before it is written the store that last used that buffer
        // (n - 2) must have read it, which wait_group.read 1 ensures only because the
        // count runs on across tiles. A count restarted per tile would, after a tile with
        // an odd number of stores (one in the ragged last column of tiles), give the next
        // tile's first chunk the buffer that the still-pending last store is reading.
        int nst = 0;
        int lt = 0;
        for (int tile = pair; tile < args.total_tiles; tile += npairs, ++lt) {
            const int c = tile / tiles_per_c;
            const int r = tile - c * tiles_per_c;
            const int ti = r / args.tj_tiles, tj = r - ti * args.tj_tiles;
            // Accumulator rows: the A rows this CTA loaded; columns [0, 96) from CTA 0's B
            // rows and [96, 192) from CTA 1's, i.e. tile columns j0 .. j0 + 191 in order.
            const int r0 = ti * BM + (int)rank * HALF_M + 32 * q;
            const int j0 = tj * BN;
            const int acc = lt & 1;
            const uint32_t acc_par = (uint32_t)(lt >> 1) & 1u;
            if (!warp_wait(&tfull[acc], acc_par, abort_flag, ctl, SITE_CON | 4, tile)) {
                if (lane == 0) raise_abort();
                break;
            }
            tc_fence_after();
            // Chunks whose first column is past the matrix, and rows past it, are neither
            // read nor stored.
#pragma unroll 1
            for (int ch = 0; ch < BN / OUT_COLS; ++ch) {
                const int jst = j0 + ch * OUT_COLS;
                if (r0 >= args.N || jst >= args.N) continue;
                uint32_t p[32];  // the 128-byte row of this thread's accumulator row
                const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN + ch * OUT_COLS);
                uint32_t v[64];
                tmem_ld32(taddr, v);
                tmem_ld32(taddr + 32, v + 32);
                tmem_ld_wait();
#pragma unroll
                for (int k = 0; k < 32; ++k)
                    p[k] = pack_bf16x2(__uint_as_float(v[2 * k]), __uint_as_float(v[2 * k + 1]));
                uint8_t *ob = wbuf + (nst & 1) * WBUF_BYTES;
                ++nst;
                if (lane == 0) tma_store_wait_read<1>();
                __syncwarp();
#pragma unroll
                for (int c16 = 0; c16 < 8; ++c16) {
                    uint4 val = make_uint4(p[4 * c16], p[4 * c16 + 1], p[4 * c16 + 2], p[4 * c16 + 3]);
                    *reinterpret_cast<uint4 *>(ob + lane * 128 + ((c16 ^ (lane & 7)) << 4)) = val;
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_3d(&tmX, ob, jst, r0, c);
                    tma_store_commit();
                }
            }
            // Every TMEM read of this accumulator is complete: hand it back to the MMA.
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_remote(acc ? tempty1 : tempty0);
        }
        if (lane == 0) tma_store_wait_all<0>();
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();
    tc_fence_after();
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS)
                     : "memory");
}

cudaError_t contract_mx_setup() {
    return cudaFuncSetAttribute(contract_mx_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)cmx::SMEM);
}

cudaError_t launch_contract_mx(const ContractMxMaps &m, const ContractMxArgs &a, int grid, cudaStream_t s) {
    contract_mx_kernel<<<grid, cmx::THREADS, cmx::SMEM, s>>>(m.a, m.b, m.sa, m.sb, m.x, a);
    return cudaGetLastError();
}

}  // namespace trimul

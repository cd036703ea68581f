// contract_tc.cu - the triangle contraction on tcgen05 tensor cores, CTA pairs.
//
// For every channel c of the hidden pair features (outgoing X_c = A_c B_c^T,
// incoming X_c = A_c^T B_c; TriangleMultiplicationOutgoing, "Scaling
// biomolecular modeling with context parallelism in NVIDIA BioNeMo", section
// "Context-parallel implementation of triangle multiplication"), computed by
// pairs of CTAs on neighbouring SMs (a cluster of 2) that share one
// 256 x 256 output tile through tcgen05.mma.cta_group::2. In general form
// X[m][n] = sum_k A(m, k) B(n, k), each operand stored K-major ([rows][k]) or
// MN-major ([k][rows]) as ContractArgs says: both K-major is the outgoing
// product, both MN-major the incoming one, and the mixed forms serve the
// backward's adjoint products.
//   * CTA r of the pair loads rows [128 r, 128 r + 128) of the tile's A panel
//     and rows [128 r, 128 r + 128) of its B panel (its half of N) into its own
//     shared memory, 16 KB + 16 KB per 64-deep K block, 6 stages;
//   * one thread of CTA 0 issues M = 256, N = 256 MMAs that read both CTAs'
//     operands; CTA r's tensor memory receives rows [128 r, 128 r + 128) of
//     the fp32 accumulator (double-buffered, 2 x 256 columns);
//   * each CTA's epilogue warps drain their own half and TMA-store it.
// Per SM this moves 32 KB of operands per K block for the same MMA work that
// a single CTA with a 128 x 256 tile needs 48 KB for.
//
// The same kernel serves as the batched GEMM of the backward: M, N and K are
// separate (ContractArgs), the batch runs where the channel does, and
// kF32Out stores the accumulator as fp32 (32-column chunks) instead of bf16.
//
// Synchronisation (every wait bounded):
//   full[s]    CTA 0: armed by CTA 0's producer for the pair's 64 KB; CTA 0's
//              loads and CTA 1's loads (cta_group::2 TMA addressed to CTA 0's
//              barrier) both complete bytes on it; the MMA issuer waits on it
//   empty[s]   both CTAs, arrived by the MMA commit multicast to the pair
//   tfull[a]   both CTAs, MMA commit multicast -> epilogue warps
//   tempty[a]  CTA 0, arrivals of the 4 + 4 epilogue warps of both CTAs
// On the way out CTA 1 publishes how many phases of each stage it loaded and
// CTA 0 reconciles full[s] (arming phases only CTA 1 loaded, completing the
// bytes of phases only CTA 0 loaded), then waits for every stage to land, so
// no copy is in flight when the pair passes its final cluster barrier.
#include "kernels.h"

namespace trimul {
namespace con {
constexpr int BN = 256, BK = 64, STAGES = 6;
constexpr int HALF = 128;                         // rows per CTA of A and of B
constexpr int A_BYTES = HALF * BK * 2;            // 16 KB
constexpr int B_BYTES = HALF * BK * 2;            // 16 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;    // 32 KB
constexpr int WBUF_BYTES = 32 * 128;             // 4 KB: a drain warp's 32 rows x 128 bytes (64 bf16 or 32 fp32)
constexpr int OUT_BYTES = 4 * WBUF_BYTES;         // 16 KB: one such buffer per drain warp
constexpr int NUM_OUT = 2;
constexpr int TMEM_COLS = 512;
constexpr int THREADS = 192;
constexpr int BAR_BYTES = 256;
constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE_BYTES + NUM_OUT * OUT_BYTES + BAR_BYTES;
static_assert(SMEM <= 232448, "shared memory budget");
}  // namespace con

template <bool kF32Out>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(con::THREADS, 1)
    contract_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmX, const ContractArgs args) {
    using namespace con;
    constexpr int OUT_COLS = kF32Out ? 32 : 64;  // accumulator columns per stored chunk
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *stages = smem;
    uint8_t *outbuf = smem + STAGES * STAGE_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(outbuf + NUM_OUT * OUT_BYTES);
    uint64_t *full = bars;                 // [STAGES] (CTA 0) operands of both CTAs landed
    uint64_t *empty = bars + STAGES;       // [STAGES] MMA done reading the stage (both CTAs)
    uint64_t *tfull = bars + 2 * STAGES;   // [2]
    uint64_t *tempty = tfull + 2;          // [2] (CTA 0)
    uint64_t *dead = tempty + 2;           // never signalled (failure-path test)
    uint64_t *drain = dead + 1;
    uint64_t *peer_done = drain + 1;       // (CTA 0) CTA 1's producer has published its phase counts
    uint32_t *peer_phases = reinterpret_cast<uint32_t *>(peer_done + 1);  // [STAGES] (CTA 0) written by CTA 1
    uint32_t *tmem_slot = peer_phases + STAGES;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const int pair = (int)blockIdx.x >> 1, npairs = (int)gridDim.x >> 1;
    const KernelCtl &ctl = args.ctl;
    const int tiles_per_c = args.ti_tiles * args.tj_tiles;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);  // CTA 0's producer arms it (arrive + expect_tx)
            mbar_init(&empty[s], 1);
            peer_phases[s] = 0;
        }
        mbar_init(peer_done, 1);
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 8);  // 4 epilogue warps in each CTA
        }
        mbar_init(dead, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
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
    cluster_sync();  // barriers of both CTAs initialised, TMEM allocated in both
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    const uint32_t peer_abort = map_to_rank((const void *)abort_flag, rank ^ 1u);
    // Raise the abort in this CTA and in its peer.
    auto raise_abort = [&]() {
        *abort_flag = 1;
        st_remote_u32(peer_abort, 1u);
    };

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer (both CTAs) ----------------
            const uint32_t full0 = map_to_rank(full, 0);  // CTA 0's full[0] in the cluster window
            int stage = 0;
            uint32_t phase = 0;
            uint32_t issued = 0;  // K blocks this CTA has loaded; stages are used round-robin
            auto phases_of = [&](int s) -> uint32_t {
                return issued / STAGES + ((uint32_t)s < issued % STAGES ? 1u : 0u);
            };
            bool ok = true;
            for (int tile = pair; ok && tile < args.total_tiles; tile += npairs) {
                const int c = tile / tiles_per_c;
                const int r = tile - c * tiles_per_c;
                const int ti = r / args.tj_tiles, tj = r - ti * args.tj_tiles;
                const int i0 = ti * 256 + (int)rank * HALF;
                const int j0 = tj * BN + (int)rank * HALF;
                for (int kb = 0; kb < args.kblocks; ++kb) {
                    if (!wait_bounded(&empty[stage], phase ^ 1u, abort_flag, ctl, SITE_CON | 1, tile)) {
                        ok = false;
                        break;
                    }
                    uint8_t *sa = stages + stage * STAGE_BYTES;
                    uint8_t *sb = sa + A_BYTES;
                    const uint32_t bar = full0 + (uint32_t)(stage * 8);
                    if (rank == 0) mbar_arrive_expect_tx(&full[stage], 2 * STAGE_BYTES);
                    const int k0 = kb * BK;
                    // K-major operand [rows][k]: one box of 64 k x 128 rows. MN-major operand
                    // [k][rows]: two boxes of 64 rows x 64 k.
                    if (!args.a_mn) {
                        tma_load_3d_pair(sa, &tmA, bar, k0, i0, c);
                    } else {
                        tma_load_3d_pair(sa, &tmA, bar, i0, k0, c);
                        tma_load_3d_pair(sa + BK * 128, &tmA, bar, i0 + 64, k0, c);
                    }
                    if (!args.b_mn) {
                        tma_load_3d_pair(sb, &tmB, bar, k0, j0, c);
                    } else {
                        tma_load_3d_pair(sb, &tmB, bar, j0, k0, c);
                        tma_load_3d_pair(sb + BK * 128, &tmB, bar, j0 + 64, k0, c);
                    }
                    ++issued;
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) raise_abort();
            if (rank == 1) {
                // Publish the phase counts to CTA 0, then signal it.
#pragma unroll
                for (int s = 0; s < STAGES; ++s) st_remote_u32(map_to_rank(&peer_phases[s], 0), phases_of(s));
                fence_acq_rel_cluster();
                mbar_arrive_remote(map_to_rank(peer_done, 0));
            } else {
                // Reconcile every stage with CTA 1's loads, then let all of them land.
                const bool peer_ok = wait_drain(peer_done, 0, ctl.timeout_ns);
                fence_acq_rel_cluster();  // CTA 1's counts, released before its arrival, are visible
#pragma unroll
                for (int s = 0; s < STAGES; ++s) {
                    const uint32_t n0 = phases_of(s);
                    const uint32_t n1 = peer_ok ? peer_phases[s] : n0;
                    if (n1 > n0) mbar_arrive_expect_tx(&full[s], STAGE_BYTES);  // a phase only CTA 1 loaded
                    if (n0 > n1) mbar_complete_tx(&full[s], STAGE_BYTES);       // a phase only CTA 0 loaded
                    const uint32_t n = n0 > n1 ? n0 : n1;
                    if (n > 0) wait_drain(&full[s], (n - 1) & 1u, ctl.timeout_ns);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            // ---------------- MMA issuer (CTA 0) ----------------
            const uint32_t idesc = idesc_bf16(256, BN, args.a_mn, args.b_mn);
            const bool stall = (ctl.debug_flags & 0x1u) != 0;
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
                for (int kb = 0; kb < args.kblocks; ++kb) {
                    if (stall && !wait_bounded(dead, 0, abort_flag, ctl, SITE_CON | 7, tile)) {
                        ok = false;
                        break;
                    }
                    if (!wait_bounded(&full[stage], phase, abort_flag, ctl, SITE_CON | 3, tile)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_u32(stages + stage * STAGE_BYTES);
                    const uint32_t sb = sa + A_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk) {
                        const uint64_t ad = args.a_mn ? sdesc_sw128(sa + kk * 2048, BK * 128, 1024)
                                                      : sdesc_sw128(sa + kk * 32, 16, 1024);
                        const uint64_t bd = args.b_mn ? sdesc_sw128(sb + kk * 2048, BK * 128, 1024)
                                                      : sdesc_sw128(sb + kk * 32, 16, 1024);
                        mma_bf16_pair(d, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
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
            // This CTA's accumulator rows are the A rows it loaded; accumulator columns
            // [0,128) come from CTA 0's B rows and [128,256) from CTA 1's, i.e. tile
            // columns j0 .. j0 + 255 in order.
            const int r0 = ti * 256 + (int)rank * HALF + 32 * q;
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
                if (r0 >= args.M || jst >= args.Ncols) continue;
                uint32_t p[32];  // the 128-byte row of this thread's accumulator row
                const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN + ch * OUT_COLS);
                if (kF32Out) {
                    tmem_ld32(taddr, p);
                    tmem_ld_wait();
                } else {
                    uint32_t v[64];
                    tmem_ld32(taddr, v);
                    tmem_ld32(taddr + 32, v + 32);
                    tmem_ld_wait();
#pragma unroll
                    for (int k = 0; k < 32; ++k)
                        p[k] = pack_bf16x2(__uint_as_float(v[2 * k]), __uint_as_float(v[2 * k + 1]));
                }
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
    cluster_sync();  // no CTA leaves while its peer may still touch its shared or tensor memory
    tc_fence_after();
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS)
                     : "memory");
}

size_t contract_tc_smem() { return con::SMEM; }

cudaError_t contract_tc_setup() {
    cudaError_t e = cudaFuncSetAttribute(contract_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)con::SMEM);
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(contract_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)con::SMEM);
}

cudaError_t launch_contract_tc(const ContractMaps &m, const ContractArgs &a, int grid, cudaStream_t s) {
    if (a.out_f32)
        contract_tc_kernel<true><<<grid, con::THREADS, con::SMEM, s>>>(m.a, m.b, m.x, a);
    else
        contract_tc_kernel<false><<<grid, con::THREADS, con::SMEM, s>>>(m.a, m.b, m.x, a);
    return cudaGetLastError();
}

}  // namespace trimul

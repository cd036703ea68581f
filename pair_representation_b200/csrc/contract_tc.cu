// contract_tc.cu - the triangle contraction on tcgen05 tensor cores.
//
// For every channel c of the hidden pair features, outgoing computes
// X_c = A_c B_c^T (x_ij = sum_k a_ik b_jk) and incoming X_c = A_c^T B_c
// (x_ij = sum_k a_ki b_kj): 128 independent N x N x N products, the step the
// layer's name refers to (TriangleMultiplicationOutgoing, "Scaling
// biomolecular modeling with context parallelism in NVIDIA BioNeMo", section
// "Context-parallel implementation of triangle multiplication").
//
// a, b and x are channel-major [128][N][ld] bf16 arrays in the workspace.
// Both directions read the same arrays: outgoing feeds the tensor core
// K-major tiles (k contiguous), incoming feeds the transposed operands as
// MN-major tiles (i or j contiguous) selected by the instruction descriptor,
// so nothing is transposed in memory.
//
// Kernel shape: persistent, one CTA per SM, 128 x 256 output tiles, 64-deep
// K blocks in a 4-stage TMA ring, fp32 accumulators double-buffered in tensor
// memory (2 x 256 columns), and warp roles:
//   warp 0      TMA producer (one thread)
//   warp 1      TMEM allocator and MMA issuer (one thread)
//   warps 2..5  epilogue: TMEM -> registers -> bf16 -> swizzled smem -> TMA store
// Tiles are ordered channel-major so CTAs resident together share one
// channel's panels in L2. Out-of-range rows / k are zero-filled by TMA on load
// and clipped on store, so ragged N needs no masking.
#include "kernels.h"

namespace trimul {
namespace con {
constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;            // 16 KB
constexpr int B_BYTES = BN * BK * 2;            // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;  // 48 KB
constexpr int OUT_COLS = 64;
constexpr int OUT_BYTES = BM * OUT_COLS * 2;    // 16 KB
constexpr int NUM_OUT = 2;
constexpr int TMEM_COLS = 512;
constexpr int THREADS = 192;
constexpr int BAR_BYTES = 256;
constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE_BYTES + NUM_OUT * OUT_BYTES + BAR_BYTES;
static_assert(SMEM <= 232448, "shared memory budget");
}  // namespace con

__global__ void __launch_bounds__(con::THREADS, 1)
    contract_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                       const __grid_constant__ CUtensorMap tmX, const ContractArgs args) {
    using namespace con;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *stages = smem;
    uint8_t *outbuf = smem + STAGES * STAGE_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(outbuf + NUM_OUT * OUT_BYTES);
    uint64_t *full = bars;                 // [STAGES] TMA -> MMA
    uint64_t *empty = bars + STAGES;       // [STAGES] MMA -> TMA
    uint64_t *tfull = bars + 2 * STAGES;   // [2] MMA -> epilogue
    uint64_t *tempty = tfull + 2;          // [2] epilogue -> MMA
    uint64_t *dead = tempty + 2;           // never signalled (failure-path test)
    uint64_t *drain = dead + 1;            // MMA completion before teardown
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    volatile int *epi_go = abort_flag + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const KernelCtl &ctl = args.ctl;
    const int tiles_per_c = args.ti_tiles * args.tj_tiles;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 4);  // one arrival per epilogue warp
        }
        mbar_init(dead, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        *epi_go = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        tma_prefetch_desc(&tmX);
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer ----------------
            int stage = 0;
            uint32_t phase = 0, ever = 0, par = 0;
            bool ok = true;
            for (int tile = blockIdx.x; ok && tile < args.total_tiles; tile += gridDim.x) {
                const int c = tile / tiles_per_c;
                const int r = tile - c * tiles_per_c;
                const int ti = r / args.tj_tiles, tj = r - ti * args.tj_tiles;
                const int i0 = ti * BM, j0 = tj * BN;
                for (int kb = 0; kb < args.kblocks; ++kb) {
                    if (!wait_bounded(&empty[stage], phase ^ 1u, abort_flag, ctl, SITE_CON | 1, tile)) {
                        ok = false;
                        break;
                    }
                    uint8_t *sa = stages + stage * STAGE_BYTES;
                    uint8_t *sb = sa + A_BYTES;
                    mbar_arrive_expect_tx(&full[stage], STAGE_BYTES);
                    const int k0 = kb * BK;
                    if (!args.incoming) {
                        tma_load_3d(sa, &tmA, &full[stage], k0, i0, c);
                        tma_load_3d(sb, &tmB, &full[stage], k0, j0, c);
                    } else {
                        // MN-major: 64-wide row blocks, each BK k-rows of 128 B.
                        tma_load_3d(sa, &tmA, &full[stage], i0, k0, c);
                        tma_load_3d(sa + BK * 128, &tmA, &full[stage], i0 + 64, k0, c);
#pragma unroll
                        for (int h = 0; h < 4; ++h) tma_load_3d(sb + h * BK * 128, &tmB, &full[stage], j0 + 64 * h, k0, c);
                    }
                    ever |= 1u << stage;
                    par = (par & ~(1u << stage)) | (phase << stage);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // Let every load already issued land before shared memory is released.
            for (int s = 0; s < STAGES; ++s)
                if ((ever >> s) & 1u) wait_drain(&full[s], (par >> s) & 1u, ctl.timeout_ns);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer ----------------
            const uint32_t idesc = idesc_bf16(BM, BN, args.incoming, args.incoming);
            const bool stall = (ctl.debug_flags & 0x1u) != 0;
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            int lt = 0;
            for (int tile = blockIdx.x; ok && tile < args.total_tiles; tile += gridDim.x, ++lt) {
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
                        uint64_t ad, bd;
                        if (!args.incoming) {
                            ad = sdesc_sw128(sa + kk * 32, 16, 1024);
                            bd = sdesc_sw128(sb + kk * 32, 16, 1024);
                        } else {
                            ad = sdesc_sw128(sa + kk * 2048, BK * 128, 1024);
                            bd = sdesc_sw128(sb + kk * 2048, BK * 128, 1024);
                        }
                        mma_bf16(d, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
                    }
                    mma_commit(&empty[stage]);  // frees the smem stage once these MMAs have read it
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                mma_commit(&tfull[acc]);
            }
            // No MMA may still be writing tensor memory at teardown.
            mma_commit(drain);
            wait_drain(drain, 0, ctl.timeout_ns);
        }
    } else {
        // ---------------- epilogue warps 2..5 ----------------
        const int q = warp & 3;  // TMEM lane quadrant this warp may access
        const int row = q * 32 + lane;
        const bool leader = (threadIdx.x == 64);
        int lt = 0;
        for (int tile = blockIdx.x; tile < args.total_tiles; tile += gridDim.x, ++lt) {
            const int c = tile / tiles_per_c;
            const int r = tile - c * tiles_per_c;
            const int ti = r / args.tj_tiles, tj = r - ti * args.tj_tiles;
            const int i0 = ti * BM, j0 = tj * BN;
            const int acc = lt & 1;
            const uint32_t acc_par = (uint32_t)(lt >> 1) & 1u;
            if (leader) *epi_go = wait_bounded(&tfull[acc], acc_par, abort_flag, ctl, SITE_CON | 4, tile) ? 1 : 0;
            named_bar_sync(1, 128);
            if (!*epi_go) break;
            tc_fence_after();
            // Chunks whose first column is past N are neither read nor stored.
            const int nch = min(BN / OUT_COLS, (args.N - j0 + OUT_COLS - 1) / OUT_COLS);
#pragma unroll 1
            for (int ch = 0; ch < nch; ++ch) {
                uint32_t v[64];
                const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN + ch * OUT_COLS);
                tmem_ld32(taddr, v);
                tmem_ld32(taddr + 32, v + 32);
                tmem_ld_wait();
                if (ch == nch - 1) {
                    tc_fence_before();
                    if (lane == 0) mbar_arrive(&tempty[acc]);
                }
                uint32_t p[32];
#pragma unroll
                for (int k = 0; k < 32; ++k) p[k] = pack_bf16x2(__uint_as_float(v[2 * k]), __uint_as_float(v[2 * k + 1]));
                uint8_t *ob = outbuf + (ch & 1) * OUT_BYTES;
                if (leader) tma_store_wait_read<1>();  // the store that last used `ob` has read it
                named_bar_sync(1, 128);
#pragma unroll
                for (int c16 = 0; c16 < 8; ++c16) {
                    uint4 val = make_uint4(p[4 * c16], p[4 * c16 + 1], p[4 * c16 + 2], p[4 * c16 + 3]);
                    *reinterpret_cast<uint4 *>(ob + row * 128 + ((c16 ^ (row & 7)) << 4)) = val;
                }
                fence_proxy_async_smem();
                named_bar_sync(1, 128);
                if (leader) {
                    tma_store_3d(&tmX, ob, j0 + ch * OUT_COLS, i0, c);
                    tma_store_commit();
                }
            }
        }
        if (leader) tma_store_wait_all<0>();
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, TMEM_COLS);
}

size_t contract_tc_smem() { return con::SMEM; }

cudaError_t contract_tc_setup() {
    return cudaFuncSetAttribute(contract_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)con::SMEM);
}

cudaError_t launch_contract_tc(const ContractMaps &m, const ContractArgs &a, int grid, cudaStream_t s) {
    contract_tc_kernel<<<grid, con::THREADS, con::SMEM, s>>>(m.a, m.b, m.x, a);
    return cudaGetLastError();
}

}  // namespace trimul

// atomattn_tc.cu - sequence-local atom attention on tcgen05 tensor cores.
//
// AlphaFold3's atom attention limited to windows of 32 queries x 128 keys,
// the stacked windows computed as one batched attention ("Scaling
// biomolecular modeling with context parallelism in NVIDIA BioNeMo", section
// "Efficient sequence-local atom attention"; semantics in include/atomattn.h).
//
// Work unit: (batch b, head h, group g of 4 consecutive windows). Its 128
// query atoms 128g .. 128g + 127 are the rows of one M = 128 MMA against the
// 224 key atoms the 4 windows cover together (128g - 48 .. 128g + 175):
//   S[128][224] = Q K^T            (tcgen05, TMEM columns [0, 224))
// Row r (window 4g + r / 32) uses only its window's 128 slots, columns
// [32 (r / 32), 32 (r / 32) + 128) of S; its softmax runs in the thread that
// owns TMEM lane r, and its probabilities go to shared memory as row r of a
// [128][256] K-major operand P whose other slots stay 0. Then
//   O[128][64] = P V               (tcgen05, TMEM columns [256, 320))
// over 256 key rows (slots 224 .. 255 have P = 0).
//
// Q, K and V are TMA-loaded as rows of 64 bf16: the head pair (h & ~1, h | 1),
// so that every operand has 128-byte rows (128-byte swizzle). S contracts the
// head's 32 of them (the K steps at byte offset 64 (h & 1)), and O's columns
// [32 (h & 1), 32 (h & 1) + 32) are the head's output.
//
// Warps 0-3: softmax and epilogue (thread = query row = TMEM lane). Warp 4,
// one thread: TMA loads (double-buffered stages) and MMA issue. Barriers, all
// waits bounded:
//   full[s]  TMA bytes of stage s landed              (producer -> MMA)
//   sfull    S of the unit is in TMEM                  (MMA commit -> warps 0-3)
//   pready   P written, S and the previous O read      (4 warp arrivals -> MMA)
//   ofull    O of the unit is in TMEM, stage free      (MMA commit -> warps 0-3, producer)
#include "kernels.h"

namespace trimul {
namespace aa {
constexpr int QW = 32, KW = 128;             // window: 32 queries, 128 key slots
constexpr int KOFF = (QW - KW) / 2;          // -48: first key atom of a window, from its first query
constexpr int WPG = 4;                       // windows per unit
constexpr int ROWS = QW * WPG;               // 128 query rows
constexpr int UNION = QW * (WPG - 1) + KW;   // 224 key rows of S
constexpr int VROWS = 256;                   // key rows of the second product
constexpr int ROWB = 128;                    // bytes per operand row (64 bf16)
constexpr int Q_BYTES = ROWS * ROWB;         // 16 KB
constexpr int K_BYTES = UNION * ROWB;        // 28 KB
constexpr int V_BYTES = VROWS * ROWB;        // 32 KB
constexpr int STAGE_BYTES = Q_BYTES + K_BYTES + V_BYTES;
constexpr int P_BLOCK = ROWS * 128;          // one 64-slot block of P (16 KB)
constexpr int P_BYTES = 4 * P_BLOCK;
constexpr int S_COL = 0, O_COL = 256, TMEM_COLS = 512;
constexpr int THREADS = 160;
constexpr int BAR_BYTES = 128;
constexpr size_t SMEM = 1024 + 2 * (size_t)STAGE_BYTES + P_BYTES + BAR_BYTES;
static_assert(STAGE_BYTES % 1024 == 0, "stage alignment");
static_assert(SMEM <= 232448, "shared memory budget");
}  // namespace aa

namespace {

__device__ __forceinline__ uint32_t p_chunk_addr(uint32_t pbase, int row, int cu) {
    // 16-byte chunk cu (slots 8 cu .. 8 cu + 7) of row `row` in the swizzled P operand.
    return pbase + (uint32_t)((cu >> 3) * aa::P_BLOCK + row * 128 + (((cu & 7) ^ (row & 7)) << 4));
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

struct Unit {
    int b, h, g;
};
__device__ __forceinline__ Unit unit_of(long long u, const AttnArgs &a) {
    Unit x;
    x.g = (int)(u % a.groups);
    const long long t = u / a.groups;
    x.h = (int)(t % a.heads);
    x.b = (int)(t / a.heads);
    return x;
}

}  // namespace

__global__ void __launch_bounds__(aa::THREADS, 1)
    atomattn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const AttnArgs args) {
    using namespace aa;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *stage_base = smem;
    uint8_t *pbuf = smem + 2 * STAGE_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(pbuf + P_BYTES);
    uint64_t *full = bars;        // [2]
    uint64_t *sfull = bars + 2;
    uint64_t *pready = bars + 3;
    uint64_t *ofull = bars + 4;
    uint64_t *drain = bars + 5;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 6);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const KernelCtl &ctl = args.ctl;
    const long long nunits = args.units;
    const int my_units = blockIdx.x < nunits ? (int)((nunits - 1 - blockIdx.x) / gridDim.x + 1) : 0;

    if (threadIdx.x == 0) {
        mbar_init(&full[0], 1);
        mbar_init(&full[1], 1);
        mbar_init(sfull, 1);
        mbar_init(pready, 4);
        mbar_init(ofull, 1);
        mbar_init(drain, 1);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    const uint32_t pbase = smem_u32(pbuf);
    if (warp < 4) {
        // P slots outside the row's window are 0 for every unit: write them once.
        const int row = threadIdx.x, q = warp;
        for (int cu = 0; cu < 32; ++cu)
            if (cu < 4 * q || cu >= 4 * q + 16) st_shared_v4(p_chunk_addr(pbase, row, cu), 0u, 0u, 0u, 0u);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 4) {
        if (lane == 0) {
            // ---------------- TMA producer and MMA issuer ----------------
            const uint32_t idesc_s = idesc_bf16(128, UNION, 0, 0);
            const uint32_t idesc_o = idesc_bf16(128, 64, 0, 1);
            int issued = 0, landed = 0;
            auto issue = [&](int lu) {
                const Unit un = unit_of(blockIdx.x + (long long)lu * gridDim.x, args);
                uint8_t *st = stage_base + (lu & 1) * STAGE_BYTES;
                const int x = (un.h & ~1) * 32, a0 = un.g * ROWS;
                mbar_arrive_expect_tx(&full[lu & 1], STAGE_BYTES);
                tma_load_3d(st, &tmQ, &full[lu & 1], x, a0, un.b);
                tma_load_3d(st + Q_BYTES, &tmK, &full[lu & 1], x, a0 + KOFF, un.b);
                tma_load_3d(st + Q_BYTES + K_BYTES, &tmV, &full[lu & 1], x, a0 + KOFF, un.b);
                ++issued;
            };
            auto mma_s = [&](int lu) -> bool {
                if (!wait_bounded(&full[lu & 1], (uint32_t)(lu >> 1) & 1u, abort_flag, ctl, SITE_ATT | 1, lu))
                    return false;
                ++landed;
                tc_fence_after();
                const Unit un = unit_of(blockIdx.x + (long long)lu * gridDim.x, args);
                const uint32_t st = smem_u32(stage_base + (lu & 1) * STAGE_BYTES);
                const uint32_t kofs = (uint32_t)(un.h & 1) * 64;  // the head's 32 elements in the 64-element row
#pragma unroll
                for (int kk = 0; kk < 2; ++kk)
                    mma_bf16(tmem + S_COL, sdesc_sw128(st + kofs + kk * 32, 16, 1024),
                             sdesc_sw128(st + Q_BYTES + kofs + kk * 32, 16, 1024), idesc_s, kk ? 1u : 0u);
                mma_commit(sfull);
                return true;
            };
            bool ok = true;
            if (my_units > 0) issue(0);
            if (my_units > 1) issue(1);
            if (my_units > 0) ok = mma_s(0);
            for (int lu = 0; ok && lu < my_units; ++lu) {
                if (!wait_bounded(pready, (uint32_t)lu & 1u, abort_flag, ctl, SITE_ATT | 2, lu)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t vst = smem_u32(stage_base + (lu & 1) * STAGE_BYTES) + Q_BYTES + K_BYTES;
#pragma unroll
                for (int kk = 0; kk < VROWS / 16; ++kk)
                    mma_bf16(tmem + O_COL, sdesc_sw128(pbase + (kk >> 2) * P_BLOCK + (kk & 3) * 32, 16, 1024),
                             sdesc_sw128(vst + kk * 2048, V_BYTES, 1024), idesc_o, kk ? 1u : 0u);
                mma_commit(ofull);
                if (lu + 1 < my_units && !(ok = mma_s(lu + 1))) break;
                if (lu + 2 < my_units) {
                    // The stage of unit lu is free once its second product has completed.
                    if (!wait_bounded(ofull, (uint32_t)lu & 1u, abort_flag, ctl, SITE_ATT | 3, lu)) {
                        ok = false;
                        break;
                    }
                    issue(lu + 2);
                }
            }
            if (!ok) *abort_flag = 1;
            // Let every copy in flight land and every MMA complete before the CTA exits.
            for (int lu = landed; lu < issued; ++lu) wait_drain(&full[lu & 1], (uint32_t)(lu >> 1) & 1u, ctl.timeout_ns);
            mma_commit(drain);
            wait_drain(drain, 0, ctl.timeout_ns);
        }
    } else {
        // ---------------- softmax and epilogue: thread = query row ----------------
        const int q = warp, row = threadIdx.x;
        const uint32_t lanebase = tmem + ((uint32_t)(q * 32) << 16);
        const float log2e = 1.4426950408889634f;
        for (int lu = 0; lu < my_units; ++lu) {
            const Unit un = unit_of(blockIdx.x + (long long)lu * gridDim.x, args);
            const int w = un.g * WPG + q;                 // this warp's window
            const int atom_q = un.g * ROWS + row;         // this thread's query atom
            const int k0 = w * QW + KOFF;                 // atom of key slot 0
            // Bias row of this query (prefetched before S is ready).
            uint4 bias[16];
            const bool has_bias = args.bias != nullptr && w < args.n_windows;
            if (has_bias) {
                const uint4 *bp = reinterpret_cast<const uint4 *>(
                    args.bias + ((((size_t)un.b * args.n_windows + w) * args.heads + un.h) * QW + lane) * KW);
#pragma unroll
                for (int i = 0; i < 16; ++i) bias[i] = __ldg(bp + i);
            }
            // Key validity: lane l decides slots 4l .. 4l + 3; bit e of vb[e] (lane l) <- slot 4l + e.
            uint32_t vb[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int a = k0 + 4 * lane + e;
                bool ok = a >= 0 && a < args.n;
                if (ok && args.mask) ok = __bfloat162float(args.mask[(size_t)un.b * args.n + a]) != 0.f;
                vb[e] = __ballot_sync(0xffffffffu, ok);
            }
            if (!warp_wait(sfull, (uint32_t)lu & 1u, abort_flag, ctl, SITE_ATT | 4, lu)) break;
            tc_fence_after();
            uint32_t s[128];
#pragma unroll
            for (int c = 0; c < 4; ++c) tmem_ld32(lanebase + (uint32_t)(S_COL + 32 * q + 32 * c), s + 32 * c);
            tmem_ld_wait();
            // Logits in the log2 domain; invalid slots -inf.
            float mx = -INFINITY;
#pragma unroll
            for (int j = 0; j < 128; ++j) {
                float bj = 0.f;
                if (has_bias) {
                    const __nv_bfloat162 *bb = reinterpret_cast<const __nv_bfloat162 *>(&bias[j >> 3]);
                    const float2 f = __bfloat1622float2(bb[(j & 7) >> 1]);
                    bj = (j & 1) ? f.y : f.x;
                }
                const bool valid = (vb[j & 3] >> (j >> 2)) & 1u;
                const float l = valid ? (__uint_as_float(s[j]) * args.scale + bj) * log2e : -INFINITY;
                s[j] = __float_as_uint(l);
                mx = fmaxf(mx, l);
            }
            const float m = mx == -INFINITY ? 0.f : mx;
            float sum = 0.f;
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                uint32_t pk[4];
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    const int j = 8 * c + 2 * t;
                    const __nv_bfloat162 pp =
                        __floats2bfloat162_rn(exp2f(__uint_as_float(s[j]) - m), exp2f(__uint_as_float(s[j + 1]) - m));
                    const float2 pr = __bfloat1622float2(pp);
                    sum += pr.x + pr.y;
                    pk[t] = *reinterpret_cast<const uint32_t *>(&pp);
                }
                st_shared_v4(p_chunk_addr(pbase, row, 4 * q + c), pk[0], pk[1], pk[2], pk[3]);
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(pready);
            if (!warp_wait(ofull, (uint32_t)lu & 1u, abort_flag, ctl, SITE_ATT | 5, lu)) break;
            tc_fence_after();
            uint32_t o[32];
            tmem_ld32(lanebase + (uint32_t)(O_COL + 32 * (un.h & 1)), o);
            tmem_ld_wait();
            if (atom_q < args.n) {
                const float inv = sum > 0.f ? 1.f / sum : 0.f;
                uint4 *op = reinterpret_cast<uint4 *>(args.out + (((size_t)un.b * args.n + atom_q) * args.heads + un.h) * 32);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    uint32_t pk[4];
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        const __nv_bfloat162 v = __floats2bfloat162_rn(__uint_as_float(o[8 * i + 2 * t]) * inv,
                                                                       __uint_as_float(o[8 * i + 2 * t + 1]) * inv);
                        pk[t] = *reinterpret_cast<const uint32_t *>(&v);
                    }
                    op[i] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, TMEM_COLS);
}

size_t atomattn_tc_smem() { return aa::SMEM; }

cudaError_t atomattn_tc_setup() {
    return cudaFuncSetAttribute(atomattn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)aa::SMEM);
}

cudaError_t launch_atomattn_tc(const AttnMaps &m, const AttnArgs &a, int grid, cudaStream_t s) {
    atomattn_tc_kernel<<<grid, aa::THREADS, aa::SMEM, s>>>(m.q, m.k, m.v, a);
    return cudaGetLastError();
}

}  // namespace trimul

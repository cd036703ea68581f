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
//   O[128][32] = P V               (tcgen05, TMEM columns [256, 288) or [288, 320) by unit parity)
// over 256 key rows (slots 224 .. 255 have P = 0).
//
// Q, K and V are TMA-loaded as rows of one head's 32 bf16 (64-byte rows, 64-byte
// swizzle): S contracts them in two K = 16 steps, and O = P V is M = 128, N = 32.
// The unit's bias (4 windows x 32 rows x 128 slots, 32 KB) is TMA-loaded into the
// same stage (128-byte swizzle) and read from shared memory by the softmax warps,
// each lane its own row.
//
// Warps 0-15: softmax and epilogue; warp w serves the query rows of TMEM lane
// quarter w & 3 and a quarter of their slots. Warp 16, one thread: TMA loads
// (double-buffered stages) and MMA issue. Barriers, all waits bounded:
//   full[s]  TMA bytes of stage s landed              (producer -> MMA)
//   sfull    S of the unit is in TMEM                  (MMA commit -> warps 0-15)
//   s_read   S of the unit is in the warps' registers  (16 warp arrivals -> MMA issues the next S)
//   pready   P written, S and the O of two units back read (16 warp arrivals -> MMA)
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
constexpr int ROWB = 64;                     // bytes per operand row (one head's 32 bf16)
constexpr int Q_BYTES = ROWS * ROWB;         // 8 KB
constexpr int K_BYTES = UNION * ROWB;        // 14 KB
constexpr int V_BYTES = VROWS * ROWB;        // 16 KB
constexpr int QKV_BYTES = Q_BYTES + K_BYTES + V_BYTES;
constexpr int BIAS_HALF = QW * 128;          // one window's 32 rows x 64 slots (4 KB, 128-byte rows)
constexpr int BIAS_WIN = 2 * BIAS_HALF;      // one window's 32 x 128 slots
constexpr int BIAS_BYTES = WPG * BIAS_WIN;   // 32 KB
constexpr int STAGE_BYTES = QKV_BYTES + BIAS_BYTES;
constexpr int P_BLOCK = ROWS * 128;          // one 64-slot block of P (16 KB)
constexpr int P_BYTES = 4 * P_BLOCK;
constexpr int S_COL = 0, O_COL = 256, TMEM_COLS = 512;
constexpr int WORKER_WARPS = 16;             // 4 per TMEM lane quarter, 32 of a row's 128 slots each
constexpr int THREADS = (WORKER_WARPS + 1) * 32;
constexpr int RED_BYTES = 2 * 2 * 4 * ROWS * 4;  // [max, sum][unit parity][key part][row] floats
constexpr int BAR_BYTES = 128;  // 11 mbarriers, TMEM address, abort flag
constexpr size_t SMEM = 1024 + 2 * (size_t)STAGE_BYTES + P_BYTES + RED_BYTES + BAR_BYTES;
static_assert(STAGE_BYTES % 1024 == 0 && QKV_BYTES % 1024 == 0, "stage alignment");
static_assert(SMEM <= 232448, "shared memory budget");
}  // namespace aa

namespace {

__device__ __forceinline__ uint32_t p_chunk_addr(uint32_t pbase, int row, int cu) {
    // 16-byte chunk cu (slots 8 cu .. 8 cu + 7) of row `row` in the swizzled P operand.
    return pbase + (uint32_t)((cu >> 3) * aa::P_BLOCK + row * 128 + (((cu & 7) ^ (row & 7)) << 4));
}

// 2^x on the MUFU (ex2.approx, relative error about 2^-22; 2^-inf = 0).
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// 2-byte load on the read-only path, kept where it is written (an early prefetch
// that the compiler must not sink to the first use).
__device__ __forceinline__ uint16_t ldg_early_u16(const uint16_t *p) {
    uint16_t v;
    asm volatile("ld.global.nc.u16 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}

// Unit u = (b * heads + h) * groups + g. A CTA visits u = blockIdx.x + lu * gridDim.x;
// the decode is done once and then stepped without division.
struct Unit {
    int b, h, g;
};
__device__ __forceinline__ Unit unit_of(int u, const AttnArgs &a) {
    Unit x;
    x.g = u % a.groups;
    const int t = u / a.groups;
    x.h = t % a.heads;
    x.b = t / a.heads;
    return x;
}
__device__ __forceinline__ void unit_step(Unit &x, const AttnArgs &a) {
    x.g += gridDim.x;
    while (x.g >= a.groups) {
        x.g -= a.groups;
        if (++x.h == a.heads) {
            x.h = 0;
            ++x.b;
        }
    }
}

}  // namespace

__global__ void __launch_bounds__(aa::THREADS, 1)
    atomattn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmBias,
                       const AttnArgs args) {
    using namespace aa;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *stage_base = smem;
    uint8_t *pbuf = smem + 2 * STAGE_BYTES;
    float *red = reinterpret_cast<float *>(pbuf + P_BYTES);  // [2][2][4][128]
    uint64_t *bars = reinterpret_cast<uint64_t *>(pbuf + P_BYTES + RED_BYTES);
    uint64_t *full = bars;        // [2]
    uint64_t *sfull = bars + 2;
    uint64_t *pready = bars + 3;
    uint64_t *ofull = bars + 4;
    uint64_t *drain = bars + 5;
    uint64_t *redbar = bars + 6;  // [4] per lane quarter: its 4 warps published their partials
    uint64_t *s_read = bars + 10;  // the worker warps have read S of the unit (16 warp arrivals)
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 11);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const KernelCtl &ctl = args.ctl;
    const long long nunits = args.units;
    const int my_units = blockIdx.x < nunits ? (int)((nunits - 1 - blockIdx.x) / gridDim.x + 1) : 0;

    if (threadIdx.x == 0) {
        mbar_init(&full[0], 1);
        mbar_init(&full[1], 1);
        mbar_init(sfull, 1);
        mbar_init(pready, WORKER_WARPS);
        mbar_init(ofull, 1);
        mbar_init(drain, 1);
        for (int i = 0; i < 4; ++i) mbar_init(&redbar[i], 4);
        mbar_init(s_read, WORKER_WARPS);
        *abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmQ);
        tma_prefetch_desc(&tmK);
        tma_prefetch_desc(&tmV);
        if (args.bias) tma_prefetch_desc(&tmBias);
    }
    if (warp == 0) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    const uint32_t pbase = smem_u32(pbuf);
    if (warp < WORKER_WARPS) {
        // P slots outside the row's window are 0 for every unit: write them once
        // (the four warps of a lane quarter split the chunks).
        const int qr = warp & 3, kp = warp >> 2, row = qr * 32 + lane;
        for (int cu = kp; cu < 32; cu += 4)
            if (cu < 4 * qr || cu >= 4 * qr + 16) st_shared_v4(p_chunk_addr(pbase, row, cu), 0u, 0u, 0u, 0u);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // The call starts here: CTA 0 clears the status word (every failure is recorded by a
    // bounded wait after ctl.timeout_ns, long after all CTAs of this one-wave grid started).
    if (blockIdx.x == 0 && threadIdx.x == 0) *ctl.status = DeviceStatus{0, 0, 0, 0};

    if (warp == WORKER_WARPS) {
        if (lane == 0) {
            // ---------------- TMA producer and MMA issuer ----------------
            const uint32_t idesc_s = idesc_bf16(128, UNION, 0, 0);
            const uint32_t idesc_o = idesc_bf16(128, 32, 0, 1);
            const uint64_t pdesc = sdesc_sw128(pbase, 16, 1024);
            int issued = 0, landed = 0;
            auto issue = [&](int lu) {
                const Unit un = unit_of((int)blockIdx.x + lu * (int)gridDim.x, args);
                uint8_t *st = stage_base + (lu & 1) * STAGE_BYTES;
                const int x = un.h * 32, a0 = un.g * ROWS;
                mbar_arrive_expect_tx(&full[lu & 1], args.bias ? STAGE_BYTES : QKV_BYTES);
                tma_load_3d(st, &tmQ, &full[lu & 1], x, a0, un.b);
                tma_load_3d(st + Q_BYTES, &tmK, &full[lu & 1], x, a0 + KOFF, un.b);
                tma_load_3d(st + Q_BYTES + K_BYTES, &tmV, &full[lu & 1], x, a0 + KOFF, un.b);
                if (args.bias) {
                    // Windows 4g .. 4g + 3, each as two boxes of 32 rows x 64 slots; windows past
                    // the last one are out of bounds and read as 0.
#pragma unroll
                    for (int w = 0; w < WPG; ++w)
#pragma unroll
                        for (int half = 0; half < 2; ++half)
                            tma_load_5d(st + QKV_BYTES + w * BIAS_WIN + half * BIAS_HALF, &tmBias, &full[lu & 1],
                                        64 * half, 0, un.h, un.g * WPG + w, un.b);
                }
                ++issued;
            };
            auto mma_s = [&](int lu) -> bool {
                if (!wait_bounded(&full[lu & 1], (uint32_t)(lu >> 1) & 1u, abort_flag, ctl, SITE_ATT | 1, lu))
                    return false;
                ++landed;
                tc_fence_after();
                const uint32_t st = smem_u32(stage_base + (lu & 1) * STAGE_BYTES);
#pragma unroll
                for (int kk = 0; kk < 2; ++kk)
                    mma_bf16(tmem + S_COL, sdesc_sw64(st + kk * 32, 16, 512), sdesc_sw64(st + Q_BYTES + kk * 32, 16, 512),
                             idesc_s, kk ? 1u : 0u);
                mma_commit(sfull);
                return true;
            };
            bool ok = true;
            if (my_units > 0) issue(0);
            if (my_units > 1) issue(1);
            if (my_units > 0) ok = mma_s(0);
            for (int lu = 0; ok && lu < my_units; ++lu) {
                if (lu + 1 < my_units) {
                    // S of the next unit overwrites S as soon as the worker warps have read it,
                    // so it is computed while they finish this unit's softmax.
                    if (!wait_bounded(s_read, (uint32_t)lu & 1u, abort_flag, ctl, SITE_ATT | 9, lu)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    if (!(ok = mma_s(lu + 1))) break;
                }
                if (!wait_bounded(pready, (uint32_t)lu & 1u, abort_flag, ctl, SITE_ATT | 2, lu)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // Descriptor start addresses count 16-byte units in their low bits:
                // step K by adding to the descriptor.
                const uint64_t vdesc = sdesc_sw64(smem_u32(stage_base + (lu & 1) * STAGE_BYTES) + Q_BYTES + K_BYTES,
                                                  V_BYTES, 512);
                const uint32_t od = tmem + O_COL + 32 * (lu & 1);
#pragma unroll
                for (int kk = 0; kk < VROWS / 16; ++kk)
                    mma_bf16(od, pdesc + (uint64_t)(((kk >> 2) * P_BLOCK + (kk & 3) * 32) >> 4),
                             vdesc + (uint64_t)((kk * 16 * ROWB) >> 4), idesc_o, kk ? 1u : 0u);
                mma_commit(ofull);
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
        // Warp (qr, kp) = (warp & 3, warp >> 2) owns query rows 32 qr .. 32 qr + 31
        // (TMEM lane quarter qr) and slots 32 kp .. 32 kp + 31 of their window.
        // Unit lu: its bias rows are in its stage (shared memory), its key-mask value was
        // loaded during unit lu - 1; logits stay in registers; partial row maxima and sums are exchanged
        // among the quarter's 4 warps through `red` (double-buffered by unit
        // parity) through one mbarrier phase per unit; P is written once the
        // previous unit's second product has finished reading it; then that
        // unit's output columns 8 kp .. 8 kp + 7 (O buffer (lu - 1) & 1) are stored.
        const int qr = warp & 3, kp = warp >> 2, row = qr * 32 + lane;
        const uint32_t lanebase = tmem + ((uint32_t)(qr * 32) << 16);
        const float log2e = 1.4426950408889634f;
        float *red_max = red, *red_sum = red + 2 * 4 * ROWS;
        uint16_t mk_n = 0;
        const bool hb = args.bias != nullptr;
        auto prefetch = [&](const Unit &un) {
            const int w = un.g * WPG + qr, at = w * QW + KOFF + 32 * kp + lane;
            mk_n = (at < 0 || at >= args.n) ? (uint16_t)0
                   : args.mask ? ldg_early_u16(reinterpret_cast<const uint16_t *>(args.mask) + (size_t)un.b * args.n + at)
                               : (uint16_t)0x3f80u;  // bf16 1.0
        };
        Unit prev{0, 0, 0};
        float sum_prev = 0.f;
        bool ok = true;
        // Output columns 8 kp .. 8 kp + 7 of unit lu (its second product has completed): the
        // tensor-memory load is issued first, the normalisation and store after the wait.
        auto load_o = [&](int lu, uint32_t (&o)[8]) {
            tc_fence_after();
            asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                         : "=r"(o[0]), "=r"(o[1]), "=r"(o[2]), "=r"(o[3]), "=r"(o[4]), "=r"(o[5]), "=r"(o[6]),
                           "=r"(o[7])
                         : "r"(lanebase + (uint32_t)(O_COL + 32 * (lu & 1) + 8 * kp)));
        };
        auto store_o = [&](uint32_t (&o)[8]) {
            tmem_ld_wait_regs(o);
            const int atom_q = prev.g * ROWS + row;
            if (atom_q < args.n) {
                const float inv = sum_prev > 0.f ? 1.f / sum_prev : 0.f;
                uint32_t pk[4];
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    const __nv_bfloat162 v = __floats2bfloat162_rn(__uint_as_float(o[2 * t]) * inv,
                                                                   __uint_as_float(o[2 * t + 1]) * inv);
                    pk[t] = *reinterpret_cast<const uint32_t *>(&v);
                }
                *reinterpret_cast<uint4 *>(args.out + (((size_t)prev.b * args.n + atom_q) * args.heads + prev.h) * 32 +
                                           8 * kp) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            }
        };
        Unit cur = unit_of((int)blockIdx.x, args);
        if (my_units > 0) prefetch(cur);
        for (int lu = 0; lu < my_units; ++lu) {
            const Unit un = cur;
            unit_step(cur, args);  // the next unit of this CTA
            const uint32_t vb = __ballot_sync(0xffffffffu, (mk_n & 0x7fffu) != 0);  // slot 32 kp + i valid: bit i
            if (!(ok = warp_wait(sfull, (uint32_t)lu & 1u, abort_flag, ctl, SITE_ATT | 4, lu))) break;
            // The stage's bias (TMA-written) is read below: observe its barrier here too (the
            // issuing thread waited on it before S, so this only makes the bytes visible).
            if (hb && !(ok = warp_wait(&full[lu & 1], (uint32_t)(lu >> 1) & 1u, abort_flag, ctl, SITE_ATT | 10, lu)))
                break;
            tc_fence_after();
            // Logits of the 32 slots in the log2 domain (invalid: -inf) and their maximum. This
            // lane's bias row is row `lane` of window qr's tile, slots 32 kp .. 32 kp + 31 in
            // 16-byte chunks 4 (kp & 1) .. 4 (kp & 1) + 3 of its 64-slot half kp / 2
            // (128-byte swizzle: chunk ^ (lane & 7)).
            float l[32];
            float mx4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
            {
                uint32_t sv[32];
                tmem_ld32(lanebase + (uint32_t)(S_COL + 32 * qr + 32 * kp), sv);
                // The bias row is read from shared memory while the S load is in flight.
                uint4 bcs[4];
                const uint8_t *brow = stage_base + (lu & 1) * STAGE_BYTES + QKV_BYTES + qr * BIAS_WIN +
                                      (kp >> 1) * BIAS_HALF + lane * 128;
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    bcs[c] = hb ? *reinterpret_cast<const uint4 *>(brow + (((4 * (kp & 1) + c) ^ (lane & 7)) << 4))
                                : make_uint4(0u, 0u, 0u, 0u);
                tmem_ld_wait_regs(sv);
                // S is in registers: the next unit's S may overwrite it.
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(s_read);
                // l = s (scale log2 e) + bias log2 e, two slots at a time (packed fp32x2).
                const float2 sc2 = make_float2(args.scale * log2e, args.scale * log2e);
                const float2 l2e = make_float2(log2e, log2e);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const uint4 bc = bcs[c];
                    const uint32_t bw[4] = {bc.x, bc.y, bc.z, bc.w};
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int t = 8 * c + 2 * u;
                        const float2 b2 = make_float2(__uint_as_float(bw[u] << 16), __uint_as_float(bw[u] & 0xFFFF0000u));
                        const float2 lv = __ffma2_rn(make_float2(__uint_as_float(sv[t]), __uint_as_float(sv[t + 1])), sc2,
                                                     __fmul2_rn(b2, l2e));
                        l[t] = lv.x;
                        l[t + 1] = lv.y;
                    }
                }
                if (vb != 0xFFFFFFFFu) {  // warp-uniform: some of the 32 slots are masked or outside the sequence
#pragma unroll
                    for (int t = 0; t < 32; ++t)
                        if (!((vb >> t) & 1u)) l[t] = -INFINITY;
                }
#pragma unroll
                for (int t = 0; t < 32; ++t) mx4[t & 3] = fmaxf(mx4[t & 3], l[t]);
            }
            if (lu + 1 < my_units) prefetch(cur);
            float *rm = red_max + (lu & 1) * 4 * ROWS, *rs = red_sum + (lu & 1) * 4 * ROWS;
            rm[kp * ROWS + row] = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
            __syncwarp();
            if (lane == 0) mbar_arrive(&redbar[qr]);
            if (!(ok = warp_wait(&redbar[qr], (uint32_t)lu & 1u, abort_flag, ctl, SITE_ATT | 7, lu))) break;
            float mx = fmaxf(fmaxf(rm[row], rm[ROWS + row]), fmaxf(rm[2 * ROWS + row], rm[3 * ROWS + row]));
            const float m = mx == -INFINITY ? 0.f : mx;
            if (lu > 0) {
                // The previous unit's row sum (its partial sums were published before this barrier).
                const float *ps = red_sum + ((lu - 1) & 1) * 4 * ROWS;
                sum_prev = ps[row] + ps[ROWS + row] + ps[2 * ROWS + row] + ps[3 * ROWS + row];
            }
            // P is free once the previous unit's second product has completed; its output is then
            // in tensor memory, and its load runs under the exponentials below.
            if (lu > 0 && !(ok = warp_wait(ofull, (uint32_t)(lu - 1) & 1u, abort_flag, ctl, SITE_ATT | 5, lu))) break;
            uint32_t o_prev[8];
            if (lu > 0) load_o(lu - 1, o_prev);
            // Probabilities (bf16), their partial sum, and this warp's 4 chunks of row `row` of P.
            // p = 2^(l - m) (hardware ex2; a masked slot's -inf gives 0), rounded to bf16; the
            // row sum adds the rounded values, the ones the second product uses.
            float2 s2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
            const float2 nm2 = make_float2(-m, -m);
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t pk[4];
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    const int j = 8 * c + 2 * t;
                    const float2 d = __fadd2_rn(make_float2(l[j], l[j + 1]), nm2);
                    pk[t] = pack_bf16x2(ex2_approx(d.x), ex2_approx(d.y));
                    s2[t & 1] = __fadd2_rn(s2[t & 1], make_float2(__uint_as_float(pk[t] << 16),
                                                                  __uint_as_float(pk[t] & 0xFFFF0000u)));
                }
                st_shared_v4(p_chunk_addr(pbase, row, 4 * qr + 4 * kp + c), pk[0], pk[1], pk[2], pk[3]);
            }
            rs[kp * ROWS + row] = (s2[0].x + s2[0].y) + (s2[1].x + s2[1].y);
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(pready);
            if (lu > 0) store_o(o_prev);
            prev = un;
        }
        if (ok && my_units > 0) {
            // The last unit's partial sums.
            __syncwarp();
            if (lane == 0) mbar_arrive(&redbar[qr]);
            ok = warp_wait(&redbar[qr], (uint32_t)my_units & 1u, abort_flag, ctl, SITE_ATT | 8, 0);
        }
        if (ok && my_units > 0) {
            const float *ps = red_sum + ((my_units - 1) & 1) * 4 * ROWS;
            sum_prev = ps[row] + ps[ROWS + row] + ps[2 * ROWS + row] + ps[3 * ROWS + row];
            if (warp_wait(ofull, (uint32_t)(my_units - 1) & 1u, abort_flag, ctl, SITE_ATT | 6, 0)) {
                uint32_t o_last[8];
                load_o(my_units - 1, o_last);
                store_o(o_last);
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
    atomattn_tc_kernel<<<grid, aa::THREADS, aa::SMEM, s>>>(m.q, m.k, m.v, m.bias, a);
    return cudaGetLastError();
}

}  // namespace trimul

// kernels.h - launch interface between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"

namespace trimul {

constexpr int kC = 128;  // c_z == c_h in this version

// ---- bf16 tensor-core path (tcgen05 + TMA) --------------------------------

// What the prologue writes:
//   PRO_BF16     a, b in bf16, channel-major [c][rows][ld]; tiles of 128 cells of one row.
//   PRO_MX_ROWS  a, b as MXFP8 operands of the outgoing contraction (operand row i,
//                K = column k): E4M3 [c][N][ldq] and E8M0 scales; same tiles, each
//                gating warp's 32 cells x 32 channels being 32 whole blocks.
//   PRO_MX_COLS  the same for the incoming contraction (operand row = column i of
//                a and b, K = residue row k): tiles of 32 rows x 4 columns, each
//                gating warp holding one column's 32 rows, again 32 whole blocks.
enum { PRO_BF16 = 0, PRO_MX_ROWS = 1, PRO_MX_COLS = 2 };

struct PrologueArgs {
    int N;
    int jt_tiles;     // PRO_BF16 / PRO_MX_ROWS: ceil(N / 128) tiles per residue row;
                      // PRO_MX_COLS: ceil(N / 4) groups of 4 columns per block of 32 rows
    int total_tiles;  // rows * jt_tiles (rows = N for the whole layer, fewer for a row shard);
                      // PRO_MX_COLS: ceil(N / 32) * jt_tiles
    float eps;
    int has_mask;                              // mask rows arrive by TMA (tensor map `mask`)
    const __nv_bfloat16 *ln_w, *ln_b;          // [128] or null
    const __nv_bfloat16 *b_a, *b_ag, *b_b, *b_bg;
    // MXFP8 modes: the scale arrays of the A (a) and B (b) operands, in the layout the
    // contraction reads (mx_scale_offset with these row tiles, K chunks and chunks per tile).
    uint8_t *sf[2];
    int sf_rows[2], sf_row_tiles[2], sf_chunks[2];
    int kchunks;
    // Nonzero: the call starts here, and CTA 0 zeroes the status word before anything else
    // (every recorded failure comes from a bounded wait that ran for ctl.timeout_ns, long
    // after all CTAs of this one-wave grid have started).
    int clear_status;
    KernelCtl ctl;
};

struct PrologueMaps {
    CUtensorMap w[4];  // W_a, W_ag, W_b, W_bg: 2-D [128 out][128 in], box 64 x 128, swizzle 128B
    CUtensorMap z;     // 3-D (c, j, i) over z, swizzle 128B; box (64, 128, 1), PRO_MX_COLS (64, 1, 32)
    CUtensorMap mask;  // 2-D (j, i) over the [rows][pitch] bf16 mask, box (128, 1), no swizzle;
                       // PRO_MX_COLS: (k, i) over the transposed mask, box (32, 4)
    CUtensorMap a, b;  // 3-D (x, row, c): PRO_BF16 over a / b [c][rows][ld], box (32, 1, 32), swizzle 64B;
                       // MXFP8 over the E4M3 operands [c][N][ldq] (uint8), box (32, 1, 32), no swizzle
};

// X[c][m][n] = sum_k A_c(m, k) B_c(n, k) for m < M, n < Ncols, k < K and every
// batch index c (a channel of the contraction, or a chunk of the backward's
// GEMMs): the triangle contraction is M = Ncols = K = N over 128 channels.
struct ContractArgs {
    int M, Ncols, K;
    int a_mn, b_mn;   // operand storage: 0 = K-major [rows][k], 1 = MN-major [k][rows]
    int ti_tiles;     // ceil(M / 256)
    int tj_tiles;     // ceil(Ncols / 256)
    int total_tiles;  // batch * ti_tiles * tj_tiles
    int kblocks;      // ceil(K / 64)
    int out_f32;      // X is fp32 (else bf16)
    KernelCtl ctl;
};

struct ContractMaps {
    CUtensorMap a, b;  // K-major: box (64 k, 128 rows, 1); MN-major: box (64 rows, 64 k, 1); swizzle 128B
    CUtensorMap x;     // 3-D (n, m, c) over X, box (64 bf16 | 32 fp32, 32, 1), swizzle 128B
};

struct EpilogueArgs {
    int N;
    int jt_tiles;
    int total_tiles;
    float eps;
    const __nv_bfloat16 *ln_in_w, *ln_in_b;
    const __nv_bfloat16 *ln_out_w, *ln_out_b;
    const __nv_bfloat16 *b_g, *b_o;
    KernelCtl ctl;
};

struct EpilogueMaps {
    CUtensorMap wg, wo;  // 2-D [128][128], box 64 x 128, swizzle 128B
    CUtensorMap z;       // as in the prologue
    CUtensorMap x;       // 3-D (j, i, c) over x, box (64, 1, 128), swizzle 128B
    CUtensorMap out;     // 3-D (c, j, i) over out, box (32, 32, 1), swizzle 64B
};

size_t prologue_tc_smem();
size_t epilogue_tc_smem();
cudaError_t prologue_tc_setup();
cudaError_t epilogue_tc_setup();
cudaError_t launch_prologue_tc(const PrologueMaps &m, const PrologueArgs &a, int mode, int grid, cudaStream_t s);
// Copies the [rows][N] mask into rows of pitch ld (zero past column N), for a tensor map.
cudaError_t launch_mask_pad(const __nv_bfloat16 *mask, __nv_bfloat16 *dst, int N, int rows, int ld, cudaStream_t s);
// dst[i][k] = mask[k][i] for i, k < N, zero for N <= k < ld (the transposed mask the
// PRO_MX_COLS prologue reads).
cudaError_t launch_mask_transpose(const __nv_bfloat16 *mask, __nv_bfloat16 *dst, int N, int ld, cudaStream_t s);
size_t contract_tc_smem();
cudaError_t contract_tc_setup();
// Clusters of 2 CTAs, one 256 x 256 output tile per pair; grid = 2 x pairs.
cudaError_t launch_contract_tc(const ContractMaps &m, const ContractArgs &a, int grid, cudaStream_t s);
cudaError_t launch_epilogue_tc(const EpilogueMaps &m, const EpilogueArgs &a, int grid, cudaStream_t s);

// ---- MXFP8 contraction (mx_tc.cu) ------------------------------------------------

// Quantizer: src [128][N][ld] bf16 (operand rows m, K index k: src[c][m][k], or
// src[c][k][m] when transposed) -> q [128][N][ldq] E4M3 (row m, k contiguous)
// and E8M0 scales per block of 32 along k, laid out per row tile of
// rows_per_tile rows (chunks_per_tile chunks of 128 rows) and per 128-wide K
// chunk (512 bytes per chunk, see mx_tc.cu).
struct MxQuantArgs {
    const __nv_bfloat16 *src;
    int N;
    size_t ld;
    uint8_t *q;
    size_t ldq;        // multiple of 16
    uint8_t *sf;
    int rows_per_tile;  // 128 (A) or 192 (B)
    int row_tiles;
    int kchunks;       // ceil(N / 128)
    int chunks_per_tile;
};

struct ContractMxArgs {
    int N;
    int ti_tiles;      // ceil(N / 256)
    int tj_tiles;      // ceil(N / 192)
    int total_tiles;   // 128 * ti_tiles * tj_tiles
    int kchunks;       // ceil(N / 128)
    int a_row_tiles;   // 2 * ti_tiles (128-row halves)
    int b_row_tiles;   // tj_tiles
    KernelCtl ctl;
};

struct ContractMxMaps {
    CUtensorMap a, b;    // 3-D (k, m, c) over q [128][N][ldq] uint8, boxes (128, 128 | 96, 1), swizzle 128B
    CUtensorMap sa, sb;  // 2-D (16 bytes, rows) over the scale arrays, boxes (16, 32 | 64)
    CUtensorMap x;       // 3-D (j, i, c) over x, box (64, 32, 1), swizzle 128B
};

cudaError_t launch_mx_quant(const MxQuantArgs &a, int transposed, cudaStream_t s);
cudaError_t contract_mx_setup();
// Clusters of 2 CTAs, one 256 x 192 output tile per pair; grid = 2 x pairs.
cudaError_t launch_contract_mx(const ContractMxMaps &m, const ContractMxArgs &a, int grid, cudaStream_t s);

// ---- backward (bf16 forward intermediates, fp32 gradients) -----------------------

// Gradient sums over cells, [kSumCount][128] floats in the backward workspace.
enum BwdSum { S_B_G, S_B_O, S_B_A, S_B_AG, S_B_B, S_B_BG, S_LN_OUT_W, S_LN_OUT_B, S_LN_IN_W, S_LN_IN_B, kSumCount };

// Projection blocks of the [cells][5 * 128] arrays P (pre-activations) and D
// (their gradients), and of the stacked weight [5 * 128][128].
enum ProjBlock { P_G, P_A, P_AG, P_B, P_BG, kProjBlocks };

// The per-cell backward kernels work on a block of `rows` rows of the N x N
// grid, rows i0 .. i0 + rows - 1: cell-major arrays ([cells][...]) are passed
// already offset to the block's first cell (cell (i0 + r, j) at index r N + j);
// channel-major arrays ([128][N][ld]) and the mask are passed whole and indexed
// by the global row.

// LayerNorm of each cell: out = (v - mean) * rstd * gamma + beta as bf16
// [cells][128], and (mean, rstd) per cell. src is cell-major [cells][128] or,
// when channel_major, [128][N][ld].
struct LnFwdArgs {
    const __nv_bfloat16 *src;
    int channel_major;
    int N, rows, i0;
    size_t ld;
    float eps;
    const __nv_bfloat16 *gamma, *beta;  // or null
    __nv_bfloat16 *out;
    float2 *stats;
};

// LayerNorm adjoint: dsrc = rstd * (dn - mean(dn) - n * mean(dn * n)) with
// dn = dh * gamma and n recomputed from src and stats; dgamma += dh * n and
// dbeta += dh over all cells. dsrc has src's layout (bf16).
struct LnBwdArgs {
    const float *dh;  // [cells][128]
    const __nv_bfloat16 *src;
    int channel_major;
    int N, rows, i0;
    size_t ld;
    const float2 *stats;
    const __nv_bfloat16 *gamma;  // or null
    __nv_bfloat16 *dsrc;
    float *dgamma, *dbeta;
};

// Output gate adjoint, per cell and channel: g = sigmoid(P_G + b_g),
// y = Y + b_o, dy = dout * g, dP_G = dout * y * g * (1 - g).
struct GateBwdArgs {
    const __nv_bfloat16 *dout;  // [cells][128]
    const __nv_bfloat16 *P;     // [cells][5 * 128]
    const __nv_bfloat16 *Y;     // [cells][128]
    const __nv_bfloat16 *b_g, *b_o;
    __nv_bfloat16 *dy;  // [cells][128]
    __nv_bfloat16 *dg;  // dP_G of cell m at dg + m * dg_stride (128 channels)
    size_t dg_stride;
    float *db_g, *db_o;  // or null: no sums
    long long cells;
};

// Gating and mask adjoint of a and b: from dA, dB ([128][N][ld] bf16) and P,
// writes D blocks P_A .. P_BG and adds their sums over cells to db.
struct ProjBwdArgs {
    const __nv_bfloat16 *dA, *dB;
    const __nv_bfloat16 *P;
    const __nv_bfloat16 *mask;  // [N][N] or null
    const __nv_bfloat16 *b_a, *b_ag, *b_b, *b_bg;
    __nv_bfloat16 *D;
    float *db;  // [4][128]: b_a, b_ag, b_b, b_bg
    int N, rows, i0;
    size_t ld;
};

// Weight gradients: the rows of [W_g; W_a; W_ag; W_b; W_bg; W_o] gradients,
// each GEMM partial (one per chunk of cells) being [kWgradRows][128] fp32.
constexpr int kWgradRows = (kProjBlocks + 1) * kC;
// One reduction adds the partials of one block of rows to a running sum in
// double (rows row0 .. row0 + rows of the stacked gradient), and the last block
// writes the sums out.
struct WgradReduceArgs {
    const float *partial;  // [slots][kWgradRows][128]
    int slots;
    int row0, rows;
    double *acc;  // [kWgradRows][128]
    int first, last;
    float *dst[kProjBlocks + 1];  // [128][128] each (block order above), or null
};

cudaError_t backward_setup();
// Each launcher sizes its grid as one wave of resident blocks on `sms` SMs.
cudaError_t launch_ln_fwd(const LnFwdArgs &a, int sms, cudaStream_t s);
cudaError_t launch_ln_bwd(const LnBwdArgs &a, int sms, cudaStream_t s);
cudaError_t launch_gate_bwd(const GateBwdArgs &a, int sms, cudaStream_t s);
cudaError_t launch_proj_bwd(const ProjBwdArgs &a, int sms, cudaStream_t s);
cudaError_t launch_wgrad_reduce(const WgradReduceArgs &a, cudaStream_t s);

// ---- sequence-local atom attention (atomattn_tc.cu) ---------------------------

struct AttnArgs {
    int batch, n, heads;
    int groups;      // ceil(n / 128): units of 4 windows per (batch, head)
    int n_windows;   // ceil(n / 32)
    long long units; // batch * heads * groups
    const __nv_bfloat16 *bias;  // [batch][n_windows][heads][32][128] or null
    const __nv_bfloat16 *mask;  // [batch][n] or null
    __nv_bfloat16 *out;         // [batch][n][heads][32]
    float scale;                // 1 / sqrt(32)
    KernelCtl ctl;
};

struct AttnMaps {
    CUtensorMap q, k, v;  // 3-D (heads * 32, n, batch), boxes (32, 128 | 224 | 256, 1), swizzle 64B
    CUtensorMap bias;     // 5-D (128 slots, 32 rows, heads, n_windows, batch), box (64, 32, 1, 1, 1), swizzle 128B
};

size_t atomattn_tc_smem();
cudaError_t atomattn_tc_setup();
cudaError_t launch_atomattn_tc(const AttnMaps &m, const AttnArgs &a, int grid, cudaStream_t s);

// ---- static scratch of trimul_forward_noalloc (noalloc.cu) --------------------

// Device address of the library's static scratch array on the current device;
// TRIMUL_OK or TRIMUL_ERR_CUDA.
int noalloc_scratch_address(void **out);

// ---- fp32 CUDA-core path ----------------------------------------------------

struct F32Layer {
    int N;
    size_t ld;
    float eps;
    const float *mask;
    const float *ln_in_w, *ln_in_b, *ln_out_w, *ln_out_b;
    const float *w_a, *w_ag, *w_b, *w_bg, *w_g, *w_o;
    const float *b_a, *b_ag, *b_b, *b_bg, *b_g, *b_o;
    float *a, *b, *x;  // workspace sections, [128][N][ld]
};

cudaError_t launch_prologue_f32(const float *z, const F32Layer &L, int grid, cudaStream_t s);
cudaError_t launch_contract_f32(const F32Layer &L, int incoming, cudaStream_t s);
cudaError_t launch_epilogue_f32(const float *z, float *out, const F32Layer &L, int grid, cudaStream_t s);

}  // namespace trimul

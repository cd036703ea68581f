// kernels.h - launch interface between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"

namespace trimul {

constexpr int kC = 128;  // c_z == c_h in this version

// ---- bf16 tensor-core path (tcgen05 + TMA) --------------------------------

struct PrologueArgs {
    int N;
    int jt_tiles;     // ceil(N / 128): 128-cell tiles per residue row
    int total_tiles;  // N * jt_tiles
    float eps;
    int has_mask;                              // mask rows arrive by TMA (tensor map `mask`)
    const __nv_bfloat16 *ln_w, *ln_b;          // [128] or null
    const __nv_bfloat16 *b_a, *b_ag, *b_b, *b_bg;
    KernelCtl ctl;
};

struct PrologueMaps {
    CUtensorMap w[4];  // W_a, W_ag, W_b, W_bg: 2-D [128 out][128 in], box 64 x 128, swizzle 128B
    CUtensorMap z;     // 3-D (c, j, i) over z, box (64, 128, 1), swizzle 128B
    CUtensorMap mask;  // 2-D (j, i) over the [N][pitch] bf16 mask, box (128, 1), no swizzle
    CUtensorMap a, b;  // 3-D (j, i, c) over a / b [c][N][ld], box (32, 1, 32), swizzle 64B
};

struct ContractArgs {
    int N;
    int incoming;
    int ti_tiles;     // ceil(N / 256)
    int tj_tiles;     // ceil(N / 256)
    int total_tiles;  // 128 * ti_tiles * tj_tiles
    int kblocks;      // ceil(N / 64)
    KernelCtl ctl;
};

struct ContractMaps {
    CUtensorMap a, b;  // outgoing: box (64 k, 128 rows, 1); incoming: box (64 rows, 64 k, 1); swizzle 128B
    CUtensorMap x;     // 3-D (j, i, c) over x, box (64, 128, 1), swizzle 128B
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
cudaError_t launch_prologue_tc(const PrologueMaps &m, const PrologueArgs &a, int grid, cudaStream_t s);
// Copies the [N][N] mask into rows of pitch ld (zero past column N), for a tensor map.
cudaError_t launch_mask_pad(const __nv_bfloat16 *mask, __nv_bfloat16 *dst, int N, int ld, cudaStream_t s);
size_t contract_tc_smem();
cudaError_t contract_tc_setup();
// Clusters of 2 CTAs, one 256 x 256 output tile per pair; grid = 2 x pairs.
cudaError_t launch_contract_tc(const ContractMaps &m, const ContractArgs &a, int grid, cudaStream_t s);
cudaError_t launch_epilogue_tc(const EpilogueMaps &m, const EpilogueArgs &a, int grid, cudaStream_t s);

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

/*
 * trimul.h - C ABI of the B200 (sm_100a) triangle multiplicative update.
 *
 * The layer is the pair-representation update the pages call
 * TriangleMultiplicationOutgoing, invoked as layer(x, mask) after loading a
 * state dict ("Scaling biomolecular modeling with context parallelism in
 * NVIDIA BioNeMo", section "Context-parallel implementation of triangle
 * multiplication"), together with its incoming counterpart. Per cell (i, j)
 * of the N x N pair representation z (c_z channels):
 *
 *   zh    = LayerNorm_in(z)                                   (over c_z)
 *   a     = mask * sigmoid(W_ag zh + b_ag) * (W_a zh + b_a)  (c_h channels)
 *   b     = mask * sigmoid(W_bg zh + b_bg) * (W_b zh + b_b)
 *   x_ij  = sum_k a_ik * b_jk      (TRIMUL_OUTGOING)
 *   x_ij  = sum_k a_ki * b_kj      (TRIMUL_INCOMING)
 *   out   = sigmoid(W_g zh + b_g) * (W_o LayerNorm_out(x) + b_o)
 *
 * LayerNorm uses the biased variance over its channels and eps inside the
 * square root. The mask multiplies a and b at their own cell only.
 *
 * Layouts (row-major, contiguous, element type = params.dtype):
 *   z, out   [N][N][c_z]   channel-last pair representation
 *   mask     [N][N]        or NULL (all ones)
 *   W_a, W_ag, W_b, W_bg  [c_h][c_z];  W_g [c_z][c_z];  W_o [c_z][c_h]
 *            PyTorch Linear layout [out][in], y = W x + b
 *   biases, LayerNorm weight/bias: vectors, or NULL (bias 0, gamma 1, beta 0)
 *
 * Ownership and threading: the caller owns every buffer, including the
 * workspace. The library allocates nothing, frees nothing and does not
 * synchronise in trimul_forward or the stage calls: work is enqueued on
 * `stream` and the call returns. Its only global state is per-device launch
 * configuration (maximum shared memory attribute, SM count, cached driver
 * entry point), set up once and guarded for concurrent callers.
 *
 * Errors: every call returns TRIMUL_OK (0) or a negative code; no exception
 * crosses this boundary. Argument errors are detected on the host before any
 * work is enqueued. Errors found by a kernel (a bounded wait that ran out) are
 * written to a status word in the workspace and read with trimul_device_status.
 *
 * Version 1 supports c_z == c_h == 128, batch 1, dtype F32 (CUDA-core fp32
 * kernels) or BF16 (tcgen05 tensor-core kernels with fp32 accumulation).
 */
#ifndef TRIMUL_B200_H
#define TRIMUL_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* A CUDA stream (cudaStream_t); NULL is the legacy default stream. */
typedef struct CUstream_st *trimul_stream_t;

enum trimul_direction { TRIMUL_OUTGOING = 0, TRIMUL_INCOMING = 1 };
enum trimul_dtype { TRIMUL_DTYPE_F32 = 0, TRIMUL_DTYPE_BF16 = 1 };

enum trimul_status {
    TRIMUL_OK = 0,
    TRIMUL_ERR_INVALID_ARG = -1,  /* NULL required pointer, N < 1 or too large, bad direction */
    TRIMUL_ERR_UNSUPPORTED = -2,  /* c_z or c_h != 128, unknown dtype, no sm_100 device */
    TRIMUL_ERR_MISALIGNED = -3,   /* a pointer the kernels read with TMA is not 16-byte aligned */
    TRIMUL_ERR_ALIAS = -4,        /* out overlaps z, the mask or the workspace */
    TRIMUL_ERR_WORKSPACE = -5,    /* workspace NULL or smaller than trimul_workspace_size_dtype */
    TRIMUL_ERR_CUDA = -6,         /* a CUDA runtime / driver call failed (launch, tensor map) */
    TRIMUL_ERR_TIMEOUT = -7,      /* device: a bounded in-kernel wait ran out; results invalid */
    TRIMUL_ERR_DEVICE = -8        /* device: another kernel-detected fault; results invalid */
};

/* Debug flags (0 in production). */
#define TRIMUL_DEBUG_STALL_CONTRACT 0x1u /* contraction's MMA issuer waits on a barrier nothing
                                            signals, so its bounded wait runs out (failure test) */

typedef struct trimul_params {
    int N;              /* residues; 1 <= N <= 16384 */
    int c_z, c_h;       /* channels; both must be 128 in version 1 */
    int dtype;          /* enum trimul_dtype: element type of z, mask, weights, out */
    float ln_eps;       /* LayerNorm epsilon for both LayerNorms (1e-5 = torch default) */
    const void *ln_in_w, *ln_in_b;     /* [c_z] or NULL */
    const void *w_a, *w_ag, *w_b, *w_bg; /* [c_h][c_z], required */
    const void *b_a, *b_ag, *b_b, *b_bg; /* [c_h] or NULL */
    const void *w_g, *b_g;             /* [c_z][c_z] required; [c_z] or NULL */
    const void *ln_out_w, *ln_out_b;   /* [c_h] or NULL */
    const void *w_o, *b_o;             /* [c_z][c_h] required; [c_z] or NULL */
    void *workspace;                   /* device memory, 256-byte aligned */
    size_t workspace_bytes;
    uint32_t timeout_ms;               /* bound on any in-kernel wait; 0 = 2000 ms */
    uint32_t debug_flags;              /* TRIMUL_DEBUG_*; 0 in production */
} trimul_params;

/* Bytes of workspace that trimul_forward needs for any dtype (sized for the
 * fp32 element). Returns 0 for invalid sizes. The workspace holds a 256-byte
 * status header and a, b, x as [c_h][N][ld] with ld = N rounded up to 64 for
 * BF16 (every row starts on a 128-byte boundary) and to 8 for F32. */
size_t trimul_workspace_size(int N, int c_z, int c_h);

/* Exact bytes of workspace for one dtype (<= trimul_workspace_size). */
size_t trimul_workspace_size_dtype(int N, int c_z, int c_h, int dtype);

/* The whole layer: out = TriMul_direction(z, mask). Enqueues three kernels
 * (prologue, contraction, epilogue) on `stream` after clearing the workspace
 * status word. z, out, weights and the workspace must be 16-byte aligned;
 * out must not overlap z, mask or the workspace. Asynchronous. */
int trimul_forward(const void *z, const void *mask, const trimul_params *p, int direction,
                   void *out, trimul_stream_t stream);

/* The three stages of trimul_forward, for callers that time or check them one
 * at a time. Each is asynchronous and needs the same params.
 *  prologue: z, mask -> a, b in the workspace (channel-major [c_h][N][ld])
 *  contract: a, b -> x in the workspace, x_c = a_c b_c^T (outgoing) or a_c^T b_c
 *  epilogue: x, z -> out
 * trimul_prologue also clears the status word. */
int trimul_prologue(const void *z, const void *mask, const trimul_params *p, trimul_stream_t stream);
int trimul_contract(const trimul_params *p, int direction, trimul_stream_t stream);
int trimul_epilogue(const void *z, const trimul_params *p, void *out, trimul_stream_t stream);

/* Device pointers of a, b and x inside p->workspace and their leading
 * dimension in elements (each is [c_h][N][ld] of p->dtype). Host-only. */
int trimul_workspace_views(const trimul_params *p, void **a, void **b, void **x, size_t *ld);

/* Synchronises `stream`, then returns the status word the kernels wrote
 * since it was last cleared: TRIMUL_OK, TRIMUL_ERR_TIMEOUT or
 * TRIMUL_ERR_DEVICE (or TRIMUL_ERR_CUDA if reading it failed). If `detail` is
 * not NULL it receives 4 ints: code, site, block index, auxiliary value.
 * With p->workspace NULL it reads the status word of the static scratch that
 * trimul_forward_noalloc uses on the current device. */
int trimul_device_status(const trimul_params *p, trimul_stream_t stream, int *detail);

/* Static description of a status code. */
const char *trimul_error_string(int code);

/* Human-readable detail of the last error this thread saw (the failing CUDA
 * call and its message), or "" if none. Valid until the next call. */
const char *trimul_last_error_detail(void);

/* Bytes of the library's static scratch array used by trimul_forward_noalloc:
 * room for the bf16 layer at N <= 128 and the fp32 layer at N <= 88. */
#define TRIMUL_NOALLOC_SCRATCH_BYTES (256u + 3u * 4194304u)

/* trimul_forward for callers that cannot allocate device memory. The pages
 * have no counterpart of this entry point; it exists for callers such as a
 * plugin whose host application owns all device memory and forbids other
 * allocations, or a latency-critical loop that must not risk an allocation.
 *
 * Same arguments and results as trimul_forward, except that p->workspace and
 * p->workspace_bytes are ignored: the scratch lives in a file-scope device
 * array of TRIMUL_NOALLOC_SCRATCH_BYTES inside the library, which every GPU
 * that loads the library keeps until the process exits. Sizes that do not fit
 * it (bf16 N > 128, fp32 N > 88) return TRIMUL_ERR_WORKSPACE before any work
 * is enqueued. Nothing is allocated or freed.
 *
 * All calls share the one array and a call leaves its contents behind (the
 * status word is cleared at the start of each call): calls whose GPU work
 * overlaps, on different streams or from different host threads, race and
 * give wrong results. The first call with a given device current looks up
 * the array's device address for that device; make that first call before
 * any stream capture. trimul_device_status, given a params block whose
 * workspace is NULL, reads the status word this entry point's kernels wrote
 * (an in-kernel timeout leaves the output invalid and is reported there). */
int trimul_forward_noalloc(const void *z, const void *mask, const trimul_params *p, int direction,
                           void *out, trimul_stream_t stream);

/* ---- Shard stage calls (the layer split over several GPUs) -------------------
 * The pages' subject is running this layer on many GPUs ("Scaling
 * biomolecular modeling with context parallelism in NVIDIA BioNeMo", sections
 * "2-D tiling of the pair representation" and "Context-parallel
 * implementation of triangle multiplication"). These calls are the per-GPU
 * pieces of the plainest such split: each GPU projects a block of residue
 * rows (all channels), the channels are exchanged so that each GPU contracts
 * a block of channels over all rows, x is exchanged back to row blocks, and
 * each GPU finishes its rows. The exchanges are the caller's (NCCL send/recv
 * through torch.distributed in pair_representation_b200.sharded); the
 * prologue and epilogue are per cell, so a row block is just a grid of
 * rows x N cells. All buffers are caller-owned device memory, 16-byte
 * aligned; ld = N rounded up to 64. BF16 only (TRIMUL_ERR_UNSUPPORTED
 * otherwise); p->N is the full residue count and p->workspace holds the status
 * word and scratch for re-pitching mask rows:
 * trimul_shard_workspace_size(N, rows) bytes. Asynchronous. */
size_t trimul_shard_workspace_size(int N, int rows);

/* z_rows [rows][N][c_z] and mask_rows [rows][N] (or NULL) of a block of
 * residue rows -> a, b [c_h][rows][ld] (channel-major). Clears the status word. */
int trimul_prologue_rows(const void *z_rows, const void *mask_rows, const trimul_params *p, int rows,
                         void *a, void *b, trimul_stream_t stream);

/* The triangle contraction of `channels` (1..c_h) channels over all N rows:
 * a, b, x [channels][N][ld]; x_c = a_c b_c^T (outgoing) or a_c^T b_c. */
int trimul_contract_channels(const trimul_params *p, int direction, int channels, const void *a,
                             const void *b, void *x, trimul_stream_t stream);

/* z_rows [rows][N][c_z] and x_rows [c_h][rows][ld] of a block of residue rows
 * -> out_rows [rows][N][c_z]. */
int trimul_epilogue_rows(const void *z_rows, const void *x_rows, const trimul_params *p, int rows,
                         void *out_rows, trimul_stream_t stream);

/* ---- MXFP8 contraction ------------------------------------------------------
 * The layer with its triangle contraction in MXFP8, the Blackwell
 * microscaling format the BioNeMo recipes list among their training
 * precisions ("Scaling biomolecular modeling with context parallelism in
 * NVIDIA BioNeMo", the precision list), read as OCP Microscaling (MX) v1.0:
 * a and b, as the prologue stores them in bf16, are quantised in blocks of 32
 * along the contracted index k (along the rows of a and b for
 * TRIMUL_OUTGOING, down their columns for TRIMUL_INCOMING) to E4M3 elements
 * (round to nearest even, saturated at +-448) sharing an E8M0 scale
 * 2^(floor(log2 max|v|) - 8); the contraction then runs on tcgen05
 * block-scaled MMAs (kind::mxf8f6f4) with fp32 accumulation and writes x in
 * bf16. The epilogue is that of trimul_forward. trimul_forward_mxfp8 runs the
 * prologue in a quantising form (trimul_prologue_mxfp8): it rounds a and b to
 * bf16 exactly as trimul_prologue stores them and writes their E4M3 codes and
 * scales straight into the workspace, so no bf16 copy of a and b is stored or
 * read back.
 *
 * BF16 only (TRIMUL_ERR_UNSUPPORTED otherwise). p->workspace must hold
 * trimul_workspace_size_mxfp8(N, c_z, c_h) bytes: the bf16 sections of
 * trimul_forward followed by the E4M3 operands and their scales
 * (TRIMUL_ERR_WORKSPACE if smaller). Everything else as for trimul_forward:
 * asynchronous, nothing allocated, status word in the workspace. */
size_t trimul_workspace_size_mxfp8(int N, int c_z, int c_h);
int trimul_forward_mxfp8(const void *z, const void *mask, const trimul_params *p, int direction,
                         void *out, trimul_stream_t stream);

/* Stage calls of the MXFP8 layer (trimul_forward_mxfp8 = trimul_prologue_mxfp8,
 * trimul_mma_mxfp8, trimul_epilogue on one stream):
 *   trimul_prologue_mxfp8  z, mask -> the E4M3 operands and scales of
 *                          `direction`'s contraction (the bf16 a, b sections
 *                          are left untouched);
 *   trimul_mma_mxfp8       the block-scaled contraction of the operands in the
 *                          workspace -> x (bf16); the operands already encode
 *                          the direction;
 *   trimul_contract_mxfp8  a, b (bf16, in the workspace) -> x: quantises them
 *                          (a separate pass) and runs trimul_mma_mxfp8. */
int trimul_prologue_mxfp8(const void *z, const void *mask, const trimul_params *p, int direction,
                          trimul_stream_t stream);
int trimul_mma_mxfp8(const trimul_params *p, trimul_stream_t stream);
int trimul_contract_mxfp8(const trimul_params *p, int direction, trimul_stream_t stream);

/* Device pointers of the quantised operands inside p->workspace (host-only):
 * aq, bq are [c_h][N][ldq] E4M3 codes, operand row m with k contiguous (for
 * TRIMUL_INCOMING the transposes of a_c and b_c); sa, sb the E8M0 scale bytes
 * (exponent + 127) of a (per 128-row half of each 256-row output tile) and b
 * (per 192-row output tile), each per 128-wide K chunk in 512-byte chunks of
 * 128 rows x 4 blocks: row r, block kb at (r % 32) * 16 + ((r % 128) / 32) * 4
 * + kb % 4. */
int trimul_mxfp8_views(const trimul_params *p, void **aq, void **bq, void **sa, void **sb, size_t *ldq);

/* ---- Backward -------------------------------------------------------------
 * Gradients of a loss L through one forward call. Given dout = dL/dout
 * ([N][N][c_z], dtype of z), trimul_backward writes dz = dL/dz ([N][N][c_z],
 * dtype of z) and, into the fp32 buffers of trimul_grads, dL/d(each weight,
 * bias and LayerNorm affine), overwriting them. The mask is an input and gets
 * no gradient. A parameter that trimul_params leaves NULL (bias 0, gamma 1,
 * beta 0) still gets its gradient when its output pointer is set; a NULL output
 * pointer skips that gradient.
 *
 * The forward intermediates are recomputed (unless g->flags has
 * TRIMUL_BWD_REUSE_FORWARD): the call enqueues the prologue and the
 * contraction into p->workspace, then the backward steps, which keep their
 * intermediates (bf16, with fp32 for the LayerNorm adjoints' inputs) in
 * g->workspace. The contraction's adjoint (per channel dA_c = dX_c B_c and
 * dB_c = dX_c^T A_c outgoing, dA_c = B_c dX_c^T and dB_c = A_c dX_c incoming)
 * runs on the forward's tcgen05 contraction kernel with the operands in other
 * transposes, and so do the plain GEMMs (projections, weight gradients) as
 * batched rectangular products with fp32 accumulation; the LayerNorm, gate and
 * mask adjoints run in the library's own per-cell kernels. No vendor library
 * is called. Weight gradients are summed per chunk of 4096 cells by GEMM and
 * over the chunks in double, so they are deterministic; bias and LayerNorm
 * gradients are fp32 sums (atomic, so their last bits may vary between runs).
 *
 * BF16 only in this version (TRIMUL_ERR_UNSUPPORTED for F32). dout and dz
 * must be 16-byte aligned and must not overlap each other, z, the mask or
 * either workspace. Asynchronous. */
typedef struct {
    float *d_w_a, *d_w_ag, *d_w_b, *d_w_bg; /* [c_h][c_z] */
    float *d_w_g;                           /* [c_z][c_z] */
    float *d_w_o;                           /* [c_z][c_h] */
    float *d_b_a, *d_b_ag, *d_b_b, *d_b_bg; /* [c_h] */
    float *d_b_g, *d_b_o;                   /* [c_z] */
    float *d_ln_in_w, *d_ln_in_b;           /* [c_z] */
    float *d_ln_out_w, *d_ln_out_b;         /* [c_h] */
    void *workspace;                        /* device memory, 256-byte aligned */
    size_t workspace_bytes;                 /* >= trimul_backward_workspace_size_rows(.., 1) */
    uint32_t flags;                         /* TRIMUL_BWD_*; 0 = recompute the forward */
} trimul_grads;

/* trimul_grads.flags: p->workspace still holds the a, b and x that the last
 * trimul_forward(z, mask, p, direction, ...) left there (same z, mask, weights,
 * direction and workspace, nothing written to the workspace since), so the
 * backward skips recomputing them. With any of that not true the gradients are
 * wrong; no check is made. */
#define TRIMUL_BWD_REUSE_FORWARD 0x1u

/* Bytes of backward workspace (trimul_grads.workspace) for N: with this much
 * the per-cell intermediates of the whole grid fit at once (about 5 KB per
 * cell at c_z = c_h = 128). */
size_t trimul_backward_workspace_size(int N, int c_z, int c_h);

/* Bytes of backward workspace when the per-cell steps run over blocks of
 * `rows` rows (1 <= rows <= N; 0 for an invalid argument). trimul_backward
 * takes whatever workspace it is given, at least this for rows = 1, and uses
 * the largest block of rows that fits: the per-cell intermediates then take
 * about 4.1 KB per cell of one block, beside about 1 KB per cell of the whole
 * grid (dL/dx, dL/da and dL/db channel-major, dP_g) and the weight-gradient
 * partials (96 B per cell). Blocks smaller than the grid cost a second
 * LayerNorm and projection of each block's z; the result of every cell is
 * computed the same way, so dz is the same bit for bit and the parameter
 * gradients differ only in the order of their fp32 sums. */
size_t trimul_backward_workspace_size_rows(int N, int c_z, int c_h, int rows);

/* The block of rows trimul_backward uses with a workspace of workspace_bytes:
 * N when the whole grid fits, else the largest block that fits, 0 when none
 * does (the call then returns TRIMUL_ERR_WORKSPACE) or for an invalid size.
 * Host only. */
int trimul_backward_block_rows(int N, int c_z, int c_h, size_t workspace_bytes);

int trimul_backward(const void *z, const void *mask, const trimul_params *p, int direction, const void *dout,
                    void *dz, const trimul_grads *g, trimul_stream_t stream);

/* Library version (major * 100 + minor). */
int trimul_version(void);

#ifdef __cplusplus
}
#endif

#endif /* TRIMUL_B200_H */

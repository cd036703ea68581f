/*
 * atomattn.h - C ABI of sequence-local (windowed) atom attention on B200 (sm_100a).
 *
 * The pages ("Scaling biomolecular modeling with context parallelism in NVIDIA
 * BioNeMo", section "Efficient sequence-local atom attention") describe
 * AlphaFold3's atom attention as limited to local windows of 32 queries by 128
 * keys, the stacked windows computed as one batched attention. This library
 * computes the attention core of that step:
 *
 *   window w holds the query atoms 32w .. 32w + 31 and the key atoms
 *   32w - 48 .. 32w + 79 (key slot s = atom 32w - 48 + s, s in [0, 128));
 *   for each batch element, head h and query atom i of window w:
 *     l_s   = q_i . k_s / sqrt(32) + bias[w][h][i - 32w][s]     (valid slots s)
 *     out_i = sum_s softmax(l)_s v_s
 *   a slot is valid when its atom lies in [0, n_atoms) and its atom_mask is not
 *   0; a query with no valid slot gets 0.
 *
 * The projections, gating and output projection around this core are per-atom
 * Linear layers and not part of the library.
 *
 * Layouts (row-major, contiguous, bf16):
 *   q, k, v, out  [batch][n_atoms][heads][32]
 *   bias          [batch][ceil(n_atoms / 32)][heads][32][128], or NULL (no bias)
 *   atom_mask     [batch][n_atoms], or NULL (all atoms valid keys)
 * q, k, v, out and bias must be 16-byte aligned, atom_mask 2-byte aligned; out
 * must not overlap any input or the workspace.
 *
 * Ownership, threading and errors follow trimul.h: the caller owns every
 * buffer, the call enqueues on `stream` and returns TRIMUL_OK or a negative
 * trimul_status; argument errors are found on the host; a bounded in-kernel
 * wait that runs out is recorded in the workspace's status word
 * (atomattn_device_status). Computed on tcgen05 tensor cores (bf16 operands,
 * fp32 logits, softmax and accumulation; the probabilities enter the second
 * product as bf16).
 */
#ifndef ATOMATTN_B200_H
#define ATOMATTN_B200_H

#include "trimul.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct atomattn_params {
    int batch;        /* >= 1 */
    int n_atoms;      /* >= 1 */
    int heads;        /* 1 .. 64; batch * heads * ceil(n_atoms / 128) < 2^31 */
    int head_dim;     /* must be 32 */
    const void *q, *k, *v;
    const void *bias;       /* or NULL */
    const void *atom_mask;  /* or NULL */
    void *workspace;        /* device memory, 256-byte aligned, >= atomattn_workspace_size() */
    size_t workspace_bytes;
    uint32_t timeout_ms;    /* bound on each in-kernel wait; 0 = 2000 ms */
} atomattn_params;

/* Bytes of workspace (the device status word). */
size_t atomattn_workspace_size(void);

int atomattn_forward(const atomattn_params *p, void *out, trimul_stream_t stream);

/* Synchronises `stream`, then reads the status word: TRIMUL_OK, TRIMUL_ERR_TIMEOUT
 * or TRIMUL_ERR_DEVICE; detail[4] (optional) receives code, site, block, aux. */
int atomattn_device_status(const atomattn_params *p, trimul_stream_t stream, int *detail);

#ifdef __cplusplus
}
#endif

#endif /* ATOMATTN_B200_H */

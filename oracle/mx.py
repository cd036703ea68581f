"""CPU float64 oracle for an MXFP8 triangle contraction (test infrastructure).

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: imported by ``tests/``;
the product path never imports or runs it.

The pages list MXFP8 among the Blackwell training precisions ("Scaling
biomolecular modeling with context parallelism in NVIDIA BioNeMo", the
precision list of the BioNeMo recipes) without defining it. The definition
taken here is the public OCP Microscaling Formats (MX) specification v1.0:

  * a block of 32 values shares one scale X = 2^e (E8M0: e in [-127, 127]);
  * each value is stored as an FP8 E4M3 element P_i (1 sign, 4 exponent bits
    with bias 7, 3 mantissa bits; largest normal 448, smallest normal 2^-6,
    subnormals down to 2^-9, no infinities);
  * conversion of a block V: e = floor(log2(max |V_i|)) - 8 (8 = the exponent
    of E4M3's largest normal), X = 2^e, P_i = V_i / X rounded to nearest (ties
    to even) and saturated to +-448; an all-zero block takes the smallest scale
    and zero elements;
  * the value of element i is X * P_i.

For the contraction the blocks run along the contracted index k: outgoing
x_ij = sum_k a_ik b_jk blocks a along k for each (i, channel) and b along k
for each (j, channel); incoming x_ij = sum_k a_ki b_kj blocks along k (the
first index) likewise. A last block shorter than 32 (N not a multiple of 32)
is a block of its own. The contraction of the dequantised operands is then
exact in float64 (E4M3 products have at most 8 significant bits).
"""
from __future__ import annotations

import numpy as np

BLOCK = 32
E4M3_MAX = 448.0
E4M3_EMAX = 8            # exponent of the largest normal
E4M3_EMIN = -6           # exponent of the smallest normal
E4M3_MANT = 3
SCALE_EMIN, SCALE_EMAX = -127, 127


def e4m3_round(x):
    """Round to the nearest E4M3 value (ties to even), saturating at +-448."""
    x = np.asarray(x, dtype=np.float64)
    ax = np.abs(x)
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    e = np.maximum(e, E4M3_EMIN)                      # subnormals share the quantum of the smallest binade
    quantum = np.exp2(e - E4M3_MANT)
    r = np.rint(ax / quantum) * quantum               # rint: ties to even
    r = np.minimum(r, E4M3_MAX)
    return np.copysign(r, x)


def mx_quantize_blocks(v, axis):
    """MXFP8 conversion of v in blocks of 32 along `axis`.

    Returns (elements P as float64 E4M3 values, scale exponents e per block,
    dequantised values X * P), the exponent array having v's shape with `axis`
    replaced by the number of blocks.
    """
    v = np.moveaxis(np.asarray(v, dtype=np.float64), axis, -1)
    n = v.shape[-1]
    nb = (n + BLOCK - 1) // BLOCK
    pad = nb * BLOCK - n
    vp = np.concatenate([v, np.zeros(v.shape[:-1] + (pad,))], axis=-1) if pad else v
    blocks = vp.reshape(v.shape[:-1] + (nb, BLOCK))
    amax = np.abs(blocks).max(axis=-1)
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(amax > 0, amax, 1.0))) - E4M3_EMAX
    e = np.where(amax > 0, e, SCALE_EMIN)
    e = np.clip(e, SCALE_EMIN, SCALE_EMAX)
    X = np.exp2(e)[..., None]
    P = e4m3_round(blocks / X)
    deq = (P * X).reshape(vp.shape)[..., :n]
    P = P.reshape(vp.shape)[..., :n]
    return np.moveaxis(P, -1, axis), np.moveaxis(e, -1, axis), np.moveaxis(deq, -1, axis)


def mx_contract(a, b, direction):
    """x [N][N][c] from a, b [N][N][c] quantised to MXFP8 along the contracted index.

    outgoing: x_ij = sum_k A_ik B_jk, blocks of a and b along their second index;
    incoming: x_ij = sum_k A_ki B_kj, blocks along their first index.
    """
    incoming = direction in ("incoming", 1)
    axis = 0 if incoming else 1
    _, _, aq = mx_quantize_blocks(a, axis)
    _, _, bq = mx_quantize_blocks(b, axis)
    if incoming:
        return np.einsum("kic,kjc->ijc", aq, bq)
    return np.einsum("ikc,jkc->ijc", aq, bq)


def mx_contract_grid(a, b, direction, I):
    """The MXFP8 contraction on the cells I x I only: x [len(I)][len(I)][c].

    The operands are quantised in full (blocks along k need every k), then only
    the rows (outgoing) or columns (incoming) of the sampled residues are
    contracted, exactly as mx_contract would for those cells.
    """
    incoming = direction in ("incoming", 1)
    axis = 0 if incoming else 1
    I = np.asarray(I)
    _, _, aq = mx_quantize_blocks(a, axis)
    _, _, bq = mx_quantize_blocks(b, axis)
    if incoming:
        return np.einsum("kic,kjc->ijc", aq[:, I], bq[:, I])
    return np.einsum("ikc,jkc->ijc", aq[I], bq[I])

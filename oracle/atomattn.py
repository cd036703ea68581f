"""CPU float64 oracle for sequence-local (windowed) atom attention (test infrastructure).

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: imported by ``tests/``
and by ``bench.py``'s CPU timing leg; the product path never imports or runs it.

The pages ("Scaling biomolecular modeling with context parallelism in NVIDIA
BioNeMo", section "Efficient sequence-local atom attention") state only that
AlphaFold3 limits atom attention to local windows of 32 by 128 and computes
the stacked windows as one batched attention. Readings taken here (each the
plainest one that agrees with that statement):

  * atoms form one sequence per batch element; queries are split into
    consecutive windows of 32 (window w holds atoms 32w .. 32w + 31, the last
    window may be short);
  * window w attends to the 128 keys centred on it, atoms
    32w + 16 - 64 .. 32w + 16 + 63, i.e. 32w - 48 .. 32w + 79; keys outside
    [0, n_atoms) or with atom_mask 0 take no part;
  * multi-head attention on projected q, k, v ([batch][atom][head][d]) with
    logits q.k / sqrt(d) plus an optional additive bias per window, head,
    query and key slot ([batch][window][head][32][128]; key slot s is atom
    32w - 48 + s), softmax over the window's keys, output sum_k p v;
  * a query with no valid key gets a zero output.

The projections, gating and output projection around the attention core are
plain per-atom Linear layers and are not part of this path.
"""
from __future__ import annotations

import numpy as np

Q_WIN, K_WIN = 32, 128
K_OFFSET = (Q_WIN - K_WIN) // 2  # first key of window w is 32 w - 48


def key_range(w: int):
    """[first, last) atom indices of window w's key slots (may leave [0, n))."""
    k0 = Q_WIN * w + K_OFFSET
    return k0, k0 + K_WIN


def n_windows(n_atoms: int) -> int:
    return (n_atoms + Q_WIN - 1) // Q_WIN


def atom_attention(q, k, v, bias=None, atom_mask=None):
    """Windowed attention, float64.

    q, k, v: [batch][n_atoms][heads][d]; bias: [batch][n_windows][heads][32][128]
    or None; atom_mask: [batch][n_atoms] or None. Returns [batch][n_atoms][heads][d].
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, n, H, d = q.shape
    out = np.zeros_like(q)
    scale = 1.0 / np.sqrt(d)
    for b in range(B):
        for w in range(n_windows(n)):
            q0, q1 = Q_WIN * w, min(Q_WIN * (w + 1), n)
            k0, k1 = key_range(w)
            slots = np.arange(k0, k1)
            valid = (slots >= 0) & (slots < n)
            if atom_mask is not None:
                m = np.zeros(K_WIN, dtype=bool)
                m[valid] = np.asarray(atom_mask[b])[slots[valid]] != 0
                valid = m
            if not valid.any():
                continue
            ks, vs = k[b, slots[valid]], v[b, slots[valid]]          # [nk][H][d]
            logits = np.einsum("qhd,khd->hqk", q[b, q0:q1], ks) * scale  # [H][nq][nk]
            if bias is not None:
                bw = np.asarray(bias[b, w], dtype=np.float64)          # [H][32][128]
                logits = logits + bw[:, : q1 - q0][:, :, valid]
            logits -= logits.max(axis=-1, keepdims=True)
            p = np.exp(logits)
            p /= p.sum(axis=-1, keepdims=True)
            out[b, q0:q1] = np.einsum("hqk,khd->qhd", p, vs)
    return out

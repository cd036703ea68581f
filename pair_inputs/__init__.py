"""Seeded synthetic inputs for the triangle multiplicative update.

This module is the only code shared by the CPU oracle and the GPU path. It
draws random numbers and lays them out; it holds none of the layer's
arithmetic (no LayerNorm, projection, gating or contraction).

Workloads follow the shapes the pages name for the pair representation
("Scaling biomolecular modeling with context parallelism in NVIDIA BioNeMo":
the Boltz-2 training crop of 768 residues and the 3,605-residue four-chain
complex, both in the section on unlocking token scaling). The pages' own
structures, MSAs and trained weights are not used; every tensor here is a
seeded stand-in with the stated distribution.

Recipe (per workload, base seed ``s``):
  * z[i] (one residue row, shape [N, c_z]) ~ N(0, 1) from
    ``default_rng([s, 0, i])`` in float32, so rows can be drawn in parallel
    or on demand. With ``channel_scale`` each channel c is then multiplied
    by s_c ~ U(0.5, 2) drawn from ``default_rng([s, 1])``.
  * Weights W_a, W_ag, W_b, W_bg, W_g, W_o (PyTorch Linear layout
    [out][in]) ~ N(0, 1/c_in) from ``default_rng([s, 2, k])`` for k = 0..5.
  * Optional random LayerNorm affines and biases (used by pin tests only)
    from ``default_rng([s, 3, k])``.
  * mask[i][j] = m_i * m_j with m_i = 1 for residues i < n_valid, else 0.
  * bf16 workloads round every drawn value to bfloat16 (round to nearest
    even) and keep it in float32 storage, so both sides see identical,
    exactly representable inputs.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

WEIGHT_NAMES = ("w_a", "w_ag", "w_b", "w_bg", "w_g", "w_o")
BIAS_NAMES = ("b_a", "b_ag", "b_b", "b_bg", "b_g", "b_o")
LN_NAMES = ("ln_in_w", "ln_in_b", "ln_out_w", "ln_out_b")


@dataclass(frozen=True)
class Workload:
    """One synthetic workload: sizes, precision, mask and seed."""

    name: str
    N: int
    dtype: str  # "f32" or "bf16"
    directions: tuple
    n_valid: int  # residues [0, n_valid) have m_i = 1
    seed: int
    channel_scale: bool = False
    c_z: int = 128
    c_h: int = 128
    chains: tuple = field(default=())

    @property
    def cells(self) -> int:
        return self.N * self.N


# The five workloads. Seeds are the workload index minus one.
WORKLOADS = {
    1: Workload("tiny_fp32_N64", 64, "f32", ("outgoing",), 64, 0),
    2: Workload("padded_bf16_N384", 384, "bf16", ("outgoing", "incoming"), 384 - 38, 1),
    3: Workload("crop768_bf16", 768, "bf16", ("outgoing", "incoming"), 768, 2,
                channel_scale=True, chains=(500, 268)),
    4: Workload("complex2048_bf16", 2048, "bf16", ("outgoing", "incoming"), 2000, 3,
                chains=(900, 700, 400)),
    5: Workload("complex3605_bf16", 3605, "bf16", ("outgoing", "incoming"), 3605, 4,
                chains=(1900, 1100, 482, 123)),
}


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even), in place.

    Works on the bit pattern: add 0x7FFF plus the lowest kept bit, then clear
    the 16 discarded bits. Inputs here are finite.
    """
    u = x.view(np.uint32)
    u += np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    u &= np.uint32(0xFFFF0000)
    return x


def _threads() -> int:
    return max(1, min(16, os.cpu_count() or 1))


def draw_z(N: int, c: int, seed: int, channel_scale: bool = False, bf16: bool = False,
           rows=None) -> np.ndarray:
    """Draw z (float32, [len(rows) or N][N][c]) row by row from per-row streams."""
    rows = list(range(N)) if rows is None else list(rows)
    z = np.empty((len(rows), N, c), dtype=np.float32)
    scale = None
    if channel_scale:
        scale = np.random.default_rng([seed, 1]).uniform(0.5, 2.0, size=c).astype(np.float32)

    def one(t):
        i = rows[t]
        np.random.default_rng([seed, 0, i]).standard_normal((N, c), dtype=np.float32, out=z[t])
        if scale is not None:
            z[t] *= scale
        if bf16:
            round_bf16(z[t])

    if len(rows) > 8:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(one, range(len(rows))))
    else:
        for t in range(len(rows)):
            one(t)
    return z


def draw_weights(c_z: int, c_h: int, seed: int, bf16: bool = False) -> dict:
    """Draw the six Linear weights ([out][in], N(0, 1/c_in)) as float32."""
    shapes = {"w_a": (c_h, c_z), "w_ag": (c_h, c_z), "w_b": (c_h, c_z), "w_bg": (c_h, c_z),
              "w_g": (c_z, c_z), "w_o": (c_z, c_h)}
    out = {}
    for k, name in enumerate(WEIGHT_NAMES):
        shp = shapes[name]
        w = np.random.default_rng([seed, 2, k]).standard_normal(shp, dtype=np.float32)
        w *= np.float32(1.0 / np.sqrt(shp[1]))
        out[name] = round_bf16(w) if bf16 else w
    return out


def draw_affines(c_z: int, c_h: int, seed: int, bf16: bool = False) -> dict:
    """Random LayerNorm affines and biases (pin tests only; workloads use none)."""
    sizes = {"ln_in_w": c_z, "ln_in_b": c_z, "ln_out_w": c_h, "ln_out_b": c_h,
             "b_a": c_h, "b_ag": c_h, "b_b": c_h, "b_bg": c_h, "b_g": c_z, "b_o": c_z}
    out = {}
    for k, name in enumerate(LN_NAMES + BIAS_NAMES):
        rng = np.random.default_rng([seed, 3, k])
        if name in ("ln_in_w", "ln_out_w"):
            v = rng.uniform(0.5, 1.5, size=sizes[name]).astype(np.float32)
        else:
            v = (0.5 * rng.standard_normal(sizes[name])).astype(np.float32)
        out[name] = round_bf16(v) if bf16 else v
    return out


def residue_mask(N: int, n_valid: int) -> np.ndarray:
    """m_i: 1 for residues below n_valid, 0 for the padded tail."""
    m = np.zeros(N, dtype=np.float32)
    m[:n_valid] = 1.0
    return m


def pair_mask(m: np.ndarray) -> np.ndarray:
    """mask[i][j] = m_i * m_j as a float32 [N][N] array."""
    return np.multiply.outer(m, m).astype(np.float32)


def random_pair_mask(N: int, seed: int, p_zero: float = 0.2) -> np.ndarray:
    """A mask with independent 0/1 entries (pin tests and edge cases)."""
    rng = np.random.default_rng([seed, 4])
    return (rng.uniform(size=(N, N)) >= p_zero).astype(np.float32)


def make_workload(w: Workload, affine: bool = False, with_z: bool = True) -> dict:
    """All inputs of a workload as float32 numpy arrays.

    Keys: z [N][N][c_z] (omitted when with_z is False), mask [N][N], m [N],
    the six weights, and (when ``affine``) LayerNorm affines and biases.
    """
    bf16 = w.dtype == "bf16"
    d = {}
    if with_z:
        d["z"] = draw_z(w.N, w.c_z, w.seed, w.channel_scale, bf16)
    d["m"] = residue_mask(w.N, w.n_valid)
    d["mask"] = pair_mask(d["m"])
    d.update(draw_weights(w.c_z, w.c_h, w.seed, bf16))
    if affine:
        d.update(draw_affines(w.c_z, w.c_h, w.seed, bf16))
    return d


def random_case(N: int, seed: int, c_z: int = 128, c_h: int = 128, bf16: bool = False,
                affine: bool = True, mask: str = "random") -> dict:
    """A small random case for edge tests: any N, random mask and affines."""
    d = {"z": draw_z(N, c_z, seed, False, bf16)}
    if mask == "random":
        d["mask"] = random_pair_mask(N, seed)
    elif mask == "ones":
        d["mask"] = np.ones((N, N), dtype=np.float32)
    elif mask == "zeros":
        d["mask"] = np.zeros((N, N), dtype=np.float32)
    else:
        raise ValueError(mask)
    d.update(draw_weights(c_z, c_h, seed, bf16))
    if affine:
        d.update(draw_affines(c_z, c_h, seed, bf16))
    return d


def sample_grid(N: int, seed: int, n_random: int = 24, tile: int = 128, pair_tile: int = 256) -> np.ndarray:
    """Sorted residue indices for a sampled check: tile edges, ragged tail, random.

    Used on both axes, so the sampled cells are the grid I x I: corners, the
    first two 128-tile boundaries and those near the end, every boundary of a
    256-wide pair tile (255/256, 511/512, 767/768, ...), the last (ragged)
    tile, and random rows.
    """
    s = {0, 1, N - 2, N - 1}
    for t in range(tile, N, tile):
        if t in (tile, 2 * tile) or t >= N - tile or t % pair_tile == 0:
            s.update((t - 1, t))
    last_tile = (N - 1) // tile * tile
    s.update((last_tile, min(N - 1, last_tile + 1)))
    rng = np.random.default_rng([seed, 5])
    s.update(int(v) for v in rng.integers(0, N, size=n_random))
    return np.array(sorted(v for v in s if 0 <= v < N), dtype=np.int32)

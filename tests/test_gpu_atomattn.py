"""GPU parity of windowed atom attention (atomattn_forward, through the C ABI)
against the float64 oracle (oracle/atomattn.py).

Bars: rel-L2 <= 1e-2 and max-abs <= 3e-2 on the output. Derivation: the
outputs are convex combinations of v (|v| of order 1, here N(0, 1)); the path
rounds the probabilities (relative 2^-8 at most, independent per key) and the
output (2^-8 relative) to bf16 and computes logits and sums in fp32, so the
error is about 2^-8 |out| from the output rounding plus a random-sign sum of
the probability roundings, well under 1e-2 of the norm; max-abs allows 2^-8
of the largest |out| (about 4) with a factor of 2 for the probability term.
"""
import numpy as np
import pytest
import torch

import pair_representation_b200 as tm
from gpu_helpers import as_bf16, max_abs, rel_l2
from oracle.atomattn import atom_attention as oracle_attention

pytestmark = pytest.mark.gpu

REL, ABS = 1e-2, 3e-2


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from pair_representation_b200 import build
    build.build()
    tm.lib()


def draw(B, n, H, seed, bias=True, mask="tail"):
    rng = np.random.default_rng([seed, 21])
    q, k, v = (as_bf16(rng.standard_normal((B, n, H, 32))) for _ in range(3))
    b = as_bf16(rng.standard_normal((B, (n + 31) // 32, H, 32, 128))) if bias else None
    m = None
    if mask == "tail":
        m = np.ones((B, n), dtype=np.float32)
        m[:, n - max(1, n // 20):] = 0
        m[:, rng.integers(0, n, size=max(1, n // 50))] = 0
    elif mask == "zeros":
        m = np.zeros((B, n), dtype=np.float32)
    return q, k, v, b, m


def run(q, k, v, b, m):
    dev = torch.device("cuda", 0)
    t = lambda a: None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(dev).to(torch.bfloat16)
    out, p = tm.atom_attention(t(q), t(k), t(v), t(b), t(m))
    torch.cuda.synchronize()
    rc, detail = tm.atomattn_device_status(p)
    assert rc == 0, (rc, detail)
    return out.double().cpu().numpy()


@pytest.mark.parametrize("B,n,H", [(1, 1, 2), (1, 32, 2), (2, 100, 4), (1, 128, 4), (1, 129, 2), (2, 257, 4),
                                   (3, 300, 2), (1, 1000, 6), (1, 100, 1), (2, 257, 3), (1, 300, 5)])
def test_atomattn_parity(B, n, H):
    q, k, v, b, m = draw(B, n, H, seed=n + 7 * H)
    got = run(q, k, v, b, m)
    ref = oracle_attention(q, k, v, b, m)
    assert np.isfinite(got).all()
    assert rel_l2(got, ref) <= REL, rel_l2(got, ref)
    assert max_abs(got, ref) <= ABS, max_abs(got, ref)


def test_atomattn_without_bias_or_mask():
    q, k, v, _, _ = draw(2, 333, 4, seed=3, bias=False, mask=None)
    got = run(q, k, v, None, None)
    ref = oracle_attention(q, k, v)
    assert rel_l2(got, ref) <= REL and max_abs(got, ref) <= ABS


def test_atomattn_zero_mask_gives_zero():
    q, k, v, b, m = draw(1, 200, 2, seed=4, mask="zeros")
    got = run(q, k, v, b, m)
    assert np.abs(got).max() == 0.0


def test_atomattn_full_size():
    """The benchmark's shape (8 x 18432 atoms, 4 heads), every output against the oracle."""
    q, k, v, b, m = draw(8, 18432, 4, seed=5)
    got = run(q, k, v, b, m)
    ref = oracle_attention(q, k, v, b, m)
    assert rel_l2(got, ref) <= REL and max_abs(got, ref) <= ABS

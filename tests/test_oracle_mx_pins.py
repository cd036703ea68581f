"""Pins for the MXFP8 oracle (oracle/mx.py), CPU only.

Checked against things other than the oracle itself:
  * E4M3 rounding against the value set decoded from all 256 bit patterns by
    the format's definition (brute force: nearest value, ties to the even
    mantissa, saturation at 448, sign symmetry);
  * the block scale rule on closed forms (powers of two, 448-scaled blocks,
    zero blocks, a lone subnormal-range value);
  * blocks of 32 along the contracted index, including a short last block;
  * the contraction equals numpy matmul of the dequantised operands per
    channel, and stays within the format's error bound of the exact product;
  * planted mistakes (scale off by one, blocks along the wrong axis) fail.
"""
import numpy as np
import pytest

from oracle.mx import BLOCK, e4m3_round, mx_contract, mx_contract_grid, mx_quantize_blocks


def e4m3_values():
    """All finite E4M3 values, decoded from the 8-bit patterns (S EEEE MMM, bias 7; S.1111.111 is NaN)."""
    vals = []
    for code in range(256):
        s, e, m = code >> 7, (code >> 3) & 15, code & 7
        if e == 15 and m == 7:
            continue  # NaN
        v = (m / 8.0) * 2.0 ** -6 if e == 0 else (1 + m / 8.0) * 2.0 ** (e - 7)
        vals.append((-v if s else v, m))
    return vals


def nearest_even(x, table):
    """Nearest value in the table; on a tie, the one with even mantissa field."""
    best = None
    for v, m in table:
        d = abs(v - x)
        if best is None or d < best[0] - 1e-300 or (abs(d - best[0]) <= 1e-300 and m % 2 == 0 and best[2] % 2 == 1):
            best = (d, v, m)
    return best[1]


def test_e4m3_value_set():
    vals = sorted({v for v, _ in e4m3_values()})
    assert max(vals) == 448.0 and min(vals) == -448.0
    pos = [v for v in vals if v > 0]
    assert min(pos) == 2.0 ** -9 and len(pos) == 126
    for v in vals:
        assert e4m3_round(v) == v


def test_e4m3_rounding_brute_force():
    table = e4m3_values()
    vals = sorted({v for v, _ in table})
    rng = np.random.default_rng(1)
    xs = list(rng.uniform(-440, 440, 400)) + list(rng.standard_normal(400) * 0.05)
    xs += [(a + b) / 2 for a, b in zip(vals[:-1], vals[1:])]  # every midpoint: a tie
    for x in xs:
        assert e4m3_round(x) == nearest_even(x, table), x


def test_e4m3_saturates():
    for x in (448.0, 464.0, 480.0, 1e6):
        assert e4m3_round(x) == 448.0 and e4m3_round(-x) == -448.0


def test_block_scale_closed_forms():
    # amax 1 -> e = -8, X = 2^-8, the 1 maps to 256 (exact in E4M3).
    v = np.zeros(32)
    v[5] = 1.0
    P, e, deq = mx_quantize_blocks(v, 0)
    assert e[0] == -8 and P[5] == 256.0 and deq[5] == 1.0
    # amax 448 * 2^3 -> e = floor(log2(3584)) - 8 = 3, element 448.
    v = np.full(32, 0.5)
    v[0] = 448.0 * 8
    P, e, deq = mx_quantize_blocks(v, 0)
    assert e[0] == 3 and P[0] == 448.0 and deq[0] == 3584.0
    assert deq[1] == e4m3_round(0.5 / 8) * 8
    # amax just below the next power of two: 511 -> e = 0, elements saturate at 448.
    v = np.full(32, 511.0)
    P, e, _ = mx_quantize_blocks(v, 0)
    assert e[0] == 0 and np.all(P == 448.0)
    # zero block
    P, e, deq = mx_quantize_blocks(np.zeros(32), 0)
    assert np.all(P == 0) and np.all(deq == 0) and e[0] == -127


def test_blocks_follow_the_axis_and_short_tail():
    rng = np.random.default_rng(2)
    v = rng.standard_normal((3, 70))
    v[1, 64:] *= 1000.0                     # the short last block (6 values) has its own scale
    _, e, deq = mx_quantize_blocks(v, 1)
    assert e.shape == (3, 3)
    assert e[1, 2] > e[1, 1] + 5
    # each block alone gives the same result
    for r in range(3):
        for blk in range(3):
            lo, hi = blk * BLOCK, min((blk + 1) * BLOCK, 70)
            _, e1, d1 = mx_quantize_blocks(v[r, lo:hi], 0)
            assert e1[0] == e[r, blk] and np.array_equal(d1, deq[r, lo:hi])


@pytest.mark.parametrize("direction", ["outgoing", "incoming"])
def test_contraction_is_matmul_of_dequantised(direction):
    N = 70
    rng = np.random.default_rng(3)
    a = rng.standard_normal((N, N, 4)) * np.exp(rng.uniform(-3, 3, (N, N, 1)))
    b = rng.standard_normal((N, N, 4))
    x = mx_contract(a, b, direction)
    axis = 0 if direction == "incoming" else 1
    aq = mx_quantize_blocks(a, axis)[2]
    bq = mx_quantize_blocks(b, axis)[2]
    for c in range(4):
        ref = aq[:, :, c].T @ bq[:, :, c] if direction == "incoming" else aq[:, :, c] @ bq[:, :, c].T
        np.testing.assert_allclose(x[:, :, c], ref, rtol=1e-12, atol=1e-12)
    # error bound against the exact product: each element within 1/8 relative (E4M3 rounding
    # 2^-4, saturation of the block maximum up to 1 - 448/512), plus 2^-9 X for subnormals.
    exact = np.einsum("kic,kjc->ijc", a, b) if direction == "incoming" else np.einsum("ikc,jkc->ijc", a, b)
    bound = np.einsum("kic,kjc->ijc", np.abs(a), np.abs(b)) if direction == "incoming" else \
        np.einsum("ikc,jkc->ijc", np.abs(a), np.abs(b))
    assert np.all(np.abs(x - exact) <= 0.27 * bound + 1e-9)


def test_planted_mistakes_fail():
    rng = np.random.default_rng(4)
    a = rng.standard_normal((64, 64, 2))
    b = rng.standard_normal((64, 64, 2))
    x = mx_contract(a, b, "outgoing")
    # blocks along the wrong axis give a different result
    aw = mx_quantize_blocks(a, 0)[2]
    bw = mx_quantize_blocks(b, 0)[2]
    wrong = np.einsum("ikc,jkc->ijc", aw, bw)
    assert np.abs(wrong - x).max() > 1e-6
    # a scale one binade too large loses resolution: no longer equal to the oracle's
    P, e, _ = mx_quantize_blocks(a, 1)
    Xb = np.exp2(np.repeat(e + 1, BLOCK, axis=1))[:, :64]
    coarse = e4m3_round(a / Xb) * Xb
    assert np.abs(coarse - mx_quantize_blocks(a, 1)[2]).max() > 0


@pytest.mark.parametrize("direction", ["outgoing", "incoming"])
def test_grid_mode_equals_full_contraction(direction):
    """mx_contract_grid on I x I is the full mx_contract restricted to I x I."""
    rng = np.random.default_rng(77)
    N = 45
    a = rng.standard_normal((N, N, 3)) * np.exp2(rng.integers(-6, 7, size=(N, 1, 3)))
    b = rng.standard_normal((N, N, 3))
    I = np.array([0, 3, 31, 32, 44])
    full = mx_contract(a, b, direction)
    np.testing.assert_array_equal(mx_contract_grid(a, b, direction, I), full[np.ix_(I, I)])

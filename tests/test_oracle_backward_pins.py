"""Pins for the float64 backward oracle (oracle/backward.py), CPU only.

The backward oracle is checked against something other than itself:
  * central differences of the C forward oracle (a separate implementation),
    with Richardson extrapolation; every input is drawn on a dyadic grid so
    that each perturbation is exact in the oracle's float32 inputs, which
    leaves the differences accurate to about 1e-10 relative;
  * the direction identity for gradients: incoming(z, mask; W_a, W_ag, W_b,
    W_bg) = outgoing(z^T, mask^T; W_b, W_bg, W_a, W_ag)^T, so the incoming
    gradients must equal the outgoing ones of the transposed problem with the
    a- and b-side weights swapped;
  * N = 1, where x = a * b cell by cell.
"""
import numpy as np
import pytest

import oracle
from oracle.backward import AFFINES, BIASES, WEIGHTS, trimul_backward

pytestmark = pytest.mark.filterwarnings("ignore")

GRID = {"z": 10, "w": 14, "v": 12}  # values are multiples of 2^-k


def _grid(x, k):
    return (np.round(np.asarray(x, dtype=np.float64) * 2.0 ** k) / 2.0 ** k).astype(np.float32)


def dyadic_case(N, seed, affine=True, mask="random"):
    rng = np.random.default_rng([seed, 77])
    c = 128
    case = {"z": _grid(rng.standard_normal((N, N, c)) * 1.5 + 0.3, GRID["z"])}
    for k in WEIGHTS:
        case[k] = _grid(rng.standard_normal((c, c)) / np.sqrt(c), GRID["w"])
    if affine:
        for k in BIASES:
            case[k] = _grid(rng.standard_normal(c) * 0.2, GRID["v"])
        case["ln_in_w"] = _grid(1.0 + 0.3 * rng.standard_normal(c), GRID["v"])
        case["ln_in_b"] = _grid(0.2 * rng.standard_normal(c), GRID["v"])
        case["ln_out_w"] = _grid(1.0 + 0.3 * rng.standard_normal(c), GRID["v"])
        case["ln_out_b"] = _grid(0.2 * rng.standard_normal(c), GRID["v"])
    if mask == "random":
        m = (rng.random((N, N)) < 0.8).astype(np.float32)
        m[0, 0] = 1.0
        case["mask"] = m
    elif mask == "ones":
        case["mask"] = np.ones((N, N), dtype=np.float32)
    return case


def _loss(case, direction, dout):
    return float((oracle.trimul(case, direction, threads=1) * dout).sum())


def _fd(case, direction, dout, name, idx, k):
    """Richardson-extrapolated central difference of the loss in case[name][idx]."""
    base = case[name]

    def at(delta):
        c2 = dict(case)
        v = base.copy()
        v[idx] = np.float32(np.float64(base[idx]) + delta)
        assert np.float64(v[idx]) == np.float64(base[idx]) + delta  # exact perturbation
        c2[name] = v
        return _loss(c2, direction, dout)

    h = 2.0 ** -k
    d1 = (at(h) - at(-h)) / (2 * h)
    d2 = (at(h / 2) - at(-h / 2)) / h
    return (4 * d2 - d1) / 3


def _check(case, direction, seed, n_pick):
    N = case["z"].shape[0]
    dout = np.random.default_rng([seed, 5]).standard_normal((N, N, 128))
    grads = trimul_backward(case, direction, dout)
    rng = np.random.default_rng([seed, 6])
    for name in ["z"] + list(WEIGHTS) + list(BIASES) + list(AFFINES):
        if name not in case:
            continue
        g = grads[name]
        k = GRID["z"] if name == "z" else GRID["w"] if name in WEIGHTS else GRID["v"]
        flat = rng.choice(g.size, size=min(n_pick, g.size), replace=False)
        scale = np.abs(g).max() + 1e-12
        for f in flat:
            idx = np.unravel_index(f, g.shape)
            fd = _fd(case, direction, dout, name, idx, k)
            assert abs(fd - g[idx]) <= 1e-7 * scale + 1e-9 * abs(fd), (direction, name, idx, fd, g[idx], scale)


@pytest.mark.parametrize("direction", ["outgoing", "incoming"])
def test_backward_matches_finite_differences(direction):
    case = dyadic_case(3, 11, affine=True, mask="random")
    _check(case, direction, 11, n_pick=6)


def test_backward_finite_differences_without_affines():
    """NULL biases and affines: gradients still defined (zeros / ones in the forward)."""
    case = dyadic_case(2, 12, affine=False, mask="ones")
    grads = trimul_backward(case, "outgoing", np.ones((2, 2, 128)))
    assert np.isfinite(grads["b_a"]).all() and np.isfinite(grads["ln_out_w"]).all()
    _check(case, "outgoing", 12, n_pick=4)


def test_backward_direction_identity():
    case = dyadic_case(4, 13, affine=True, mask="random")
    dout = np.random.default_rng(1).standard_normal((4, 4, 128))
    g_in = trimul_backward(case, "incoming", dout)
    t = dict(case)
    t["z"] = np.ascontiguousarray(case["z"].transpose(1, 0, 2))
    t["mask"] = np.ascontiguousarray(case["mask"].T)
    swap = {"w_a": "w_b", "w_ag": "w_bg", "w_b": "w_a", "w_bg": "w_ag",
            "b_a": "b_b", "b_ag": "b_bg", "b_b": "b_a", "b_bg": "b_ag"}
    for k, v in swap.items():
        t[k] = case[v]
    g_out = trimul_backward(t, "outgoing", dout.transpose(1, 0, 2))
    np.testing.assert_allclose(g_in["z"], g_out["z"].transpose(1, 0, 2), rtol=1e-10, atol=1e-12)
    for k in ("w_g", "w_o", "b_g", "b_o") + AFFINES:
        np.testing.assert_allclose(g_in[k], g_out[k], rtol=1e-10, atol=1e-12)
    for k, v in swap.items():
        np.testing.assert_allclose(g_in[k], g_out[v], rtol=1e-10, atol=1e-12)


def test_backward_n1_closed_form():
    """N = 1: x = a * b, so dL/dp_a = dx * m * sig(p_ag) * b and so on; checked through
    the weight gradient of W_a against the hand-derived chain for one cell."""
    case = dyadic_case(1, 14, affine=False, mask="ones")
    rng = np.random.default_rng(3)
    dout = rng.standard_normal((1, 1, 128))
    g = trimul_backward(case, "outgoing", dout)
    z = case["z"][0, 0].astype(np.float64)
    zh = (z - z.mean()) / np.sqrt(((z - z.mean()) ** 2).mean() + 1e-5)
    W = {k: case[k].astype(np.float64) for k in WEIGHTS}
    sig = lambda t: 1 / (1 + np.exp(-t))
    pa, pag, pb, pbg = (W[k] @ zh for k in ("w_a", "w_ag", "w_b", "w_bg"))
    a, b = sig(pag) * pa, sig(pbg) * pb
    x = a * b
    xh = (x - x.mean()) / np.sqrt(((x - x.mean()) ** 2).mean() + 1e-5)
    gg = sig(W["w_g"] @ zh)
    dy = dout[0, 0] * gg
    dxh = W["w_o"].T @ dy
    n = xh
    r = 1 / np.sqrt(((x - x.mean()) ** 2).mean() + 1e-5)
    dx = r * (dxh - dxh.mean() - n * (dxh * n).mean())
    dpa = dx * b * sig(pag)
    np.testing.assert_allclose(g["w_a"], np.outer(dpa, zh), rtol=1e-10, atol=1e-13)

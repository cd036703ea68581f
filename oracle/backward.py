"""CPU float64 gradients of the triangle multiplicative update (test infrastructure).

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: imported by ``tests/``
alone; the product path never imports or runs it.

For L = sum over cells and channels of out * dout, ``trimul_backward`` returns
dL/dz and dL/d(every weight, bias and LayerNorm affine) of the layer the pages
call TriangleMultiplicationOutgoing / TriangleMultiplicationIncoming ("Scaling
biomolecular modeling with context parallelism in NVIDIA BioNeMo", section
"Context-parallel implementation of triangle multiplication"). The mask is an
input, not a parameter, and gets no gradient.

The forward is restated step by step in numpy float64 (the same readings as the
C oracle: biased variance, eps inside the square root, mask on a and b at their
own cells, gate from the normalised z), and the gradients are taken by reverse
accumulation through those steps, in reverse order:

  forward                                   backward
  zh = LN_in(z)                             dz from dzh (LayerNorm rule)
  p_w = zh W_w^T + b_w, w in a,ag,b,bg      dW_w = sum dp_w (x) zh, dzh += dp_w W_w
  a = m sig(p_ag) p_a, b = m sig(p_bg) p_b  dp_a = da m sig(p_ag), dp_ag = da m p_a sig'(p_ag)
  x = contraction(a, b)                     da, db from dx (the contraction's adjoint)
  xh = LN_out(x)                            dx from dxh (LayerNorm rule)
  g = sig(zh W_g^T + b_g), y = xh W_o^T + b_o, out = g y
                                            dy = dout g, dg = dout y, ...

A parameter the case leaves out (a NULL bias or affine) is taken as zero (bias,
beta) or one (gamma), and its gradient is still returned.

Pinned in tests/test_oracle_backward_pins.py against central differences of the
C forward oracle (a separate implementation), on inputs drawn on a dyadic grid
so that every perturbation is exact in the oracle's float32 inputs.
"""
from __future__ import annotations

import numpy as np

WEIGHTS = ("w_a", "w_ag", "w_b", "w_bg", "w_g", "w_o")
BIASES = ("b_a", "b_ag", "b_b", "b_bg", "b_g", "b_o")
AFFINES = ("ln_in_w", "ln_in_b", "ln_out_w", "ln_out_b")


def _sig(t):
    return 1.0 / (1.0 + np.exp(-t))


def _ln_forward(v, gamma, beta, eps):
    """LayerNorm over the last axis: returns (out, normalised n, rstd r)."""
    mu = v.mean(axis=-1, keepdims=True)
    d = v - mu
    r = 1.0 / np.sqrt((d * d).mean(axis=-1, keepdims=True) + eps)
    n = d * r
    return n * gamma + beta, n, r


def _ln_backward(dout, n, r, gamma):
    """Adjoint of LayerNorm: returns (dv, dgamma, dbeta), sums over all leading axes."""
    dgamma = (dout * n).reshape(-1, n.shape[-1]).sum(axis=0)
    dbeta = dout.reshape(-1, n.shape[-1]).sum(axis=0)
    dn = dout * gamma
    dv = r * (dn - dn.mean(axis=-1, keepdims=True) - n * (dn * n).mean(axis=-1, keepdims=True))
    return dv, dgamma, dbeta


def _param(case, name, shape, default):
    v = case.get(name)
    return np.full(shape, default, dtype=np.float64) if v is None else np.asarray(v, dtype=np.float64)


def trimul_backward(case: dict, direction, dout, eps: float = 1e-5) -> dict:
    """Gradients of sum(out * dout) for one direction ("outgoing"/"incoming" or 0/1).

    Returns a dict with "z" ([N][N][c_z]) and every name of WEIGHTS, BIASES and
    AFFINES, all float64.
    """
    incoming = direction in ("incoming", 1)
    z = np.asarray(case["z"], dtype=np.float64)
    N, _, c_z = z.shape
    W = {k: np.asarray(case[k], dtype=np.float64) for k in WEIGHTS}
    c_h = W["w_a"].shape[0]
    B = {k: _param(case, k, (W["w" + k[1:]].shape[0],), 0.0) for k in BIASES}
    g_in, b_in = _param(case, "ln_in_w", (c_z,), 1.0), _param(case, "ln_in_b", (c_z,), 0.0)
    g_out, b_out = _param(case, "ln_out_w", (c_h,), 1.0), _param(case, "ln_out_b", (c_h,), 0.0)
    m = case.get("mask")
    m = np.ones((N, N), dtype=np.float64) if m is None else np.asarray(m, dtype=np.float64)
    m = m[:, :, None]
    dout = np.asarray(dout, dtype=np.float64)

    # ---- forward, keeping what the backward needs
    zh, n_in, r_in = _ln_forward(z, g_in, b_in, eps)
    p = {k: zh @ W["w" + k].T + B["b" + k] for k in ("_a", "_ag", "_b", "_bg")}
    s_a, s_b = _sig(p["_ag"]), _sig(p["_bg"])
    a = m * s_a * p["_a"]
    b = m * s_b * p["_b"]
    if incoming:
        x = np.einsum("kic,kjc->ijc", a, b)
    else:
        x = np.einsum("ikc,jkc->ijc", a, b)
    xh, n_out, r_out = _ln_forward(x, g_out, b_out, eps)
    g = _sig(zh @ W["w_g"].T + B["b_g"])
    y = xh @ W["w_o"].T + B["b_o"]

    grads = {}
    # ---- out = g * y
    dy = dout * g
    dg = dout * y
    grads["w_o"] = np.einsum("ijn,ijk->nk", dy, xh)
    grads["b_o"] = dy.sum(axis=(0, 1))
    dxh = dy @ W["w_o"]
    dpg = dg * g * (1.0 - g)
    grads["w_g"] = np.einsum("ijn,ijk->nk", dpg, zh)
    grads["b_g"] = dpg.sum(axis=(0, 1))
    dzh = dpg @ W["w_g"]
    # ---- xh = LN_out(x)
    dx, grads["ln_out_w"], grads["ln_out_b"] = _ln_backward(dxh, n_out, r_out, g_out)
    # ---- the contraction's adjoint
    if incoming:
        da = np.einsum("ijc,kjc->kic", dx, b)
        db = np.einsum("ijc,kic->kjc", dx, a)
    else:
        da = np.einsum("ijc,jkc->ikc", dx, b)
        db = np.einsum("ijc,ikc->jkc", dx, a)
    # ---- gating and mask
    dp = {
        "_a": da * m * s_a,
        "_ag": da * m * p["_a"] * s_a * (1.0 - s_a),
        "_b": db * m * s_b,
        "_bg": db * m * p["_b"] * s_b * (1.0 - s_b),
    }
    # ---- projections
    for k, d in dp.items():
        grads["w" + k] = np.einsum("ijn,ijk->nk", d, zh)
        grads["b" + k] = d.sum(axis=(0, 1))
        dzh = dzh + d @ W["w" + k]
    # ---- zh = LN_in(z)
    grads["z"], grads["ln_in_w"], grads["ln_in_b"] = _ln_backward(dzh, n_in, r_in, g_in)
    return grads

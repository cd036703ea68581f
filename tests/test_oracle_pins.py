"""Pins for the CPU oracle: facts the mathematics fixes, checked without the oracle's own code.

The pages print no worked example for the triangle multiplicative update, so
each pin is a closed form, an invariant, or a special case that reduces to a
library routine (torch's layer_norm / linear / sigmoid / matmul in float64).
Together they are chosen so that a plausible slip in the oracle fails at least
one of them:

  * wrong LayerNorm (unbiased variance, eps outside the root, missing affine)
      -> test_reduces_to_layer_norm_row_sums, test_single_cell_is_library_mlp
  * transposed weight, sigmoid of the wrong argument, gate on the wrong term
      -> test_single_cell_is_library_mlp, test_constant_z_closed_form
  * contraction over the wrong index / wrong transpose of b
      -> test_contraction_is_matmul, test_reduces_to_layer_norm_row_sums,
         test_transpose_identity_*
  * mask applied to the wrong cell, to g, or to the output
      -> test_zero_mask_closed_form, test_crop_invariance,
         test_reduces_to_layer_norm_row_sums (asymmetric random mask)
  * sum replaced by a mean
      -> test_constant_z_closed_form
  * row/column confusion in either direction
      -> test_permutation_equivariance, test_transpose_identity_*
  * sampled (grid) mode drifting from the full layer
      -> test_grid_matches_full
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import pair_inputs as pi

EPS = 1e-5
SAT = 40.0  # sigmoid(40) == 1.0 in double


def _t(a):
    return torch.from_numpy(np.asarray(a, dtype=np.float64))


def _ln(x, w=None, b=None):
    c = x.shape[-1]
    return F.layer_norm(x, (c,), None if w is None else _t(w), None if b is None else _t(b), EPS)


def _case(N, seed, c=128, mask="random", affine=True):
    return pi.random_case(N, seed, c_z=c, c_h=c, affine=affine, mask=mask)


def test_single_cell_is_library_mlp():
    """N = 1: x = a_11 (.) b_11, so the layer is a per-cell MLP of library modules."""
    for seed in range(3):
        d = _case(1, seed, mask="ones")
        z = _t(d["z"][0, 0])
        zh = _ln(z, d["ln_in_w"], d["ln_in_b"])
        lin = lambda x, w, b: F.linear(x, _t(d[w]), _t(d[b]))
        a = torch.sigmoid(lin(zh, "w_ag", "b_ag")) * lin(zh, "w_a", "b_a")
        b = torch.sigmoid(lin(zh, "w_bg", "b_bg")) * lin(zh, "w_b", "b_b")
        x = a * b
        expect = torch.sigmoid(lin(zh, "w_g", "b_g")) * lin(_ln(x, d["ln_out_w"], d["ln_out_b"]), "w_o", "b_o")
        for direction in ("outgoing", "incoming"):
            got = oracle.trimul(d, direction)[0, 0]
            np.testing.assert_allclose(got, expect.numpy(), rtol=1e-12, atol=1e-12)


def _identity_reduction_case(N, seed, c):
    """Weights that make a = mask*LN(z), b = mask, g = 1 and W_o = I."""
    d = _case(N, seed, c=c, mask="random")
    eye = np.eye(c, dtype=np.float32)
    zero = np.zeros((c, c), dtype=np.float32)
    d.update(w_a=eye, b_a=np.zeros(c, np.float32),
             w_ag=zero, b_ag=np.full(c, SAT, np.float32),
             w_b=zero, b_b=np.ones(c, np.float32),
             w_bg=zero, b_bg=np.full(c, SAT, np.float32),
             w_g=zero, b_g=np.full(c, SAT, np.float32),
             w_o=eye, b_o=np.zeros(c, np.float32))
    return d


@pytest.mark.parametrize("N", [1, 3, 6])
def test_reduces_to_layer_norm_row_sums(N):
    """With a = m*LN(z), b = m, g = 1, W_o = I the layer is LN_out of masked line sums.

    outgoing: x_ij = sum_k m_ik m_jk LN(z_ik)   (sum along row i)
    incoming: x_ij = sum_k m_ki m_kj LN(z_ki)   (sum down column i)
    The mask is random and asymmetric, so mask_rs vs mask_sr slips show up.
    """
    c = 32
    d = _identity_reduction_case(N, 10 + N, c)
    M = _t(d["mask"])
    zh = _ln(_t(d["z"]), d["ln_in_w"], d["ln_in_b"])
    x_out = torch.einsum("ik,jk,ikc->ijc", M, M, zh)
    x_in = torch.einsum("ki,kj,kic->ijc", M, M, zh)
    for direction, x in (("outgoing", x_out), ("incoming", x_in)):
        expect = _ln(x, d["ln_out_w"], d["ln_out_b"])
        got = oracle.trimul(d, direction)
        np.testing.assert_allclose(got, expect.numpy(), rtol=1e-10, atol=1e-10)


@pytest.mark.parametrize("N", [2, 5, 9])
def test_contraction_is_matmul(N):
    """Per channel, outgoing X_c = A_c B_c^T and incoming X_c = A_c^T B_c (np.matmul)."""
    rng = np.random.default_rng(N)
    c = 7
    a = rng.standard_normal((N, N, c))
    b = rng.standard_normal((N, N, c))
    x_out = oracle.contract(a, b, "outgoing")
    x_in = oracle.contract(a, b, "incoming")
    for ch in range(c):
        A, B = a[:, :, ch], b[:, :, ch]
        np.testing.assert_allclose(x_out[:, :, ch], A @ B.T, rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(x_in[:, :, ch], A.T @ B, rtol=1e-12, atol=1e-12)


def test_constant_z_closed_form():
    """z_ij = v everywhere, mask ones: x_ij = N * a (.) b with a, b from v alone."""
    N, c = 6, 128
    d = _case(N, 3, c=c, mask="ones")
    v = d["z"][2, 4].copy()
    d["z"] = np.broadcast_to(v, d["z"].shape).copy()
    zh = _ln(_t(v), d["ln_in_w"], d["ln_in_b"])
    lin = lambda x, w, b: F.linear(x, _t(d[w]), _t(d[b]))
    a = torch.sigmoid(lin(zh, "w_ag", "b_ag")) * lin(zh, "w_a", "b_a")
    b = torch.sigmoid(lin(zh, "w_bg", "b_bg")) * lin(zh, "w_b", "b_b")
    x = N * a * b
    cell = torch.sigmoid(lin(zh, "w_g", "b_g")) * lin(_ln(x, d["ln_out_w"], d["ln_out_b"]), "w_o", "b_o")
    expect = np.broadcast_to(cell.numpy(), (N, N, c))
    for direction in ("outgoing", "incoming"):
        np.testing.assert_allclose(oracle.trimul(d, direction), expect, rtol=1e-11, atol=1e-11)
    # The sum, not a mean: with LayerNorm's eps the N-scaled x differs from x itself.
    cell1 = torch.sigmoid(lin(zh, "w_g", "b_g")) * lin(_ln(a * b * 1e-3, d["ln_out_w"], d["ln_out_b"]), "w_o", "b_o")
    assert not np.allclose(cell1.numpy(), cell.numpy(), rtol=1e-6, atol=1e-6)


def test_zero_mask_closed_form():
    """mask = 0: a = b = 0, x = 0, LN_out(0) = beta_out, so out = g (.) (W_o beta_out + b_o)."""
    N, c = 5, 128
    d = _case(N, 4, c=c, mask="zeros")
    zh = _ln(_t(d["z"]), d["ln_in_w"], d["ln_in_b"])
    g = torch.sigmoid(F.linear(zh, _t(d["w_g"]), _t(d["b_g"])))
    o = F.linear(_t(d["ln_out_b"]), _t(d["w_o"]), _t(d["b_o"]))
    expect = (g * o).numpy()
    for direction in ("outgoing", "incoming"):
        np.testing.assert_allclose(oracle.trimul(d, direction), expect, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("direction", ["outgoing", "incoming"])
def test_permutation_equivariance(direction):
    """Relabelling residues by pi relabels the output: out(z')_ij = out(z)_pi(i)pi(j)."""
    N = 7
    d = _case(N, 5)
    perm = np.random.default_rng(5).permutation(N)
    dp = dict(d)
    dp["z"] = d["z"][perm][:, perm]
    dp["mask"] = d["mask"][perm][:, perm]
    out = oracle.trimul(d, direction)
    outp = oracle.trimul(dp, direction)
    np.testing.assert_allclose(outp, out[perm][:, perm], rtol=1e-12, atol=1e-12)


def _transposed(d, swap):
    t = dict(d)
    t["z"] = np.ascontiguousarray(d["z"].transpose(1, 0, 2))
    t["mask"] = np.ascontiguousarray(d["mask"].T)
    if swap:
        for p, q in (("w_a", "w_b"), ("w_ag", "w_bg"), ("b_a", "b_b"), ("b_ag", "b_bg")):
            t[p], t[q] = d[q], d[p]
    return t


def test_transpose_identity_swapped_weights():
    """incoming(z; W_a, W_ag, W_b, W_bg) = outgoing(z^T; W_b, W_bg, W_a, W_ag)^T.

    On z' = z^T with the a and b weights swapped, a'_rs = b_sr and b'_rs = a_sr,
    so outgoing gives x'_ij = sum_k b_ki a_kj; at (j, i) that is
    sum_k a_ki b_kj, the incoming x_ij. The gate reads z'_ji = z_ij.
    """
    d = _case(6, 6)
    inc = oracle.trimul(d, "incoming")
    out_t = oracle.trimul(_transposed(d, swap=True), "outgoing").transpose(1, 0, 2)
    np.testing.assert_allclose(inc, out_t, rtol=1e-12, atol=1e-12)


def test_transpose_identity_tied_weights():
    """With W_a = W_b and W_ag = W_bg the identity holds with the same weights."""
    d = _case(6, 7)
    for p, q in (("w_b", "w_a"), ("w_bg", "w_ag"), ("b_b", "b_a"), ("b_bg", "b_ag")):
        d[p] = d[q].copy()
    inc = oracle.trimul(d, "incoming")
    out_t = oracle.trimul(_transposed(d, swap=False), "outgoing").transpose(1, 0, 2)
    np.testing.assert_allclose(inc, out_t, rtol=1e-12, atol=1e-12)


def test_transpose_identity_same_weights_fails_in_general():
    """The same-weights form does not hold for untied weights (a and b roles differ)."""
    d = _case(5, 8)
    inc = oracle.trimul(d, "incoming")
    out_t = oracle.trimul(_transposed(d, swap=False), "outgoing").transpose(1, 0, 2)
    assert np.abs(inc - out_t).max() > 1e-3


@pytest.mark.parametrize("direction", ["outgoing", "incoming"])
def test_crop_invariance(direction):
    """Padded residues change nothing: out(z, m m^T)[valid, valid] = out(z[valid, valid], 1)."""
    N, nv = 8, 5
    d = _case(N, 9, mask="ones")
    m = pi.residue_mask(N, nv)
    d["mask"] = pi.pair_mask(m)
    full = oracle.trimul(d, direction)
    crop = dict(d)
    crop["z"] = np.ascontiguousarray(d["z"][:nv, :nv])
    crop["mask"] = np.ones((nv, nv), np.float32)
    np.testing.assert_allclose(full[:nv, :nv], oracle.trimul(crop, direction), rtol=1e-12, atol=1e-12)
    # Cells that touch a padded residue see x = 0 and follow the zero-mask form.
    zh = _ln(_t(d["z"]), d["ln_in_w"], d["ln_in_b"])
    g = torch.sigmoid(F.linear(zh, _t(d["w_g"]), _t(d["b_g"])))
    pad = (g * F.linear(_t(d["ln_out_b"]), _t(d["w_o"]), _t(d["b_o"]))).numpy()
    np.testing.assert_allclose(full[nv:, :], pad[nv:, :], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(full[:, nv:], pad[:, nv:], rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("direction", ["outgoing", "incoming"])
def test_grid_matches_full(direction):
    """The sampled I x I mode returns exactly the full layer's cells."""
    N = 11
    d = _case(N, 12)
    full = oracle.trimul(d, direction)
    I = np.array([0, 3, 4, 10], dtype=np.int32)
    np.testing.assert_allclose(oracle.trimul_grid(d, direction, I), full[np.ix_(I, I)],
                               rtol=1e-13, atol=1e-13)
    I = np.arange(N, dtype=np.int32)
    np.testing.assert_allclose(oracle.trimul_grid(d, direction, I), full, rtol=1e-13, atol=1e-13)


def test_stages_compose():
    """project -> contract -> finish is the whole layer."""
    d = _case(6, 13)
    a, b = oracle.project(d)
    for direction in ("outgoing", "incoming"):
        x = oracle.contract(a, b, direction)
        np.testing.assert_allclose(oracle.finish(d, x), oracle.trimul(d, direction),
                                   rtol=1e-13, atol=1e-13)


def test_planted_mistake_is_caught():
    """A slip planted in a copy of the oracle's inputs (a transposed W_a) breaks the N = 1 pin."""
    d = _case(1, 14, mask="ones")
    bad = dict(d)
    bad["w_a"] = np.ascontiguousarray(d["w_a"].T)
    zh = _ln(_t(d["z"][0, 0]), d["ln_in_w"], d["ln_in_b"])
    lin = lambda x, w, b: F.linear(x, _t(d[w]), _t(d[b]))
    a = torch.sigmoid(lin(zh, "w_ag", "b_ag")) * lin(zh, "w_a", "b_a")
    b = torch.sigmoid(lin(zh, "w_bg", "b_bg")) * lin(zh, "w_b", "b_b")
    expect = torch.sigmoid(lin(zh, "w_g", "b_g")) * lin(_ln(a * b, d["ln_out_w"], d["ln_out_b"]), "w_o", "b_o")
    got = oracle.trimul(bad, "outgoing")[0, 0]
    assert np.abs(got - expect.numpy()).max() > 1e-3


def _einsum_layer(d, direction, eps=EPS):
    """The whole layer restated with numpy float64 einsum, every weight random.

    Written from the definition, independent of the oracle: LayerNorm with the
    biased variance and eps inside the root; Linear in [out][in] layout; mask on
    a and b at their own cell; the contraction summed over the shared residue
    index (a_ik b_jk outgoing, a_ki b_kj incoming).
    """
    f = lambda k: np.asarray(d[k], dtype=np.float64)

    def ln(v, w, b):
        mu = v.mean(-1, keepdims=True)
        var = ((v - mu) ** 2).mean(-1, keepdims=True)
        return (v - mu) / np.sqrt(var + eps) * f(w) + f(b)

    def lin(v, w, b):
        return np.einsum("ijc,oc->ijo", v, f(w)) + f(b)

    sig = lambda t: 1.0 / (1.0 + np.exp(-t))
    zh = ln(f("z"), "ln_in_w", "ln_in_b")
    m = f("mask")[:, :, None]
    a = m * sig(lin(zh, "w_ag", "b_ag")) * lin(zh, "w_a", "b_a")
    b = m * sig(lin(zh, "w_bg", "b_bg")) * lin(zh, "w_b", "b_b")
    x = np.einsum("ikc,jkc->ijc", a, b) if direction == "outgoing" else np.einsum("kic,kjc->ijc", a, b)
    return sig(lin(zh, "w_g", "b_g")) * lin(ln(x, "ln_out_w", "ln_out_b"), "w_o", "b_o")


@pytest.mark.parametrize("N", [2, 3, 5, 8])
@pytest.mark.parametrize("direction", ["outgoing", "incoming"])
def test_brute_force_einsum_random_weights(N, direction):
    """Brute force at tiny N: random weights, LayerNorm affines, biases and a random
    0/1 mask, against the einsum restatement above, to 1e-12 relative. Unlike the
    special-weight pins, every step interacts with every other one here."""
    d = _case(N, 500 + N, mask="random")
    got = oracle.trimul(d, direction)
    ref = _einsum_layer(d, direction)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())


def test_brute_force_einsum_catches_swapped_contraction():
    """The einsum pin separates the directions: outgoing and incoming differ at N = 5
    with random weights, so a direction mix-up in the oracle would fail it."""
    d = _case(5, 505, mask="random")
    assert np.abs(_einsum_layer(d, "outgoing") - _einsum_layer(d, "incoming")).max() > 1e-3

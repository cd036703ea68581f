"""Pins for the windowed atom-attention oracle (oracle/atomattn.py), CPU only.

Each checks the oracle against something other than itself:
  * torch's scaled_dot_product_attention (a library routine) on every window,
    with the window's keys gathered and the bias and mask passed as an
    additive mask;
  * closed forms: equal logits give the mean of the valid values; a single
    valid key gives that key's value; a dominant bias selects its key;
  * the window geometry: a query's output does not change when keys outside
    its 128-key window change, and does change when one inside does;
  * a planted mistake (keys taken from the wrong offset) fails the library pin.
"""
import numpy as np
import pytest
import torch

from oracle.atomattn import atom_attention

Q_WIN, K_WIN = 32, 128


def n_windows(n):
    return (n + 31) // 32


def key_range(w):
    """Stated here from the reading (not taken from the oracle): 128 keys centred on the
    32 queries of window w, i.e. atoms 32 w - 48 .. 32 w + 79."""
    return 32 * w - 48, 32 * w + 80


def draw(B, n, H, d=32, seed=0, with_bias=True, mask_tail=0):
    rng = np.random.default_rng([seed, 11])
    q, k, v = (rng.standard_normal((B, n, H, d)) for _ in range(3))
    bias = rng.standard_normal((B, n_windows(n), H, Q_WIN, K_WIN)) if with_bias else None
    mask = None
    if mask_tail:
        mask = np.ones((B, n))
        mask[:, n - mask_tail:] = 0
        mask[:, rng.integers(0, n, size=3)] = 0
    return q, k, v, bias, mask


def sdpa_reference(q, k, v, bias, mask):
    """Per window: gather the key slots, build an additive mask, call torch SDPA."""
    B, n, H, d = q.shape
    out = np.zeros_like(q)
    for b in range(B):
        for w in range(n_windows(n)):
            q0, q1 = Q_WIN * w, min(Q_WIN * (w + 1), n)
            k0, k1 = key_range(w)
            slots = np.arange(k0, k1)
            inside = (slots >= 0) & (slots < n)
            ok = inside.copy()
            if mask is not None:
                ok[inside] = mask[b, slots[inside]] != 0
            if not ok.any():
                continue
            idx = np.clip(slots, 0, n - 1)
            add = np.where(ok, 0.0, -np.inf)[None, None, :].repeat(H, 0).repeat(q1 - q0, 1)
            if bias is not None:
                add = add + bias[b, w][:, : q1 - q0]
            qt = torch.from_numpy(q[b, q0:q1].transpose(1, 0, 2).copy())
            kt = torch.from_numpy(k[b, idx].transpose(1, 0, 2).copy())
            vt = torch.from_numpy(v[b, idx].transpose(1, 0, 2).copy())
            o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=torch.from_numpy(add))
            out[b, q0:q1] = o.numpy().transpose(1, 0, 2)
    return out


@pytest.mark.parametrize("n,mask_tail", [(32, 0), (100, 0), (257, 9), (300, 40)])
def test_matches_library_attention(n, mask_tail):
    q, k, v, bias, mask = draw(2, n, 3, seed=n, mask_tail=mask_tail)
    got = atom_attention(q, k, v, bias, mask)
    ref = sdpa_reference(q, k, v, bias, mask)
    np.testing.assert_allclose(got, ref, rtol=1e-10, atol=1e-12)


def test_without_bias_matches_library():
    q, k, v, _, _ = draw(1, 200, 2, seed=5, with_bias=False)
    np.testing.assert_allclose(atom_attention(q, k, v), sdpa_reference(q, k, v, None, None), rtol=1e-10,
                               atol=1e-12)


def test_equal_logits_give_mean_of_valid_values():
    n = 160
    q, k, v, _, _ = draw(1, n, 2, seed=6, with_bias=False)
    q[:] = 0.0
    out = atom_attention(q, k, v)
    for w in range(n_windows(n)):
        k0, k1 = key_range(w)
        lo, hi = max(k0, 0), min(k1, n)
        mean = v[0, lo:hi].mean(axis=0)
        np.testing.assert_allclose(out[0, Q_WIN * w: min(Q_WIN * (w + 1), n)], np.broadcast_to(mean, out[0, Q_WIN * w: min(Q_WIN * (w + 1), n)].shape), rtol=1e-12, atol=1e-12)


def test_single_valid_key_gives_its_value():
    n = 64
    q, k, v, bias, _ = draw(1, n, 2, seed=7)
    mask = np.zeros((1, n))
    mask[0, 40] = 1  # inside the windows of atoms 0..63 (window 0 keys -48..79, window 1 keys -16..111)
    out = atom_attention(q, k, v, bias, mask)
    np.testing.assert_allclose(out[0], np.broadcast_to(v[0, 40], out[0].shape), rtol=1e-12, atol=1e-12)


def test_dominant_bias_selects_its_key():
    n = 96
    q, k, v, bias, _ = draw(1, n, 1, seed=8)
    bias[:] = 0
    w, slot = 1, 70                       # window 1 (atoms 32..63), key slot 70 = atom 32 - 48 + 70 = 54
    bias[0, w, 0, :, slot] = 1e3
    out = atom_attention(q, k, v, bias)
    np.testing.assert_allclose(out[0, 32:64, 0], np.broadcast_to(v[0, 54, 0], (32, 32)), rtol=1e-9, atol=1e-9)


def test_window_geometry():
    """Window 2 (atoms 64..95) sees exactly atoms 16..143."""
    n = 300
    q, k, v, bias, _ = draw(1, n, 2, seed=9)
    base = atom_attention(q, k, v, bias)[0, 64:96]
    for atom, inside in ((15, False), (16, True), (143, True), (144, False)):
        k2 = k.copy()
        k2[0, atom] += 3.0
        changed = np.abs(atom_attention(q, k2, v, bias)[0, 64:96] - base).max() > 1e-9
        assert changed == inside, atom


def test_planted_offset_fails_library_pin():
    """A restatement with the window shifted by one key disagrees with the library pin."""
    import oracle.atomattn as oa
    q, k, v, bias, _ = draw(1, 100, 2, seed=10)
    saved = oa.K_OFFSET
    try:
        oa.K_OFFSET = saved + 1
        bad = oa.atom_attention(q, k, v, bias)
    finally:
        oa.K_OFFSET = saved
    assert np.abs(bad - sdpa_reference(q, k, v, bias, None)).max() > 1e-3

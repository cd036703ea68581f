"""The shared input generator: seeded, reproducible, bf16 rounding = torch's RNE cast."""
import numpy as np
import torch

import pair_inputs as pi


def test_round_bf16_matches_torch_cast():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10 ** rng.uniform(-6, 6, 100000).astype(np.float32),
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 65504.0], np.float32)])
    ours = pi.round_bf16(x.copy())
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(ours.view(np.uint32), ref.view(np.uint32))


def test_rows_are_independent_streams():
    full = pi.draw_z(9, 16, seed=3)
    part = pi.draw_z(9, 16, seed=3, rows=[4, 7])
    assert np.array_equal(full[[4, 7]], part)
    assert not np.array_equal(pi.draw_z(9, 16, seed=4), full)


def test_workload_shapes_and_masks():
    w = pi.WORKLOADS[2]
    d = pi.make_workload(w, with_z=False)
    assert d["mask"].shape == (384, 384)
    assert d["mask"][:346, :346].min() == 1.0 and d["mask"][346:].max() == 0.0 and d["mask"][:, 346:].max() == 0.0
    w4 = pi.WORKLOADS[4]
    assert w4.n_valid == sum(w4.chains) == 2000 and w4.N - w4.n_valid == 48
    assert sum(pi.WORKLOADS[5].chains) == 3605
    assert sum(pi.WORKLOADS[3].chains) == 768
    for k in ("w_a", "w_ag", "w_b", "w_bg", "w_g", "w_o"):
        assert d[k].shape == (128, 128)
        # bf16 workloads hold bf16-representable values only
        assert np.array_equal(d[k], pi.round_bf16(d[k].copy()))
    std = np.std(np.concatenate([d[k].ravel() for k in ("w_a", "w_b", "w_g", "w_o")]))
    assert abs(std - 1 / np.sqrt(128)) < 0.003


def test_channel_scale_in_range():
    z = pi.draw_z(16, 128, seed=2, channel_scale=True)
    s = np.random.default_rng([2, 1]).uniform(0.5, 2.0, size=128).astype(np.float32)
    assert s.min() >= 0.5 and s.max() <= 2.0
    base = pi.draw_z(16, 128, seed=2)
    np.testing.assert_allclose(z, base * s, rtol=0, atol=0)


def test_sample_grid_covers_edges():
    for N in (64, 384, 3605, 130, 1):
        I = pi.sample_grid(N, 0)
        assert I.min() == 0 and I.max() == N - 1
        assert np.all(np.diff(I) > 0)
        if N > 256:
            assert {127, 128, 255, 256} <= set(I.tolist())
        # every pair-tile (256) boundary inside the matrix
        assert {t - 1 for t in range(256, N, 256)} | set(range(256, N, 256)) <= set(I.tolist())

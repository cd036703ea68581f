"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Bars (written in each test):
  fp32 path: rel-L2 <= 1e-4 on the layer output.
  bf16 path: rel-L2 <= 1.5e-2 and max-abs <= 5e-2 on the layer output.
  bf16 stages (derived from bf16 storage of the stage outputs: 8 significant
  bits, unit roundoff u = 2^-8, about 2^-9 on average): prologue a, b and
  contraction x rel-L2 <= 1e-2, max-abs <= 4 * 2^-9 * max|ref| (= 2u).
"""
import numpy as np
import pytest
import torch

import oracle
import pair_inputs as pi
import pair_representation_b200 as tm
from gpu_helpers import DeviceCase, as_bf16, max_abs, rel_l2

pytestmark = pytest.mark.gpu

DIRS = {"outgoing": tm.OUTGOING, "incoming": tm.INCOMING}
BF16_REL, BF16_ABS = 1.5e-2, 5e-2
F32_REL = 1e-4


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from pair_representation_b200 import build
    build.build()
    tm.lib()


# ---------------------------------------------------------------- fp32 path

@pytest.mark.parametrize("direction", ["outgoing", "incoming"])
def test_fp32_workload1(direction):
    w = pi.WORKLOADS[1]
    case = pi.make_workload(w)
    dc = DeviceCase(case, "f32")
    got = dc.forward(DIRS[direction])
    ref = oracle.trimul(case, direction)
    assert rel_l2(got, ref) <= F32_REL


@pytest.mark.parametrize("N", [1, 7, 33, 129])
@pytest.mark.parametrize("direction", ["outgoing", "incoming"])
def test_fp32_edge_sizes(N, direction):
    case = pi.random_case(N, 100 + N, affine=True, mask="random")
    dc = DeviceCase(case, "f32")
    got = dc.forward(DIRS[direction])
    ref = oracle.trimul(case, direction)
    assert rel_l2(got, ref) <= F32_REL


# ---------------------------------------------------------------- bf16 stages

@pytest.mark.parametrize("N", [64, 129, 200, 256, 300, 385, 386, 513, 769, 1025])
@pytest.mark.parametrize("direction", ["outgoing", "incoming"])
def test_bf16_contraction_stage(N, direction):
    """x from random bf16 a, b written into the workspace, vs the oracle contraction."""
    rng = np.random.default_rng(N)
    a = as_bf16(rng.standard_normal((N, N, 128)) * 0.5)
    b = as_bf16(rng.standard_normal((N, N, 128)) * 0.5)
    case = pi.random_case(N, 1, bf16=True, mask="ones")
    dc = DeviceCase(case, "bf16")
    va, vb, vx = dc.views()
    va[:, :, :N] = torch.from_numpy(a.transpose(2, 0, 1).copy()).to(va.device).to(torch.bfloat16)
    vb[:, :, :N] = torch.from_numpy(b.transpose(2, 0, 1).copy()).to(vb.device).to(torch.bfloat16)
    vx.fill_(float("nan"))
    tm.trimul_contract(dc.p, DIRS[direction])
    torch.cuda.synchronize()
    assert tm.trimul_device_status(dc.p)[0] == 0
    got = DeviceCase.to_cell_major(vx, N)
    ref = oracle.contract(a, b, direction)
    assert np.isfinite(got).all()
    assert rel_l2(got, ref) <= 1e-2
    assert max_abs(got, ref) <= 4 * 2 ** -9 * np.abs(ref).max()


@pytest.mark.parametrize("N", [1, 100, 128, 300])
def test_bf16_prologue_stage(N):
    case = pi.random_case(N, 7 + N, bf16=True, affine=True, mask="random")
    dc = DeviceCase(case, "bf16")
    tm.trimul_prologue(dc.z, dc.mask, dc.p)
    torch.cuda.synchronize()
    assert tm.trimul_device_status(dc.p)[0] == 0
    va, vb, _ = dc.views()
    a_ref, b_ref = oracle.project(case)
    for got, ref in ((DeviceCase.to_cell_major(va, N), a_ref), (DeviceCase.to_cell_major(vb, N), b_ref)):
        assert rel_l2(got, ref) <= 1e-2
        assert max_abs(got, ref) <= 4 * 2 ** -9 * max(np.abs(ref).max(), 1e-3)


@pytest.mark.parametrize("N", [1, 100, 128, 300])
def test_bf16_epilogue_stage(N):
    """out from an oracle x (rounded to bf16) written into the workspace."""
    case = pi.random_case(N, 9 + N, bf16=True, affine=True, mask="random")
    a, b = oracle.project(case)
    x = as_bf16(oracle.contract(a, b, "outgoing"))
    dc = DeviceCase(case, "bf16")
    _, _, vx = dc.views()
    vx[:, :, :N] = torch.from_numpy(x.transpose(2, 0, 1).copy()).to(vx.device).to(torch.bfloat16)
    tm.trimul_epilogue(dc.z, dc.p, dc.out)
    torch.cuda.synchronize()
    assert tm.trimul_device_status(dc.p)[0] == 0
    got = dc.out.float().cpu().numpy()
    ref = oracle.finish(case, x)
    assert rel_l2(got, ref) <= BF16_REL
    assert max_abs(got, ref) <= BF16_ABS


@pytest.mark.parametrize("offset", [8.0, -30.0])
def test_bf16_epilogue_stage_large_mean(offset):
    """Cells whose mean is far from zero relative to their spread, in z and in x:
    the folded LayerNorms subtract mean * rowsum(W') after the MMA, which must
    cancel as the normalised inputs would."""
    N = 200
    case = pi.random_case(N, 77, bf16=True, affine=True, mask="random")
    case["z"] = as_bf16(case["z"] + offset)
    a, b = oracle.project(case)
    x = as_bf16(oracle.contract(a, b, "incoming") * 0.5 + offset)
    dc = DeviceCase(case, "bf16")
    _, _, vx = dc.views()
    vx[:, :, :N] = torch.from_numpy(x.transpose(2, 0, 1).copy()).to(vx.device).to(torch.bfloat16)
    tm.trimul_epilogue(dc.z, dc.p, dc.out)
    torch.cuda.synchronize()
    assert tm.trimul_device_status(dc.p)[0] == 0
    got = dc.out.float().cpu().numpy()
    ref = oracle.finish(case, x)
    assert rel_l2(got, ref) <= BF16_REL
    assert max_abs(got, ref) <= BF16_ABS


# ---------------------------------------------------------------- bf16 layer

@pytest.mark.parametrize("direction", ["outgoing", "incoming"])
def test_bf16_workload2_full(direction):
    """N = 384, last 38 residues padded: every output cell against the oracle."""
    w = pi.WORKLOADS[2]
    case = pi.make_workload(w)
    got = DeviceCase(case, "bf16").forward(DIRS[direction])
    ref = oracle.trimul(case, direction)
    assert rel_l2(got, ref) <= BF16_REL
    assert max_abs(got, ref) <= BF16_ABS


@pytest.mark.parametrize("N", [1, 7, 63, 129, 255, 257])
@pytest.mark.parametrize("direction", ["outgoing", "incoming"])
def test_bf16_edge_sizes(N, direction):
    """Ragged and tiny N with random masks, LayerNorm affines and biases."""
    case = pi.random_case(N, 200 + N, bf16=True, affine=True, mask="random")
    got = DeviceCase(case, "bf16").forward(DIRS[direction])
    ref = oracle.trimul(case, direction)
    assert rel_l2(got, ref) <= BF16_REL
    assert max_abs(got, ref) <= BF16_ABS


@pytest.mark.parametrize("mask", ["zeros", "ones"])
def test_bf16_degenerate_masks(mask):
    case = pi.random_case(150, 31, bf16=True, affine=True, mask=mask)
    for direction in ("outgoing", "incoming"):
        got = DeviceCase(case, "bf16").forward(DIRS[direction])
        ref = oracle.trimul(case, direction)
        assert rel_l2(got, ref) <= BF16_REL
        assert max_abs(got, ref) <= BF16_ABS


def test_bf16_null_mask_equals_ones():
    case = pi.random_case(96, 32, bf16=True, affine=False, mask="ones")
    a = DeviceCase(case, "bf16").forward(tm.OUTGOING)
    b = DeviceCase(case, "bf16", with_mask=False).forward(tm.OUTGOING)
    assert np.array_equal(a, b)


@pytest.mark.parametrize("direction", ["outgoing", "incoming"])
def test_bf16_workload3_full(direction):
    """The Boltz-2 crop (N = 768, per-channel scale on z): every output cell against
    the full oracle, in the launch configuration the bench times."""
    w = pi.WORKLOADS[3]
    case = pi.make_workload(w)
    got = DeviceCase(case, "bf16").forward(DIRS[direction])
    ref = oracle.trimul(case, direction)
    assert rel_l2(got, ref) <= BF16_REL
    assert max_abs(got, ref) <= BF16_ABS


@pytest.mark.parametrize("N", [385, 386, 513, 769, 1025])
@pytest.mark.parametrize("direction", ["outgoing", "incoming"])
def test_bf16_ragged_pair_tiles_full(N, direction):
    """Sizes whose last 256-wide pair tile is ragged (a partial upper half, or one
    64-column store chunk), where the contraction issues an odd number of stores per
    tile: every output cell against the oracle."""
    case = pi.random_case(N, 400 + N, bf16=True, affine=True, mask="random")
    got = DeviceCase(case, "bf16").forward(DIRS[direction])
    ref = oracle.trimul(case, direction)
    assert rel_l2(got, ref) <= BF16_REL
    assert max_abs(got, ref) <= BF16_ABS


@pytest.mark.parametrize("wid", [4, 5])
def test_bf16_large_workloads_sampled(wid):
    """Full-size workloads (N = 2048, 3605) in the launch configuration the bench
    times; the oracle computes the sampled grid I x I cell by cell: every 256-wide
    pair-tile edge, the first 128-tile edges, the ragged tail, the padding boundary
    of the mask and random residues."""
    w = pi.WORKLOADS[wid]
    case = pi.make_workload(w)
    I = pi.sample_grid(w.N, w.seed, n_random=16)
    if w.n_valid < w.N:
        I = np.unique(np.concatenate([I, [w.n_valid - 1, w.n_valid]])).astype(np.int32)
    dc = DeviceCase(case, "bf16")
    for direction in w.directions:
        got = dc.forward(DIRS[direction])[np.ix_(I, I)]
        ref = oracle.trimul_grid(case, direction, I)
        assert rel_l2(got, ref) <= BF16_REL, direction
        assert max_abs(got, ref) <= BF16_ABS, direction
        assert np.isfinite(dc.out.float().cpu().numpy()).all()


def test_bf16_transpose_identity_full_size():
    """A property at any size: incoming(z; W_a, W_ag, W_b, W_bg) equals
    outgoing(z^T; W_b, W_bg, W_a, W_ag)^T, here at N = 768 on the GPU alone."""
    w = pi.WORKLOADS[3]
    case = pi.make_workload(w)
    inc = DeviceCase(case, "bf16").forward(tm.INCOMING)
    t = dict(case)
    t["z"] = np.ascontiguousarray(case["z"].transpose(1, 0, 2))
    t["mask"] = np.ascontiguousarray(case["mask"].T)
    t["w_a"], t["w_b"], t["w_ag"], t["w_bg"] = case["w_b"], case["w_a"], case["w_bg"], case["w_ag"]
    out_t = DeviceCase(t, "bf16").forward(tm.OUTGOING).transpose(1, 0, 2)
    assert rel_l2(inc, out_t) <= BF16_REL

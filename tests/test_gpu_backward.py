"""GPU parity of trimul_backward (through the C ABI) against the float64
backward oracle (oracle/backward.py), bf16 path.

Inputs are the bf16-rounded cases of the forward tests, and dout is drawn and
rounded to bf16; the oracle sees the same values in float64. Bar, on every
gradient tensor (dz and each of the 16 parameter gradients):
  rel-L2 <= BWD_REL.
The GPU path stores its intermediates (a, b, x, LayerNorm outputs, dy, dx and
the pre-activation gradients) in bf16 and accumulates in fp32; see the
derivation of BWD_REL below.
"""
import numpy as np
import pytest
import torch

import oracle.backward as ob
import pair_inputs as pi
import pair_representation_b200 as tm
from gpu_helpers import DeviceCase, as_bf16, rel_l2

pytestmark = pytest.mark.gpu

DIRS = {"outgoing": tm.OUTGOING, "incoming": tm.INCOMING}
# Each gradient passes through up to six bf16 roundings of its operands (unit
# roundoff u = 2^-8, RMS relative error about u / sqrt(3) = 2.3e-3 each); with
# independent roundings their RMS errors add in quadrature to about 6e-3, and a
# factor of about 3 is left for the amplification by the LayerNorm adjoints.
BWD_REL = 2e-2
SHAPES = {"w_a": (128, 128), "w_ag": (128, 128), "w_b": (128, 128), "w_bg": (128, 128), "w_g": (128, 128),
          "w_o": (128, 128)}


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from pair_representation_b200 import build
    build.build()
    tm.lib()


def run_backward(case, direction, dout, with_mask=True, rows=None):
    """dz and the 16 parameter gradients from the library, as float64 numpy;
    with `rows`, given only the workspace for blocks of that many rows."""
    dc = DeviceCase(case, "bf16", with_mask=with_mask)
    N = dc.N
    g = tm.TrimulGrads()
    need = tm.trimul_backward_workspace_size(N) if rows is None else tm.trimul_backward_workspace_size_rows(N, rows)
    bws = torch.empty(need, dtype=torch.uint8, device="cuda")
    g.workspace, g.workspace_bytes = bws.data_ptr(), bws.numel()
    out = {}
    for f in tm.GRAD_FIELDS:
        t = torch.full(SHAPES.get(f[2:], (128,)), float("nan"), dtype=torch.float32, device="cuda")
        setattr(g, f, t.data_ptr())
        out[f[2:]] = t
    d = torch.from_numpy(np.ascontiguousarray(dout, dtype=np.float32)).to("cuda").to(torch.bfloat16)
    dz = torch.full_like(dc.z, float("nan"))
    tm.trimul_backward(dc.z, dc.mask, dc.p, DIRS[direction], d, dz, g)
    torch.cuda.synchronize()
    rc, detail = tm.trimul_device_status(dc.p)
    assert rc == 0, (rc, detail)
    res = {k: v.double().cpu().numpy() for k, v in out.items()}
    res["z"] = dz.double().cpu().numpy()
    return res


def draw_dout(N, seed):
    return as_bf16(np.random.default_rng([seed, 9]).standard_normal((N, N, 128)))


def compare(got, ref, tag):
    errs = {}
    for k in ["z"] + list(ob.WEIGHTS) + list(ob.BIASES) + list(ob.AFFINES):
        assert np.isfinite(got[k]).all(), (tag, k)
        errs[k] = rel_l2(got[k], ref[k])
    print(tag, " ".join(f"{k}={v:.2e}" for k, v in errs.items()))
    bad = {k: v for k, v in errs.items() if not v <= BWD_REL}
    assert not bad, (tag, bad)


@pytest.mark.parametrize("N", [1, 64, 129, 200])
@pytest.mark.parametrize("direction", ["outgoing", "incoming"])
def test_backward_parity(N, direction):
    case = pi.random_case(N, 300 + N, bf16=True, affine=True, mask="random")
    dout = draw_dout(N, N)
    got = run_backward(case, direction, dout)
    ref = ob.trimul_backward(case, direction, dout)
    compare(got, ref, f"N={N} {direction}")


@pytest.mark.parametrize("direction", ["outgoing", "incoming"])
def test_backward_without_affines_or_mask(direction):
    """NULL biases, LayerNorm affines and mask: every gradient is still produced."""
    N = 97
    case = pi.random_case(N, 41, bf16=True, affine=False, mask="ones")
    dout = draw_dout(N, 41)
    got = run_backward(case, direction, dout, with_mask=False)
    ref = ob.trimul_backward({k: v for k, v in case.items() if k != "mask"}, direction, dout)
    compare(got, ref, f"no-affine {direction}")


def test_backward_zero_mask():
    """mask = 0: a = b = x = 0, so nothing flows through the contraction; the
    input-gate gradients vanish and dz comes from the output gate alone."""
    N = 70
    case = pi.random_case(N, 43, bf16=True, affine=True, mask="zeros")
    dout = draw_dout(N, 43)
    got = run_backward(case, "outgoing", dout)
    ref = ob.trimul_backward(case, "outgoing", dout)
    for k in ("w_a", "w_ag", "w_b", "w_bg", "b_a", "b_ag", "b_b", "b_bg"):
        assert np.abs(got[k]).max() == 0.0, k
        assert np.abs(ref[k]).max() == 0.0, k
    for k in ("z", "w_g", "w_o", "b_g", "b_o", "ln_in_w", "ln_in_b", "ln_out_b"):
        assert rel_l2(got[k], ref[k]) <= BWD_REL, k


def test_backward_direction_identity_large():
    """At a size the oracle does not reach, a property of the exact gradients:
    incoming(z, mask; W_a, W_ag, W_b, W_bg) has the gradients of
    outgoing(z^T, mask^T; W_b, W_bg, W_a, W_ag), transposed back, with the a-
    and b-side gradients swapped. Both sides run on the GPU."""
    N = 384
    case = pi.random_case(N, 45, bf16=True, affine=True, mask="random")
    dout = draw_dout(N, 45)
    g_in = run_backward(case, "incoming", dout)
    t = dict(case)
    t["z"] = np.ascontiguousarray(case["z"].transpose(1, 0, 2))
    t["mask"] = np.ascontiguousarray(case["mask"].T)
    swap = {"w_a": "w_b", "w_ag": "w_bg", "w_b": "w_a", "w_bg": "w_ag",
            "b_a": "b_b", "b_ag": "b_bg", "b_b": "b_a", "b_bg": "b_ag"}
    for k, v in swap.items():
        t[k] = case[v]
    g_out = run_backward(t, "outgoing", np.ascontiguousarray(dout.transpose(1, 0, 2)))
    assert rel_l2(g_in["z"], g_out["z"].transpose(1, 0, 2)) <= BWD_REL
    for k in ("w_g", "w_o", "b_g", "b_o") + ob.AFFINES:
        assert rel_l2(g_in[k], g_out[k]) <= BWD_REL, k
    for k, v in swap.items():
        assert rel_l2(g_in[k], g_out[v]) <= BWD_REL, k


def test_backward_layer_api_matches_abi():
    """The layer's backward() returns what the C-ABI call returns."""
    N = 64
    case = pi.random_case(N, 47, bf16=True, affine=True, mask="random")
    dout = draw_dout(N, 47)
    ref = run_backward(case, "outgoing", dout)
    sd = {key: case[field] for field, key, _ in tm.STATE_KEYS if field in case}
    layer = tm.TriangleMultiplicationOutgoing(128, 128).load_state_dict(sd).to("cuda", torch.bfloat16)
    z = torch.from_numpy(case["z"]).to("cuda").to(torch.bfloat16)
    m = torch.from_numpy(case["mask"]).to("cuda")
    d = torch.from_numpy(dout).to("cuda").to(torch.bfloat16)
    dz, grads = layer.backward(z, d, m)
    torch.cuda.synchronize()
    assert rel_l2(dz.double().cpu().numpy(), ref["z"]) <= 1e-6
    for k, v in grads.items():
        assert rel_l2(v.double().cpu().numpy(), ref[k]) <= 1e-6, k


@pytest.mark.parametrize("direction", ["outgoing", "incoming"])
def test_backward_reusing_the_forward_matches_recompute(direction):
    """With TRIMUL_BWD_REUSE_FORWARD after a forward call on the same inputs, the
    backward skips recomputing a, b and x and returns what the recomputing call
    returns (the recompute is deterministic; only the atomically summed bias and
    LayerNorm gradients may differ in their last bits), and matches the oracle."""
    N = 129
    case = pi.random_case(N, 51, bf16=True, affine=True, mask="random")
    dout = draw_dout(N, 51)
    ref = run_backward(case, direction, dout)
    sd = {key: case[field] for field, key, _ in tm.STATE_KEYS if field in case}
    cls = tm.TriangleMultiplicationOutgoing if direction == "outgoing" else tm.TriangleMultiplicationIncoming
    layer = cls(128, 128).load_state_dict(sd).to("cuda", torch.bfloat16)
    z = torch.from_numpy(case["z"]).to("cuda").to(torch.bfloat16)
    m = torch.from_numpy(case["mask"]).to("cuda")
    d = torch.from_numpy(dout).to("cuda").to(torch.bfloat16)
    layer(z, m)
    dz, grads = layer.backward(z, d, m, reuse_forward=True)
    torch.cuda.synchronize()
    assert torch.equal(dz.double().cpu(), torch.from_numpy(ref["z"]))
    for k, v in grads.items():
        assert rel_l2(v.double().cpu().numpy(), ref[k]) <= 1e-6, k
    compare({**{k: v.double().cpu().numpy() for k, v in grads.items()}, "z": dz.double().cpu().numpy()},
            ob.trimul_backward(case, direction, dout.astype(np.float64)), "reuse")


@pytest.mark.parametrize("direction", ["outgoing", "incoming"])
def test_backward_in_row_blocks(direction):
    """Given the workspace for blocks of 37 rows, the N = 200 backward runs in
    five blocks of 37 rows and one of 15. Every cell is computed as in the
    whole-grid call, so dz is the same bit for bit; the parameter gradients
    differ only in the order of their fp32 sums. Both match the oracle."""
    N = 200
    case = pi.random_case(N, 53, bf16=True, affine=True, mask="random")
    dout = draw_dout(N, 53)
    whole = run_backward(case, direction, dout)
    blocks = run_backward(case, direction, dout, rows=37)
    assert np.array_equal(blocks["z"], whole["z"])
    for k in ob.WEIGHTS + ob.BIASES + ob.AFFINES:
        assert rel_l2(blocks[k], whole[k]) <= 1e-5, k
    compare(blocks, ob.trimul_backward(case, direction, dout), f"blocks of 37 rows {direction}")


def test_backward_single_row_blocks_through_the_layer():
    """The smallest workspace (blocks of one row) through the layer API: the
    same dz as the whole-grid call, the same gradients up to summation order."""
    N = 64
    case = pi.random_case(N, 55, bf16=True, affine=True, mask="random")
    dout = draw_dout(N, 55)
    ref = run_backward(case, "incoming", dout)
    sd = {key: case[field] for field, key, _ in tm.STATE_KEYS if field in case}
    layer = tm.TriangleMultiplicationIncoming(128, 128).load_state_dict(sd).to("cuda", torch.bfloat16)
    z = torch.from_numpy(case["z"]).to("cuda").to(torch.bfloat16)
    m = torch.from_numpy(case["mask"]).to("cuda")
    d = torch.from_numpy(dout).to("cuda").to(torch.bfloat16)
    dz, grads = layer.backward(z, d, m, block_rows=1)
    torch.cuda.synchronize()
    assert np.array_equal(dz.double().cpu().numpy(), ref["z"])
    for k, v in grads.items():
        assert rel_l2(v.double().cpu().numpy(), ref[k]) <= 1e-5, k

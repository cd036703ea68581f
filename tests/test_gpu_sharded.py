"""The shard stage calls on one GPU: P ranks emulated one after another.

The multi-GPU split (pair_representation_b200.sharded) runs the prologue on
row blocks, the contraction on channel blocks and the epilogue on row blocks,
with two exchanges between them. Here every rank's stage calls run on one GPU
in turn and the exchanges are local copies following the same ShardPlan, so
no kernel waits on another. The kernels are the same as trimul_forward's and
every cell (and every channel's contraction tile) does the same arithmetic,
so the assembled output must equal trimul_forward's bit for bit; it is also
checked against the oracle with the bf16 bars (rel-L2 <= 1.5e-2, max-abs <=
5e-2). The exchange code itself is tested on CPU ranks (test_sharded_cpu.py).
"""
import numpy as np
import pytest
import torch

import oracle
import pair_inputs as pi
import pair_representation_b200 as tm
from gpu_helpers import DeviceCase, max_abs, rel_l2
from pair_representation_b200.sharded import ShardPlan

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from pair_representation_b200 import build
    build.build()
    tm.lib()


def _emulate(dc, plan, direction, with_mask=True):
    N, ld, P = plan.N, plan.ld, plan.world
    dev, bf = dc.z.device, torch.bfloat16
    ws = torch.zeros(tm.trimul_shard_workspace_size(N, max(plan.nrows(r) for r in range(P))), dtype=torch.uint8,
                     device=dev)
    p = tm.TrimulParams.from_buffer_copy(dc.p)
    p.workspace, p.workspace_bytes = ws.data_ptr(), ws.numel()
    a_loc, b_loc = [], []
    for r in range(P):
        r0, r1 = plan.rows(r)
        a = torch.full((128, r1 - r0, ld), float("nan"), dtype=bf, device=dev)
        b = torch.full_like(a, float("nan"))
        mask = dc.mask[r0:r1] if with_mask else None
        tm.trimul_prologue_rows(dc.z[r0:r1], mask, p, r1 - r0, a, b)
        a_loc.append(a)
        b_loc.append(b)
    x_ch = []
    for q in range(P):
        c0, c1 = plan.channels(q)
        a_ch = torch.zeros((c1 - c0, N, ld), dtype=bf, device=dev)
        b_ch = torch.zeros_like(a_ch)
        for r in range(P):
            r0, r1 = plan.rows(r)
            a_ch[:, r0:r1] = a_loc[r][c0:c1]
            b_ch[:, r0:r1] = b_loc[r][c0:c1]
        x = torch.full_like(a_ch, float("nan"))
        tm.trimul_contract_channels(p, direction, c1 - c0, a_ch, b_ch, x)
        x_ch.append(x)
    out = torch.full_like(dc.z, float("nan"))
    for r in range(P):
        r0, r1 = plan.rows(r)
        x_loc = torch.zeros((128, r1 - r0, ld), dtype=bf, device=dev)
        for q in range(P):
            c0, c1 = plan.channels(q)
            x_loc[c0:c1] = x_ch[q][:, r0:r1]
        tm.trimul_epilogue_rows(dc.z[r0:r1], x_loc, p, r1 - r0, out[r0:r1])
    torch.cuda.synchronize()
    rc, detail = tm.trimul_device_status(p)
    assert rc == 0, (rc, detail)
    return out


@pytest.mark.parametrize("world", [2, 3, 8])
@pytest.mark.parametrize("N", [200, 257])
@pytest.mark.parametrize("direction", ["outgoing", "incoming"])
def test_shards_assemble_to_the_layer(world, N, direction):
    d = tm.OUTGOING if direction == "outgoing" else tm.INCOMING
    case = pi.random_case(N, 700 + N + world, bf16=True, affine=True, mask="random")
    dc = DeviceCase(case, "bf16")
    whole = torch.from_numpy(dc.forward(d))
    got = _emulate(dc, ShardPlan(N, world), d).float().cpu()
    assert torch.equal(got, whole)
    ref = oracle.trimul(case, direction)
    assert rel_l2(got.numpy(), ref) <= 1.5e-2 and max_abs(got.numpy(), ref) <= 5e-2


def test_shards_without_mask_equal_layer():
    N = 130
    case = pi.random_case(N, 77, bf16=True, affine=False, mask="ones")
    dc = DeviceCase(case, "bf16", with_mask=False)
    whole = torch.from_numpy(dc.forward(tm.INCOMING))
    got = _emulate(dc, ShardPlan(N, 4), tm.INCOMING, with_mask=False).float().cpu()
    assert torch.equal(got, whole)


def test_shard_calls_reject_bad_arguments():
    N = 64
    dc = DeviceCase(pi.random_case(N, 5, bf16=True, mask="ones"), "bf16")
    p = tm.TrimulParams.from_buffer_copy(dc.p)
    small = torch.zeros(256, dtype=torch.uint8, device=dc.z.device)
    p.workspace, p.workspace_bytes = small.data_ptr(), small.numel()
    a = torch.zeros((128, 8, 64), dtype=torch.bfloat16, device=dc.z.device)
    rc = tm.trimul_prologue_rows(dc.z[:8], None, p, 8, a, a.clone(), check=False)
    assert rc == tm.ERR["TRIMUL_ERR_WORKSPACE"]
    p.workspace, p.workspace_bytes = dc.ws.data_ptr(), dc.ws.numel()
    assert tm.trimul_prologue_rows(dc.z[:8], None, p, 0, a, a.clone(), check=False) == tm.ERR["TRIMUL_ERR_INVALID_ARG"]
    assert tm.trimul_prologue_rows(dc.z[:8], None, p, 8, a, a, check=False) == tm.ERR["TRIMUL_ERR_ALIAS"]
    x = torch.zeros((200, N, 64), dtype=torch.bfloat16, device=dc.z.device)
    assert tm.trimul_contract_channels(p, tm.OUTGOING, 129, x, x.clone(), x.clone(), check=False) == \
        tm.ERR["TRIMUL_ERR_INVALID_ARG"]


def test_sharded_module_single_rank_equals_layer():
    """The host-side module on one rank with the CUDA stages (its exchanges reduce to
    the rank's own copies): bit-identical to trimul_forward."""
    from pair_representation_b200.sharded import CudaStages, ShardedTriangleMultiplication
    N = 150
    case = pi.random_case(N, 81, bf16=True, affine=True, mask="random")
    dc = DeviceCase(case, "bf16")
    for d in (tm.OUTGOING, tm.INCOMING):
        whole = torch.from_numpy(dc.forward(d))
        p = tm.TrimulParams.from_buffer_copy(dc.p)
        ws = torch.zeros(tm.trimul_shard_workspace_size(N, N), dtype=torch.uint8, device=dc.z.device)
        p.workspace, p.workspace_bytes = ws.data_ptr(), ws.numel()
        layer = ShardedTriangleMultiplication(ShardPlan(N, 1), 0, d, CudaStages(tm, p), dc.z.device,
                                              torch.bfloat16, torch.distributed)
        got = layer(dc.z, dc.mask).float().cpu()
        torch.cuda.synchronize()
        assert tm.trimul_device_status(p)[0] == 0
        assert torch.equal(got, whole)

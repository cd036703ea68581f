"""trimul_forward_noalloc: the layer for callers that cannot allocate device memory.

Some callers have no allocator to give the layer its workspace: a plugin whose
host application owns every byte of device memory, or a latency-critical loop
that must never risk a failed or synchronising allocation. For them the
library keeps the scratch in its own static device array. These checks call
the no-allocation entry point through the C ABI twice in a row and compare
each result with trimul_forward (caller-supplied workspace) on the same
inputs, within the bf16 tolerance of the other parity tests.
"""
import numpy as np
import pytest
import torch

import pair_inputs as pi
import pair_representation_b200 as tm
from gpu_helpers import DeviceCase, max_abs, rel_l2

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from pair_representation_b200 import build
    build.build()
    tm.lib()


def test_noalloc_matches_forward_twice_in_a_row():
    calls = [(128, 301, tm.OUTGOING), (100, 302, tm.INCOMING)]
    for N, seed, direction in calls:
        case = pi.random_case(N, seed, bf16=True, affine=True, mask="random")
        dc = DeviceCase(case, "bf16")
        ref = dc.forward(direction)  # trimul_forward with the caller's workspace
        out = torch.full_like(dc.z, float("nan"))
        q = tm.TrimulParams.from_buffer_copy(dc.p)
        q.workspace, q.workspace_bytes = None, 0  # ignored by the no-allocation entry point
        tm.trimul_forward_noalloc(dc.z, dc.mask, q, direction, out)
        torch.cuda.synchronize()
        got = out.float().cpu().numpy()
        assert np.isfinite(got).all()
        assert rel_l2(got, ref) <= 1.5e-2 and max_abs(got, ref) <= 5e-2


def test_noalloc_rejects_sizes_beyond_its_scratch():
    case = pi.random_case(129, 303, bf16=True, mask="ones")
    dc = DeviceCase(case, "bf16")
    rc = tm.trimul_forward_noalloc(dc.z, dc.mask, dc.p, tm.OUTGOING, dc.out, check=False)
    assert rc == tm.ERR["TRIMUL_ERR_WORKSPACE"]

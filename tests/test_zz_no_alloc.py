"""trimul_forward_noalloc: the layer for callers that cannot allocate device memory.

Some callers have no allocator to give the layer its workspace: a plugin whose
host application owns every byte of device memory, or a latency-critical loop
that must never risk a failed or synchronising allocation. For them the
library keeps the scratch in its own static device array. These checks call
the no-allocation entry point through the C ABI, twice in a row, and compare
each result with trimul_forward (caller-supplied workspace) on the same inputs
and with the CPU oracle, within the tolerances of the other parity tests
(bf16: rel-L2 <= 1.5e-2, max-abs <= 5e-2; fp32: rel-L2 <= 1e-4). They also
check the size limit (bf16 N <= 128, fp32 N <= 88), and that a timeout inside
the no-allocation call is reported through trimul_device_status.
"""
import numpy as np
import pytest
import torch

import oracle
import pair_inputs as pi
import pair_representation_b200 as tm
from gpu_helpers import DeviceCase, max_abs, rel_l2

pytestmark = pytest.mark.gpu

DIRS = {tm.OUTGOING: "outgoing", tm.INCOMING: "incoming"}


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from pair_representation_b200 import build
    build.build()
    tm.lib()


def _noalloc(dc, direction):
    """One no-allocation call on dc's inputs; returns the output as float64 numpy."""
    out = torch.full_like(dc.z, float("nan"))
    q = tm.TrimulParams.from_buffer_copy(dc.p)
    q.workspace, q.workspace_bytes = None, 0  # ignored by the no-allocation entry point
    tm.trimul_forward_noalloc(dc.z, dc.mask, q, direction, out)
    torch.cuda.synchronize()
    rc, detail = tm.trimul_device_status(q)  # workspace NULL: the static scratch's status word
    assert rc == 0, (rc, detail)
    return out.double().cpu().numpy()


@pytest.mark.parametrize("dtype,calls", [
    ("bf16", [(128, 301, tm.OUTGOING), (100, 302, tm.INCOMING), (1, 304, tm.OUTGOING)]),
    ("f32", [(88, 305, tm.OUTGOING), (88, 306, tm.INCOMING)]),
])
def test_noalloc_matches_forward_and_oracle_twice_in_a_row(dtype, calls):
    rel_bar = 1.5e-2 if dtype == "bf16" else 1e-4
    for N, seed, direction in calls:
        case = pi.random_case(N, seed, bf16=dtype == "bf16", affine=True, mask="random")
        dc = DeviceCase(case, dtype)
        ref_fwd = dc.forward(direction)  # trimul_forward with the caller's workspace
        ref = oracle.trimul(case, DIRS[direction])
        for _ in range(2):  # the second call reuses the scratch the first left behind
            got = _noalloc(dc, direction)
            assert np.isfinite(got).all()
            assert rel_l2(got, ref_fwd) <= rel_bar
            assert rel_l2(got, ref) <= rel_bar
            if dtype == "bf16":
                assert max_abs(got, ref_fwd) <= 5e-2 and max_abs(got, ref) <= 5e-2


@pytest.mark.parametrize("dtype,N", [("bf16", 129), ("f32", 89)])
def test_noalloc_rejects_sizes_beyond_its_scratch(dtype, N):
    case = pi.random_case(N, 303, bf16=dtype == "bf16", mask="ones")
    dc = DeviceCase(case, dtype)
    rc = tm.trimul_forward_noalloc(dc.z, dc.mask, dc.p, tm.OUTGOING, dc.out, check=False)
    assert rc == tm.ERR["TRIMUL_ERR_WORKSPACE"]


def test_noalloc_timeout_is_reported_and_next_call_is_clean():
    """A contraction wait that nothing satisfies (debug flag) runs out inside the
    no-allocation call; the static scratch's status word reports it, and the next
    call clears it and matches the oracle."""
    case = pi.random_case(96, 307, bf16=True, affine=True, mask="random")
    dc = DeviceCase(case, "bf16")
    q = tm.TrimulParams.from_buffer_copy(dc.p)
    q.workspace, q.workspace_bytes = None, 0
    q.debug_flags, q.timeout_ms = tm.DEBUG_STALL_CONTRACT, 20
    tm.trimul_forward_noalloc(dc.z, dc.mask, q, tm.OUTGOING, dc.out)
    rc, detail = tm.trimul_device_status(q)
    assert rc == tm.ERR["TRIMUL_ERR_TIMEOUT"], (rc, detail)
    assert detail[0] == 1 and (detail[1] & 0xF0) == 0x20  # the contraction's wait
    got = _noalloc(dc, tm.OUTGOING)
    ref = oracle.trimul(case, "outgoing")
    assert rel_l2(got, ref) <= 1.5e-2 and max_abs(got, ref) <= 5e-2

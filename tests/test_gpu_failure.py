"""Failure detection without a GPU fault.

The contraction's MMA issuer is told (debug flag) to wait on a barrier that
nothing signals. Its bounded wait runs out after timeout_ms, the kernel
records TRIMUL_ERR_TIMEOUT in the workspace status word, every warp of the
CTA leaves its loop, in-flight copies are drained and tensor memory is
released. The host reads the status, and the same context then runs a normal
call whose result matches the oracle: nothing was left hung or corrupted.
"""
import numpy as np
import pytest
import torch

import oracle
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


def test_stalled_wait_reports_timeout_and_context_survives():
    case = pi.random_case(200, 41, bf16=True, affine=True, mask="random")
    dc = DeviceCase(case, "bf16")
    dc.p.debug_flags = tm.DEBUG_STALL_CONTRACT
    dc.p.timeout_ms = 20
    tm.trimul_forward(dc.z, dc.mask, dc.p, tm.OUTGOING, dc.out)
    rc, detail = tm.trimul_device_status(dc.p)
    assert rc == tm.ERR["TRIMUL_ERR_TIMEOUT"], (rc, detail)
    assert detail[0] == 1 and (detail[1] & 0xF0) == 0x20  # contraction site
    assert torch.cuda.synchronize() is None

    dc.p.debug_flags = 0
    dc.p.timeout_ms = 0
    got = dc.forward(tm.OUTGOING)  # asserts a clean status itself
    ref = oracle.trimul(case, "outgoing")
    assert rel_l2(got, ref) <= 1.5e-2 and max_abs(got, ref) <= 5e-2


def test_status_is_cleared_per_call():
    case = pi.random_case(64, 42, bf16=True, mask="ones")
    dc = DeviceCase(case, "bf16")
    dc.p.debug_flags = tm.DEBUG_STALL_CONTRACT
    dc.p.timeout_ms = 10
    tm.trimul_forward(dc.z, dc.mask, dc.p, tm.INCOMING, dc.out)
    assert tm.trimul_device_status(dc.p)[0] == tm.ERR["TRIMUL_ERR_TIMEOUT"]
    dc.p.debug_flags = 0
    tm.trimul_forward(dc.z, dc.mask, dc.p, tm.INCOMING, dc.out)
    assert tm.trimul_device_status(dc.p)[0] == 0
    assert np.isfinite(dc.out.float().cpu().numpy()).all()

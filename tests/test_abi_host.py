"""The C-ABI library on a machine without a GPU: it loads, exports every
symbol include/trimul.h declares, sizes the workspace, and rejects bad
arguments on the host before touching CUDA."""
import ctypes
import os
import re

import pytest

import pair_representation_b200 as tm
from pair_representation_b200 import build as tmbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    tmbuild.build()
    return tm.lib()


def _declared():
    src = open(os.path.join(ROOT, "include", "trimul.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(trimul_[a-z_]+)\s*\(", src)))


def test_exports_every_declared_symbol(L):
    names = _declared()
    assert "trimul_forward" in names and "trimul_workspace_size" in names
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(tm.EXPORTS)


def test_version_and_strings(L):
    assert L.trimul_version() == 100
    for code, name in tm.STATUS.items():
        assert L.trimul_error_string(code)
    assert L.trimul_error_string(12345) == b"unknown status"


def test_workspace_size(L):
    for N in (1, 7, 64, 384, 3605):
        ld = (N + 7) // 8 * 8
        sec = lambda es: (128 * N * ld * es + 255) // 256 * 256
        assert tm.trimul_workspace_size(N) == 256 + 3 * sec(4)
        assert tm.trimul_workspace_size_dtype(N, 128, 128, tm.DTYPE_BF16) == 256 + 3 * sec(2)
        assert tm.trimul_workspace_size_dtype(N, 128, 128, tm.DTYPE_F32) == tm.trimul_workspace_size(N)
    assert tm.trimul_workspace_size(0) == 0
    assert tm.trimul_workspace_size(16385) == 0
    assert tm.trimul_workspace_size(64, 64, 128) == 0
    assert tm.trimul_workspace_size_dtype(64, 128, 128, 7) == 0


BASE = 1 << 32  # fake, 256-byte-aligned device addresses: never dereferenced by host checks


def _params(N=64, dtype=tm.DTYPE_BF16):
    p = tm.TrimulParams()
    p.N, p.c_z, p.c_h, p.dtype, p.ln_eps = N, 128, 128, dtype, 1e-5
    for k, f in enumerate(("w_a", "w_ag", "w_b", "w_bg", "w_g", "w_o")):
        setattr(p, f, BASE + 0x100000 * (k + 1))
    p.workspace = BASE + 0x10000000
    p.workspace_bytes = tm.trimul_workspace_size(N)
    return p


Z = BASE + 0x40000000
OUT = BASE + 0x80000000
MASK = BASE + 0xC0000000


def _fwd(p, z=Z, mask=MASK, out=OUT, direction=0):
    return tm.trimul_forward(z, mask, p, direction, out, stream=0, check=False)


def test_argument_checks(L):
    E = tm.ERR
    assert tm.lib().trimul_forward(Z, MASK, None, 0, OUT, None) == E["TRIMUL_ERR_INVALID_ARG"]
    p = _params()
    assert _fwd(p, direction=2) == E["TRIMUL_ERR_INVALID_ARG"]
    assert _fwd(p, z=None) == E["TRIMUL_ERR_INVALID_ARG"]
    assert _fwd(p, out=None) == E["TRIMUL_ERR_INVALID_ARG"]
    for N in (0, -3, 16385):
        q = _params()
        q.N = N
        assert _fwd(q) == E["TRIMUL_ERR_INVALID_ARG"], N
    q = _params(); q.c_z = 64
    assert _fwd(q) == E["TRIMUL_ERR_UNSUPPORTED"]
    q = _params(); q.c_h = 256
    assert _fwd(q) == E["TRIMUL_ERR_UNSUPPORTED"]
    q = _params(); q.dtype = 5
    assert _fwd(q) == E["TRIMUL_ERR_UNSUPPORTED"]
    q = _params(); q.ln_eps = 0.0
    assert _fwd(q) == E["TRIMUL_ERR_INVALID_ARG"]
    q = _params(); q.w_g = None
    assert _fwd(q) == E["TRIMUL_ERR_INVALID_ARG"]
    q = _params(); q.w_o = BASE + 8
    assert _fwd(q) == E["TRIMUL_ERR_MISALIGNED"]
    q = _params(); q.b_a = BASE + 1
    assert _fwd(q) == E["TRIMUL_ERR_MISALIGNED"]
    q = _params(); q.workspace = None
    assert _fwd(q) == E["TRIMUL_ERR_WORKSPACE"]
    q = _params(); q.workspace_bytes = tm.trimul_workspace_size_dtype(64, 128, 128, tm.DTYPE_BF16) - 1
    assert _fwd(q) == E["TRIMUL_ERR_WORKSPACE"]
    q = _params(); q.workspace += 16
    assert _fwd(q) == E["TRIMUL_ERR_MISALIGNED"]
    assert _fwd(p, z=Z + 8) == E["TRIMUL_ERR_MISALIGNED"]
    assert _fwd(p, out=OUT + 4) == E["TRIMUL_ERR_MISALIGNED"]
    assert _fwd(p, mask=MASK + 1) == E["TRIMUL_ERR_MISALIGNED"]


def test_alias_checks(L):
    E = tm.ERR
    p = _params(N=64)
    zbytes = 64 * 64 * 128 * 2
    assert _fwd(p, out=Z) == E["TRIMUL_ERR_ALIAS"]
    assert _fwd(p, out=Z + zbytes - 16) == E["TRIMUL_ERR_ALIAS"]
    assert _fwd(p, out=MASK) == E["TRIMUL_ERR_ALIAS"]
    assert _fwd(p, out=p.workspace + 256) == E["TRIMUL_ERR_ALIAS"]
    assert _fwd(p, z=p.workspace + 1024) == E["TRIMUL_ERR_ALIAS"]
    assert _fwd(p, mask=p.workspace + 512) == E["TRIMUL_ERR_ALIAS"]


def test_valid_arguments_reach_cuda_and_fail_loudly_without_gpu(L):
    """No CPU fallback: with no GPU the first CUDA call fails and the call says so."""
    try:
        import torch
        if torch.cuda.is_available():
            pytest.skip("a GPU is present")
    except ImportError:
        pass
    p = _params()
    rc = _fwd(p)
    assert rc in (tm.ERR["TRIMUL_ERR_CUDA"], tm.ERR["TRIMUL_ERR_UNSUPPORTED"])
    with pytest.raises(tm.TrimulError):
        tm.trimul_forward(Z, MASK, p, 0, OUT, stream=0)
    assert tm.lib().trimul_contract(ctypes.byref(p), 0, None) in (tm.ERR["TRIMUL_ERR_CUDA"],
                                                                    tm.ERR["TRIMUL_ERR_UNSUPPORTED"])


def test_stage_argument_checks(L):
    E = tm.ERR
    p = _params()
    assert tm.trimul_contract(p, 3, stream=0, check=False) == E["TRIMUL_ERR_INVALID_ARG"]
    assert tm.trimul_prologue(None, MASK, p, stream=0, check=False) == E["TRIMUL_ERR_INVALID_ARG"]
    assert tm.trimul_epilogue(Z, p, Z, stream=0, check=False) == E["TRIMUL_ERR_ALIAS"]
    a, b, x, ld = tm.trimul_workspace_views(p)
    assert a == p.workspace + 256 and ld == 64
    assert b - a == x - b == 128 * 64 * 64 * 2

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
    names = set()
    for h in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if h.endswith(".h"):
            src = open(os.path.join(ROOT, "include", h)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b((?:trimul|atomattn)_[a-z0-9_]+)\s*\(", src))
    return sorted(names)


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
        ld32, ld16 = (N + 7) // 8 * 8, (N + 63) // 64 * 64  # fp32 rows on 32 B, bf16 rows on 128 B
        sec = lambda es, ld: (128 * N * ld * es + 255) // 256 * 256
        assert tm.trimul_workspace_size(N) == 256 + 3 * sec(4, ld32)
        assert tm.trimul_workspace_size_dtype(N, 128, 128, tm.DTYPE_BF16) == 256 + 3 * sec(2, ld16)
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


# ---- backward ------------------------------------------------------------------

def _bwd_layout_bytes(N, R=None):
    """Backward workspace for blocks of R rows (default: the whole grid): sums,
    weight stack, the double weight-gradient sums, the per-cell sections of one
    block, dP_G of the whole grid when R < N, dX, dA, dB channel-major, then one
    [768][128] fp32 weight-gradient partial per 4096 cells of a block."""
    R = N if R is None else R
    r = lambda v: (v + 255) // 256 * 256
    M, C, ld = R * N, 128, (N + 63) // 64 * 64
    cm = C * N * ld
    parts = [10 * C * 4, 5 * C * C * 2, 768 * C * 8, M * 8, M * 8, M * C * 2, M * C * 2, M * 5 * C * 2, M * C * 2,
             M * C * 4, M * 5 * C * 2, M * C * 2] + ([N * N * C * 2] if R < N else []) + \
            [cm * 2, cm * 2, cm * 2, (M + 4095) // 4096 * 768 * C * 4]
    return sum(r(p) for p in parts)


def test_backward_workspace_size(L):
    for N in (1, 7, 64, 129, 768):
        assert tm.trimul_backward_workspace_size(N) == _bwd_layout_bytes(N), N
        assert tm.trimul_backward_workspace_size_rows(N, N) == _bwd_layout_bytes(N), N
    for N, R in ((7, 1), (64, 5), (129, 64), (200, 37), (768, 100), (3605, 256)):
        assert tm.trimul_backward_workspace_size_rows(N, R) == _bwd_layout_bytes(N, R), (N, R)
    assert tm.trimul_backward_workspace_size(0) == 0
    assert tm.trimul_backward_workspace_size(16385) == 0
    assert tm.trimul_backward_workspace_size(64, 64, 128) == 0
    assert tm.trimul_backward_workspace_size_rows(64, 0) == 0
    assert tm.trimul_backward_workspace_size_rows(64, 65) == 0
    # The largest workload's backward: about 65 GB for the whole grid, under 18 GB in blocks of 256 rows.
    assert tm.trimul_backward_workspace_size(3605) > 60e9
    assert tm.trimul_backward_workspace_size_rows(3605, 256) < 18e9
    # Below the whole grid the size grows with the rows.
    sizes = [tm.trimul_backward_workspace_size_rows(200, R) for R in range(1, 200)]
    assert all(a < b for a, b in zip(sizes, sizes[1:]))


def test_backward_block_rows(L):
    """The block the call uses for a given workspace: the whole grid when it fits,
    else the largest block whose size fits, none below one row."""
    for N in (1, 7, 200, 768, 3605):
        full = tm.trimul_backward_workspace_size(N)
        assert tm.trimul_backward_block_rows(N, full) == N
        assert tm.trimul_backward_block_rows(N, 10 * full) == N
        one = tm.trimul_backward_workspace_size_rows(N, 1)
        assert tm.trimul_backward_block_rows(N, one - 1) == 0
        if N > 1:
            for R in sorted({1, 2, N // 3, N // 2, N - 1} - {0}):
                size = tm.trimul_backward_workspace_size_rows(N, R)
                got = tm.trimul_backward_block_rows(N, size)
                assert got >= R, (N, R, got)
                if got < N:  # the largest block that fits
                    assert tm.trimul_backward_workspace_size_rows(N, got) <= size
                    assert got == N - 1 or tm.trimul_backward_workspace_size_rows(N, got + 1) > size
    assert tm.trimul_backward_block_rows(0, 1 << 40) == 0
    assert tm.trimul_backward_block_rows(64, 1 << 40, 64, 128) == 0


DOUT = BASE + 0x100000000
DZ = BASE + 0x140000000
GWS = BASE + 0x200000000


def _grads(N=64):
    g = tm.TrimulGrads()
    g.workspace = GWS
    g.workspace_bytes = tm.trimul_backward_workspace_size(N)
    for k, f in enumerate(tm.GRAD_FIELDS):
        setattr(g, f, BASE + 0x400000000 + 0x100000 * k)
    return g


def _bwd(p, g, z=Z, mask=MASK, dout=DOUT, dz=DZ, direction=0):
    return tm.trimul_backward(z, mask, p, direction, dout, dz, g, stream=0, check=False)


def test_backward_argument_checks(L):
    E = tm.ERR
    p, g = _params(), _grads()
    assert tm.lib().trimul_backward(Z, MASK, ctypes.byref(p), 0, DOUT, DZ, None, None) == E["TRIMUL_ERR_INVALID_ARG"]
    assert _bwd(p, g, dout=None) == E["TRIMUL_ERR_INVALID_ARG"]
    assert _bwd(p, g, dz=None) == E["TRIMUL_ERR_INVALID_ARG"]
    assert _bwd(p, g, direction=2) == E["TRIMUL_ERR_INVALID_ARG"]
    assert _bwd(_params(dtype=tm.DTYPE_F32), g) == E["TRIMUL_ERR_UNSUPPORTED"]
    assert _bwd(p, g, dout=DOUT + 8) == E["TRIMUL_ERR_MISALIGNED"]
    assert _bwd(p, g, dz=DZ + 2) == E["TRIMUL_ERR_MISALIGNED"]
    q = _grads(); q.workspace = None
    assert _bwd(p, q) == E["TRIMUL_ERR_WORKSPACE"]
    q = _grads(); q.workspace_bytes = tm.trimul_backward_workspace_size_rows(64, 1) - 1
    assert _bwd(p, q) == E["TRIMUL_ERR_WORKSPACE"]
    q = _grads(); q.workspace += 128
    assert _bwd(p, q) == E["TRIMUL_ERR_MISALIGNED"]
    q = _grads(); q.d_w_o += 4
    assert _bwd(p, q) == E["TRIMUL_ERR_MISALIGNED"]
    q = _grads(); q.d_b_g += 2
    assert _bwd(p, q) == E["TRIMUL_ERR_MISALIGNED"]


def test_backward_alias_checks(L):
    E = tm.ERR
    p, g = _params(), _grads()
    zbytes = 64 * 64 * 128 * 2
    assert _bwd(p, g, dz=Z) == E["TRIMUL_ERR_ALIAS"]
    assert _bwd(p, g, dz=DOUT + zbytes - 16) == E["TRIMUL_ERR_ALIAS"]
    assert _bwd(p, g, dz=p.workspace + 256) == E["TRIMUL_ERR_ALIAS"]
    assert _bwd(p, g, dz=GWS + 4096) == E["TRIMUL_ERR_ALIAS"]
    assert _bwd(p, g, dout=GWS) == E["TRIMUL_ERR_ALIAS"]
    q = _grads(); q.workspace = p.workspace
    assert _bwd(p, q) == E["TRIMUL_ERR_ALIAS"]
    q = _grads(); q.d_w_a = q.d_w_ag
    assert _bwd(p, q) == E["TRIMUL_ERR_ALIAS"]
    q = _grads(); q.d_b_a = DZ
    assert _bwd(p, q) == E["TRIMUL_ERR_ALIAS"]
    q = _grads(); q.d_ln_in_w = GWS + 512
    assert _bwd(p, q) == E["TRIMUL_ERR_ALIAS"]


def test_backward_reaches_cuda_and_fails_loudly_without_gpu(L):
    try:
        import torch
        if torch.cuda.is_available():
            pytest.skip("a GPU is present")
    except ImportError:
        pass
    p, g = _params(), _grads()
    assert _bwd(p, g) in (tm.ERR["TRIMUL_ERR_CUDA"], tm.ERR["TRIMUL_ERR_UNSUPPORTED"])
    q = _grads()
    for f in tm.GRAD_FIELDS:
        setattr(q, f, None)  # every gradient output skipped: still a valid call
    assert _bwd(p, q) in (tm.ERR["TRIMUL_ERR_CUDA"], tm.ERR["TRIMUL_ERR_UNSUPPORTED"])


# ---- atom attention -------------------------------------------------------------

def _attn(B=2, n=100, H=4):
    p = tm.AtomAttnParams()
    p.batch, p.n_atoms, p.heads, p.head_dim = B, n, H, 32
    p.q, p.k, p.v = BASE + 0x1000000, BASE + 0x2000000, BASE + 0x3000000
    p.bias, p.atom_mask = BASE + 0x4000000, BASE + 0x5000000
    p.workspace, p.workspace_bytes = BASE + 0x6000000, tm.atomattn_workspace_size()
    return p


AOUT = BASE + 0x7000000


def test_atomattn_argument_checks(L):
    E = tm.ERR
    f = lambda p, out=AOUT: tm.atomattn_forward(p, out, stream=0, check=False)
    assert tm.atomattn_workspace_size() == 256
    assert tm.lib().atomattn_forward(None, AOUT, None) == E["TRIMUL_ERR_INVALID_ARG"]
    assert f(_attn(), out=None) == E["TRIMUL_ERR_INVALID_ARG"]
    for field, val, code in (("batch", 0, "INVALID_ARG"), ("n_atoms", 0, "INVALID_ARG"), ("heads", 0, "INVALID_ARG"),
                             ("head_dim", 64, "UNSUPPORTED"), ("heads", 65, "UNSUPPORTED"),
                             ("heads", 66, "UNSUPPORTED"), ("q", None, "INVALID_ARG"),
                             ("k", BASE + 8, "MISALIGNED"), ("bias", BASE + 0x4000008, "MISALIGNED"),
                             ("atom_mask", BASE + 1, "MISALIGNED"), ("workspace", None, "WORKSPACE"),
                             ("workspace_bytes", 255, "WORKSPACE"), ("workspace", BASE + 0x6000010, "MISALIGNED")):
        p = _attn()
        setattr(p, field, val)
        assert f(p) == E["TRIMUL_ERR_" + code], (field, val)
    assert f(_attn(), out=AOUT + 8) == E["TRIMUL_ERR_MISALIGNED"]
    p = _attn()
    assert f(p, out=p.q) == E["TRIMUL_ERR_ALIAS"]
    assert f(p, out=p.bias + 4096) == E["TRIMUL_ERR_ALIAS"]
    assert f(p, out=p.workspace - 2 * 100 * 4 * 32 * 2 + 16) == E["TRIMUL_ERR_ALIAS"]
    q = _attn()
    q.bias = None
    q.atom_mask = None  # optional inputs: still a valid call
    try:
        import torch
        gpu = torch.cuda.is_available()
    except ImportError:
        gpu = False
    if not gpu:
        assert f(q) in (E["TRIMUL_ERR_CUDA"], E["TRIMUL_ERR_UNSUPPORTED"])

"""Python binding of the B200 triangle multiplicative update (libtrimul_b200.so).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels (see include/trimul.h). PyTorch supplies device memory and streams.
There is no CPU fallback: if the library is missing or no sm_100 GPU is
present, calls raise.

Two levels:
  * C-ABI mirrors with the same names as the header (``trimul_forward``,
    ``trimul_prologue``, ``trimul_contract``, ``trimul_epilogue``,
    ``trimul_workspace_size`` ...) taking ``TrimulParams`` and raw pointers or
    tensors.
  * ``TriangleMultiplicationOutgoing`` / ``TriangleMultiplicationIncoming``:
    the layer as the pages use it (construct with the channel size, load a
    state dict, call ``layer(z, mask)``), holding device weights and the
    workspace.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "_lib", "libtrimul_b200.so")

OUTGOING, INCOMING = 0, 1
DTYPE_F32, DTYPE_BF16 = 0, 1
DEBUG_STALL_CONTRACT = 0x1
BWD_REUSE_FORWARD = 0x1

STATUS = {
    0: "TRIMUL_OK", -1: "TRIMUL_ERR_INVALID_ARG", -2: "TRIMUL_ERR_UNSUPPORTED", -3: "TRIMUL_ERR_MISALIGNED",
    -4: "TRIMUL_ERR_ALIAS", -5: "TRIMUL_ERR_WORKSPACE", -6: "TRIMUL_ERR_CUDA", -7: "TRIMUL_ERR_TIMEOUT",
    -8: "TRIMUL_ERR_DEVICE",
}
ERR = {v: k for k, v in STATUS.items()}

# Every symbol include/trimul.h and include/atomattn.h declare.
EXPORTS = ("trimul_workspace_size", "trimul_workspace_size_dtype", "trimul_forward", "trimul_prologue",
           "trimul_contract", "trimul_epilogue", "trimul_workspace_views", "trimul_device_status",
           "trimul_error_string", "trimul_last_error_detail", "trimul_version", "trimul_forward_noalloc",
           "trimul_backward", "trimul_backward_workspace_size", "trimul_backward_workspace_size_rows",
           "trimul_backward_block_rows",
           "trimul_workspace_size_mxfp8", "trimul_forward_mxfp8", "trimul_contract_mxfp8", "trimul_mxfp8_views",
           "trimul_prologue_mxfp8", "trimul_mma_mxfp8",
           "trimul_shard_workspace_size", "trimul_prologue_rows", "trimul_contract_channels", "trimul_epilogue_rows",
           "atomattn_forward", "atomattn_workspace_size", "atomattn_device_status")

# Gradient outputs of trimul_grads, in struct order; each is "d_" + a TrimulParams field.
GRAD_FIELDS = ("d_w_a", "d_w_ag", "d_w_b", "d_w_bg", "d_w_g", "d_w_o", "d_b_a", "d_b_ag", "d_b_b", "d_b_bg",
               "d_b_g", "d_b_o", "d_ln_in_w", "d_ln_in_b", "d_ln_out_w", "d_ln_out_b")


class TrimulError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        self.code = code
        detail = ""
        try:
            detail = lib().trimul_last_error_detail().decode()
        except Exception:  # noqa: BLE001 - best effort only
            pass
        super().__init__(f"{what}: {STATUS.get(code, code)}" + (f" ({detail})" if detail else ""))


class TrimulParams(ctypes.Structure):
    """Mirror of ``trimul_params`` in include/trimul.h."""

    _fields_ = [
        ("N", ctypes.c_int), ("c_z", ctypes.c_int), ("c_h", ctypes.c_int), ("dtype", ctypes.c_int),
        ("ln_eps", ctypes.c_float),
        ("ln_in_w", ctypes.c_void_p), ("ln_in_b", ctypes.c_void_p),
        ("w_a", ctypes.c_void_p), ("w_ag", ctypes.c_void_p), ("w_b", ctypes.c_void_p), ("w_bg", ctypes.c_void_p),
        ("b_a", ctypes.c_void_p), ("b_ag", ctypes.c_void_p), ("b_b", ctypes.c_void_p), ("b_bg", ctypes.c_void_p),
        ("w_g", ctypes.c_void_p), ("b_g", ctypes.c_void_p),
        ("ln_out_w", ctypes.c_void_p), ("ln_out_b", ctypes.c_void_p),
        ("w_o", ctypes.c_void_p), ("b_o", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t),
        ("timeout_ms", ctypes.c_uint32), ("debug_flags", ctypes.c_uint32),
    ]


class TrimulGrads(ctypes.Structure):
    """Mirror of ``trimul_grads`` in include/trimul.h (fp32 gradient outputs + backward workspace)."""

    _fields_ = [(f, ctypes.c_void_p) for f in GRAD_FIELDS] + [
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t), ("flags", ctypes.c_uint32)]


class AtomAttnParams(ctypes.Structure):
    """Mirror of ``atomattn_params`` in include/atomattn.h."""

    _fields_ = [
        ("batch", ctypes.c_int), ("n_atoms", ctypes.c_int), ("heads", ctypes.c_int), ("head_dim", ctypes.c_int),
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("bias", ctypes.c_void_p), ("atom_mask", ctypes.c_void_p),
        ("workspace", ctypes.c_void_p), ("workspace_bytes", ctypes.c_size_t), ("timeout_ms", ctypes.c_uint32),
    ]


_lib = None


def lib():
    """Load libtrimul_b200.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m pair_representation_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
        PP = ctypes.POINTER(TrimulParams)
        L.trimul_workspace_size.argtypes = [I, I, I]
        L.trimul_workspace_size.restype = S
        L.trimul_workspace_size_dtype.argtypes = [I, I, I, I]
        L.trimul_workspace_size_dtype.restype = S
        L.trimul_forward.argtypes = [P, P, PP, I, P, P]
        L.trimul_forward_noalloc.argtypes = [P, P, PP, I, P, P]
        L.trimul_prologue.argtypes = [P, P, PP, P]
        L.trimul_contract.argtypes = [PP, I, P]
        L.trimul_epilogue.argtypes = [P, PP, P, P]
        L.trimul_workspace_views.argtypes = [PP, ctypes.POINTER(P), ctypes.POINTER(P), ctypes.POINTER(P),
                                             ctypes.POINTER(S)]
        L.trimul_device_status.argtypes = [PP, P, ctypes.POINTER(ctypes.c_int)]
        L.trimul_error_string.argtypes = [I]
        L.trimul_error_string.restype = ctypes.c_char_p
        L.trimul_last_error_detail.argtypes = []
        L.trimul_last_error_detail.restype = ctypes.c_char_p
        L.trimul_version.argtypes = []
        L.trimul_backward_workspace_size.argtypes = [I, I, I]
        L.trimul_backward_workspace_size.restype = S
        L.trimul_backward_workspace_size_rows.argtypes = [I, I, I, I]
        L.trimul_backward_workspace_size_rows.restype = S
        L.trimul_backward_block_rows.argtypes = [I, I, I, S]
        L.trimul_backward.argtypes = [P, P, PP, I, P, P, ctypes.POINTER(TrimulGrads), P]
        L.trimul_workspace_size_mxfp8.argtypes = [I, I, I]
        L.trimul_workspace_size_mxfp8.restype = S
        L.trimul_forward_mxfp8.argtypes = [P, P, PP, I, P, P]
        L.trimul_contract_mxfp8.argtypes = [PP, I, P]
        L.trimul_prologue_mxfp8.argtypes = [P, P, PP, I, P]
        L.trimul_mma_mxfp8.argtypes = [PP, P]
        L.trimul_mxfp8_views.argtypes = [PP] + [ctypes.POINTER(P)] * 4 + [ctypes.POINTER(S)]
        L.trimul_shard_workspace_size.argtypes = [I, I]
        L.trimul_shard_workspace_size.restype = S
        L.trimul_prologue_rows.argtypes = [P, P, PP, I, P, P, P]
        L.trimul_contract_channels.argtypes = [PP, I, I, P, P, P, P]
        L.trimul_epilogue_rows.argtypes = [P, P, PP, I, P, P]
        AP = ctypes.POINTER(AtomAttnParams)
        L.atomattn_workspace_size.argtypes = []
        L.atomattn_workspace_size.restype = S
        L.atomattn_forward.argtypes = [AP, P, P]
        L.atomattn_device_status.argtypes = [AP, P, ctypes.POINTER(ctypes.c_int)]
        for f in ("trimul_forward", "trimul_forward_noalloc", "trimul_prologue", "trimul_contract", "trimul_epilogue",
                  "trimul_workspace_views", "trimul_device_status", "trimul_version", "trimul_backward",
                  "atomattn_forward", "atomattn_device_status", "trimul_forward_mxfp8", "trimul_contract_mxfp8",
                  "trimul_mxfp8_views", "trimul_prologue_mxfp8", "trimul_mma_mxfp8", "trimul_prologue_rows", "trimul_contract_channels", "trimul_epilogue_rows"):
            getattr(L, f).restype = I
        _lib = L
    return _lib


def _ptr(t):
    """Device address of a tensor, an int address, or None."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc: int, what: str):
    if rc != 0:
        raise TrimulError(rc, what)


# ---- C-ABI mirrors ---------------------------------------------------------

def trimul_workspace_size(N: int, c_z: int = 128, c_h: int = 128) -> int:
    return lib().trimul_workspace_size(N, c_z, c_h)


def trimul_workspace_size_dtype(N: int, c_z: int, c_h: int, dtype: int) -> int:
    return lib().trimul_workspace_size_dtype(N, c_z, c_h, dtype)


def trimul_forward(z, mask, params: TrimulParams, direction: int, out, stream=None, check=True) -> int:
    rc = lib().trimul_forward(_ptr(z), _ptr(mask), ctypes.byref(params), direction, _ptr(out), _stream(stream))
    if check:
        _check(rc, "trimul_forward")
    return rc


def trimul_forward_noalloc(z, mask, params: TrimulParams, direction: int, out, stream=None, check=True) -> int:
    """trimul_forward with the library's static scratch instead of params.workspace.

    For callers that cannot allocate device memory; limited to bf16 N <= 128
    and fp32 N <= 88. Overlapping calls share the scratch and race.
    """
    rc = lib().trimul_forward_noalloc(_ptr(z), _ptr(mask), ctypes.byref(params), direction, _ptr(out),
                                      _stream(stream))
    if check:
        _check(rc, "trimul_forward_noalloc")
    return rc


def trimul_prologue(z, mask, params: TrimulParams, stream=None, check=True) -> int:
    rc = lib().trimul_prologue(_ptr(z), _ptr(mask), ctypes.byref(params), _stream(stream))
    if check:
        _check(rc, "trimul_prologue")
    return rc


def trimul_contract(params: TrimulParams, direction: int, stream=None, check=True) -> int:
    rc = lib().trimul_contract(ctypes.byref(params), direction, _stream(stream))
    if check:
        _check(rc, "trimul_contract")
    return rc


def trimul_epilogue(z, params: TrimulParams, out, stream=None, check=True) -> int:
    rc = lib().trimul_epilogue(_ptr(z), ctypes.byref(params), _ptr(out), _stream(stream))
    if check:
        _check(rc, "trimul_epilogue")
    return rc


def trimul_backward_workspace_size(N: int, c_z: int = 128, c_h: int = 128) -> int:
    return lib().trimul_backward_workspace_size(N, c_z, c_h)


def trimul_backward_workspace_size_rows(N: int, rows: int, c_z: int = 128, c_h: int = 128) -> int:
    return lib().trimul_backward_workspace_size_rows(N, c_z, c_h, rows)


def trimul_backward_block_rows(N: int, workspace_bytes: int, c_z: int = 128, c_h: int = 128) -> int:
    return lib().trimul_backward_block_rows(N, c_z, c_h, workspace_bytes)


def trimul_backward(z, mask, params: TrimulParams, direction: int, dout, dz, grads: TrimulGrads, stream=None,
                    check=True) -> int:
    """dz and the fp32 parameter gradients of sum(out * dout); see trimul_backward in the header."""
    rc = lib().trimul_backward(_ptr(z), _ptr(mask), ctypes.byref(params), direction, _ptr(dout), _ptr(dz),
                               ctypes.byref(grads), _stream(stream))
    if check:
        _check(rc, "trimul_backward")
    return rc


def trimul_workspace_size_mxfp8(N: int, c_z: int = 128, c_h: int = 128) -> int:
    return lib().trimul_workspace_size_mxfp8(N, c_z, c_h)


def trimul_forward_mxfp8(z, mask, params: TrimulParams, direction: int, out, stream=None, check=True) -> int:
    """The layer with the contraction in MXFP8 (E4M3 in blocks of 32 along k, E8M0 scales)."""
    rc = lib().trimul_forward_mxfp8(_ptr(z), _ptr(mask), ctypes.byref(params), direction, _ptr(out), _stream(stream))
    if check:
        _check(rc, "trimul_forward_mxfp8")
    return rc


def trimul_contract_mxfp8(params: TrimulParams, direction: int, stream=None, check=True) -> int:
    rc = lib().trimul_contract_mxfp8(ctypes.byref(params), direction, _stream(stream))
    if check:
        _check(rc, "trimul_contract_mxfp8")
    return rc


def trimul_prologue_mxfp8(z, mask, params: TrimulParams, direction: int, stream=None, check=True) -> int:
    """The quantising prologue: z, mask -> E4M3 operands and scales of `direction`'s contraction."""
    rc = lib().trimul_prologue_mxfp8(_ptr(z), _ptr(mask), ctypes.byref(params), direction, _stream(stream))
    if check:
        _check(rc, "trimul_prologue_mxfp8")
    return rc


def trimul_mma_mxfp8(params: TrimulParams, stream=None, check=True) -> int:
    """The block-scaled contraction of the MXFP8 operands in the workspace -> x."""
    rc = lib().trimul_mma_mxfp8(ctypes.byref(params), _stream(stream))
    if check:
        _check(rc, "trimul_mma_mxfp8")
    return rc


def trimul_mxfp8_views(params: TrimulParams):
    """(aq, bq, sa, sb, ldq): device addresses of the quantised operands and scales in the workspace."""
    ptrs = [ctypes.c_void_p() for _ in range(4)]
    ldq = ctypes.c_size_t()
    _check(lib().trimul_mxfp8_views(ctypes.byref(params), *[ctypes.byref(x) for x in ptrs], ctypes.byref(ldq)),
           "trimul_mxfp8_views")
    return ptrs[0].value, ptrs[1].value, ptrs[2].value, ptrs[3].value, ldq.value


def trimul_shard_workspace_size(N: int, rows: int) -> int:
    return lib().trimul_shard_workspace_size(N, rows)


def trimul_prologue_rows(z_rows, mask_rows, params: TrimulParams, rows: int, a, b, stream=None, check=True) -> int:
    rc = lib().trimul_prologue_rows(_ptr(z_rows), _ptr(mask_rows), ctypes.byref(params), rows, _ptr(a), _ptr(b),
                                    _stream(stream))
    if check:
        _check(rc, "trimul_prologue_rows")
    return rc


def trimul_contract_channels(params: TrimulParams, direction: int, channels: int, a, b, x, stream=None,
                             check=True) -> int:
    rc = lib().trimul_contract_channels(ctypes.byref(params), direction, channels, _ptr(a), _ptr(b), _ptr(x),
                                        _stream(stream))
    if check:
        _check(rc, "trimul_contract_channels")
    return rc


def trimul_epilogue_rows(z_rows, x_rows, params: TrimulParams, rows: int, out_rows, stream=None, check=True) -> int:
    rc = lib().trimul_epilogue_rows(_ptr(z_rows), _ptr(x_rows), ctypes.byref(params), rows, _ptr(out_rows),
                                    _stream(stream))
    if check:
        _check(rc, "trimul_epilogue_rows")
    return rc


def trimul_workspace_views(params: TrimulParams):
    """(a, b, x, ld): device addresses of the workspace sections and their leading dimension."""
    a, b, x = ctypes.c_void_p(), ctypes.c_void_p(), ctypes.c_void_p()
    ld = ctypes.c_size_t()
    _check(lib().trimul_workspace_views(ctypes.byref(params), ctypes.byref(a), ctypes.byref(b),
                                        ctypes.byref(x), ctypes.byref(ld)), "trimul_workspace_views")
    return a.value, b.value, x.value, ld.value


def trimul_device_status(params: TrimulParams, stream=None):
    """(code, [code, site, block, aux]) of the workspace status word (synchronises)."""
    d = (ctypes.c_int * 4)()
    rc = lib().trimul_device_status(ctypes.byref(params), _stream(stream), d)
    return rc, list(d)


# ---- sequence-local atom attention -------------------------------------------

def atomattn_workspace_size() -> int:
    return lib().atomattn_workspace_size()


def atomattn_forward(params: AtomAttnParams, out, stream=None, check=True) -> int:
    rc = lib().atomattn_forward(ctypes.byref(params), _ptr(out), _stream(stream))
    if check:
        _check(rc, "atomattn_forward")
    return rc


def atomattn_device_status(params: AtomAttnParams, stream=None):
    """(code, [code, site, block, aux]) of the status word (synchronises)."""
    d = (ctypes.c_int * 4)()
    rc = lib().atomattn_device_status(ctypes.byref(params), _stream(stream), d)
    return rc, list(d)


def atom_attention(q, k, v, bias=None, atom_mask=None, out=None, workspace=None, stream=None):
    """Windowed atom attention (include/atomattn.h) on bf16 device tensors.

    q, k, v: [batch][n_atoms][heads][32]; bias: [batch][ceil(n_atoms/32)][heads][32][128]
    or None; atom_mask: [batch][n_atoms] or None. Returns out (allocated if None)."""
    import torch
    if q.dim() != 4 or q.shape[-1] != 32 or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must be [batch, n_atoms, heads, 32] of one shape")
    for t in (q, k, v, bias, atom_mask):
        if t is not None and (t.dtype != torch.bfloat16 or not t.is_contiguous()):
            raise ValueError("inputs must be contiguous bf16")
    B, n, H, _ = q.shape
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = torch.zeros(atomattn_workspace_size(), dtype=torch.uint8, device=q.device)
    p = AtomAttnParams()
    p.batch, p.n_atoms, p.heads, p.head_dim = B, n, H, 32
    p.q, p.k, p.v = q.data_ptr(), k.data_ptr(), v.data_ptr()
    p.bias, p.atom_mask = _ptr(bias), _ptr(atom_mask)
    p.workspace, p.workspace_bytes = workspace.data_ptr(), workspace.numel()
    atomattn_forward(p, out, stream)
    return out, p


# ---- the layer as the pages use it ------------------------------------------

# State-dict keys: (params field, key, required)
STATE_KEYS = (
    ("ln_in_w", "layer_norm_in.weight", False), ("ln_in_b", "layer_norm_in.bias", False),
    ("w_a", "linear_a_p.weight", True), ("b_a", "linear_a_p.bias", False),
    ("w_ag", "linear_a_g.weight", True), ("b_ag", "linear_a_g.bias", False),
    ("w_b", "linear_b_p.weight", True), ("b_b", "linear_b_p.bias", False),
    ("w_bg", "linear_b_g.weight", True), ("b_bg", "linear_b_g.bias", False),
    ("w_g", "linear_g.weight", True), ("b_g", "linear_g.bias", False),
    ("ln_out_w", "layer_norm_out.weight", False), ("ln_out_b", "layer_norm_out.bias", False),
    ("w_o", "linear_z.weight", True), ("b_o", "linear_z.bias", False),
)


class _TriangleMultiplication:
    """Holds device weights and a workspace; ``layer(z, mask)`` returns the update."""

    direction = OUTGOING

    def __init__(self, c_z: int = 128, c_hidden: int = 128, eps: float = 1e-5):
        self.c_z, self.c_h, self.eps = c_z, c_hidden, eps
        self.tensors = {}
        self.device = None
        self.dtype = None
        self._ws = None
        self.timeout_ms = 0
        self.debug_flags = 0

    def load_state_dict(self, sd: dict):
        """Take weights by the keys in STATE_KEYS (torch tensors or numpy arrays)."""
        import torch
        t = {}
        for field, key, required in STATE_KEYS:
            if key in sd and sd[key] is not None:
                v = sd[key]
                t[field] = v if isinstance(v, torch.Tensor) else torch.as_tensor(v)
            elif required:
                raise KeyError(key)
        self.tensors = t
        return self

    def to(self, device=None, dtype=None):
        import torch
        dtype = dtype or next(iter(self.tensors.values())).dtype
        if dtype not in (torch.float32, torch.bfloat16):
            raise ValueError("dtype must be float32 or bfloat16")
        self.tensors = {k: v.to(device=device, dtype=dtype).contiguous() for k, v in self.tensors.items()}
        self.device = self.tensors["w_a"].device  # resolved (cuda -> cuda:0)
        self.dtype = dtype
        return self

    def params(self, N: int) -> TrimulParams:
        import torch
        p = TrimulParams()
        p.N, p.c_z, p.c_h = N, self.c_z, self.c_h
        p.dtype = DTYPE_BF16 if self.dtype == torch.bfloat16 else DTYPE_F32
        p.ln_eps = self.eps
        for field, _, _ in STATE_KEYS:
            setattr(p, field, _ptr(self.tensors.get(field)))
        need = trimul_workspace_size_dtype(N, self.c_z, self.c_h, p.dtype)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(need, dtype=torch.uint8, device=self.device)
        p.workspace = self._ws.data_ptr()
        p.workspace_bytes = self._ws.numel()
        p.timeout_ms = self.timeout_ms
        p.debug_flags = self.debug_flags
        return p

    def __call__(self, z, mask=None, out=None, stream=None):
        import torch
        if z.dim() != 3 or z.shape[0] != z.shape[1] or z.shape[2] != self.c_z:
            raise ValueError("z must be [N, N, c_z]")
        if z.dtype != self.dtype or z.device != self.device:
            raise ValueError("z must match the layer's dtype and device")
        z = z.contiguous()
        if mask is not None:
            mask = mask.to(dtype=self.dtype).contiguous()
        if out is None:
            out = torch.empty_like(z)
        p = self.params(z.shape[0])
        trimul_forward(z, mask, p, self.direction, out, stream)
        return out

    def backward(self, z, dout, mask=None, stream=None, reuse_forward=False, block_rows=None):
        """Gradients of sum(layer(z, mask) * dout): (dz, {params field: fp32 gradient}).

        Every parameter gets a gradient, including the optional ones the state
        dict left out (taken as bias 0, gamma 1, beta 0 in the forward). With
        reuse_forward the call relies on the layer's last forward call having
        been ``layer(z, mask)`` with this z and mask (its a, b and x are still in
        the workspace) and does not recompute them. block_rows gives the call
        only the workspace for blocks of that many rows
        (trimul_backward_workspace_size_rows); the library then uses the largest
        block that fits in it."""
        import torch
        if z.dim() != 3 or z.shape[0] != z.shape[1] or z.shape[2] != self.c_z:
            raise ValueError("z must be [N, N, c_z]")
        if z.dtype != self.dtype or z.device != self.device or dout.shape != z.shape or dout.dtype != z.dtype:
            raise ValueError("z and dout must match each other and the layer's dtype and device")
        z, dout = z.contiguous(), dout.contiguous()
        if mask is not None:
            mask = mask.to(dtype=self.dtype).contiguous()
        N = z.shape[0]
        p = self.params(N)
        g = TrimulGrads()
        need = (trimul_backward_workspace_size(N, self.c_z, self.c_h) if block_rows is None
                else trimul_backward_workspace_size_rows(N, block_rows, self.c_z, self.c_h))
        if need == 0:
            raise ValueError("no backward workspace size for these arguments")
        if getattr(self, "_bws", None) is None or self._bws.numel() < need:
            self._bws = torch.empty(need, dtype=torch.uint8, device=self.device)
        g.workspace, g.workspace_bytes = self._bws.data_ptr(), need
        g.flags = BWD_REUSE_FORWARD if reuse_forward else 0
        cz, ch = self.c_z, self.c_h
        shapes = {"w_a": (ch, cz), "w_ag": (ch, cz), "w_b": (ch, cz), "w_bg": (ch, cz), "w_g": (cz, cz),
                  "w_o": (cz, ch), "b_a": (ch,), "b_ag": (ch,), "b_b": (ch,), "b_bg": (ch,), "b_g": (cz,),
                  "b_o": (cz,), "ln_in_w": (cz,), "ln_in_b": (cz,), "ln_out_w": (ch,), "ln_out_b": (ch,)}
        grads = {}
        for f in GRAD_FIELDS:
            grads[f[2:]] = torch.empty(shapes[f[2:]], dtype=torch.float32, device=self.device)
            setattr(g, f, grads[f[2:]].data_ptr())
        dz = torch.empty_like(z)
        trimul_backward(z, mask, p, self.direction, dout, dz, g, stream)
        return dz, grads

    def forward_host(self, z_host, mask_host=None, out_host=None, stream=None):
        """End to end from host memory: copy z (and the mask) in, run, copy out back."""
        import torch
        s = stream or torch.cuda.current_stream()
        with torch.cuda.stream(s):
            z = z_host.to(self.device, non_blocking=True)
            mask = None if mask_host is None else mask_host.to(self.device, non_blocking=True)
            out = self(z, mask, stream=s)
            if out_host is None:
                out_host = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
            out_host.copy_(out, non_blocking=True)
        return out_host


class TriangleMultiplicationOutgoing(_TriangleMultiplication):
    """x_ij = sum_k a_ik * b_jk."""
    direction = OUTGOING


class TriangleMultiplicationIncoming(_TriangleMultiplication):
    """x_ij = sum_k a_ki * b_kj."""
    direction = INCOMING

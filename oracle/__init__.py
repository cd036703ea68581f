"""CPU float64 oracle for the triangle multiplicative update (test infrastructure).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke()``
and by the CPU-baseline leg of ``bench.py``. The product path never imports,
links or runs anything here, and this package imports nothing from the
product package.

The arithmetic lives in ``trimul_oracle.c`` (plain C, double precision, one
function per step of the layer). This module only compiles it with gcc,
marshals numpy arrays and exposes:

  trimul(case, direction)         -> out [N][N][c_z]      (whole layer)
  project(case)                   -> a, b [N][N][c_h]     (LayerNorm, gates, mask)
  contract(a, b, direction)       -> x [N][N][c_h]        (triangle contraction)
  finish(case, x)                 -> out [N][N][c_z]      (output LN, gate, W_o)
  trimul_grid(case, direction, I) -> out [|I|][|I|][c_z]  (cells I x I only)

``case`` is a dict of float32 numpy arrays as made by ``pair_inputs``: z, an
optional mask, the six weights and optional LayerNorm affines and biases.
All functions take ``eps`` (LayerNorm epsilon, default 1e-5) and ``threads``.

Parity unpinned: the value of eps (1e-5, the PyTorch LayerNorm default) and
whether the projections carry biases are readings, not facts the pages fix.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "trimul_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_build", "liboracle.so")
_lock = threading.Lock()
_lib = None

DIRECTIONS = {"outgoing": 0, "incoming": 1, 0: 0, 1: 1}


class _Weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "w_a", "w_ag", "w_b", "w_bg", "w_g", "w_o",
        "b_a", "b_ag", "b_b", "b_bg", "b_g", "b_o",
        "ln_in_w", "ln_in_b", "ln_out_w", "ln_out_b")]


def build(force: bool = False) -> str:
    """Compile trimul_oracle.c into _build/liboracle.so (gcc, -O2)."""
    with _lock:
        stale = (not os.path.exists(_LIB_PATH)
                 or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
        if force or stale:
            os.makedirs(os.path.dirname(_LIB_PATH), exist_ok=True)
            tmp = _LIB_PATH + f".{os.getpid()}.tmp"
            subprocess.check_call(["gcc", "-O2", "-std=c11", "-shared", "-fPIC",
                                   "-o", tmp, _SRC, "-lm", "-lpthread"])
            os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int
        D = ctypes.c_double
        W = ctypes.POINTER(_Weights)
        lib.oracle_project.argtypes = [I, I, I, P, P, W, D, P, P, I]
        lib.oracle_contract.argtypes = [I, I, P, P, I, P, I]
        lib.oracle_finish.argtypes = [I, I, I, P, P, W, D, P, I]
        lib.oracle_trimul.argtypes = [I, I, I, P, P, W, D, I, P, I]
        lib.oracle_trimul_grid.argtypes = [I, I, I, P, P, W, D, I, I, P, P, I]
        for f in (lib.oracle_project, lib.oracle_contract, lib.oracle_finish,
                  lib.oracle_trimul, lib.oracle_trimul_grid):
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


def _threads(threads):
    return int(threads) if threads else (os.cpu_count() or 1)


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


class _Case:
    """Holds float32 copies of a case and the ctypes weight struct."""

    def __init__(self, case: dict):
        self.keep = {}
        z = _f32(case["z"])
        assert z.ndim == 3 and z.shape[0] == z.shape[1], "z must be [N][N][c_z]"
        self.N, self.c_z = z.shape[0], z.shape[2]
        self.c_h = np.asarray(case["w_a"]).shape[0]
        self.z = z
        m = case.get("mask")
        self.mask = None if m is None else _f32(m)
        if self.mask is not None:
            assert self.mask.shape == (self.N, self.N)
        self.w = _Weights()
        for name, _ in _Weights._fields_:
            v = case.get(name)
            if v is None:
                setattr(self.w, name, None)
            else:
                arr = _f32(v)
                self.keep[name] = arr
                setattr(self.w, name, arr.ctypes.data)
        for name in ("w_a", "w_ag", "w_b", "w_bg", "w_g", "w_o"):
            assert name in self.keep, f"missing weight {name}"

    def ptr(self, a):
        return None if a is None else a.ctypes.data


def trimul(case: dict, direction, eps: float = 1e-5, threads=None) -> np.ndarray:
    """The whole layer for every cell: out [N][N][c_z] float64."""
    lib = _load()
    C = _Case(case)
    out = np.empty((C.N, C.N, C.c_z), dtype=np.float64)
    rc = lib.oracle_trimul(C.N, C.c_z, C.c_h, C.ptr(C.z), C.ptr(C.mask), ctypes.byref(C.w),
                           float(eps), DIRECTIONS[direction], out.ctypes.data, _threads(threads))
    if rc:
        raise RuntimeError(f"oracle_trimul failed ({rc})")
    return out


def project(case: dict, eps: float = 1e-5, threads=None):
    """LayerNorm, gated projections and mask: a, b as [N][N][c_h] float64."""
    lib = _load()
    C = _Case(case)
    a = np.empty((C.N, C.N, C.c_h), dtype=np.float64)
    b = np.empty_like(a)
    rc = lib.oracle_project(C.N, C.c_z, C.c_h, C.ptr(C.z), C.ptr(C.mask), ctypes.byref(C.w),
                            float(eps), a.ctypes.data, b.ctypes.data, _threads(threads))
    if rc:
        raise RuntimeError(f"oracle_project failed ({rc})")
    return a, b


def contract(a: np.ndarray, b: np.ndarray, direction, threads=None) -> np.ndarray:
    """Triangle contraction of cell-major a, b ([N][N][c]) into x [N][N][c]."""
    lib = _load()
    a = np.ascontiguousarray(a, dtype=np.float64)
    b = np.ascontiguousarray(b, dtype=np.float64)
    assert a.shape == b.shape and a.ndim == 3 and a.shape[0] == a.shape[1]
    x = np.empty_like(a)
    rc = lib.oracle_contract(a.shape[0], a.shape[2], a.ctypes.data, b.ctypes.data,
                             DIRECTIONS[direction], x.ctypes.data, _threads(threads))
    if rc:
        raise RuntimeError(f"oracle_contract failed ({rc})")
    return x


def finish(case: dict, x: np.ndarray, eps: float = 1e-5, threads=None) -> np.ndarray:
    """Output LayerNorm, gate from z and W_o projection: out [N][N][c_z]."""
    lib = _load()
    C = _Case(case)
    x = np.ascontiguousarray(x, dtype=np.float64)
    assert x.shape == (C.N, C.N, C.c_h)
    out = np.empty((C.N, C.N, C.c_z), dtype=np.float64)
    rc = lib.oracle_finish(C.N, C.c_z, C.c_h, C.ptr(C.z), x.ctypes.data, ctypes.byref(C.w),
                           float(eps), out.ctypes.data, _threads(threads))
    if rc:
        raise RuntimeError(f"oracle_finish failed ({rc})")
    return out


def trimul_grid(case: dict, direction, I, eps: float = 1e-5, threads=None) -> np.ndarray:
    """The layer on the cells I x I only: out [len(I)][len(I)][c_z] float64."""
    lib = _load()
    C = _Case(case)
    I = np.ascontiguousarray(I, dtype=np.int32)
    out = np.empty((len(I), len(I), C.c_z), dtype=np.float64)
    rc = lib.oracle_trimul_grid(C.N, C.c_z, C.c_h, C.ptr(C.z), C.ptr(C.mask), ctypes.byref(C.w),
                                float(eps), DIRECTIONS[direction], len(I), I.ctypes.data,
                                out.ctypes.data, _threads(threads))
    if rc:
        raise RuntimeError(f"oracle_trimul_grid failed ({rc})")
    return out

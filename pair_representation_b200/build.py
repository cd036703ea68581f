"""Builds the CUDA library libtrimul_b200.so in-tree with nvcc for sm_100a.

    python -m pair_representation_b200.build [--verbose-ptxas]

The library links the CUDA runtime statically and fetches driver entry points
at run time, so it loads on a machine without a GPU (its calls then fail with
TRIMUL_ERR_CUDA); only the kernels need a B200.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB_DIR = os.path.join(PKG, "_lib")
LIB = os.path.join(LIB_DIR, "libtrimul_b200.so")
SOURCES = ["api.cu", "prologue_tc.cu", "contract_tc.cu", "epilogue_tc.cu", "simt_f32.cu", "noalloc.cu",
           "backward.cu", "atomattn_tc.cu", "mx_tc.cu"]
HEADERS = ["common.cuh", "kernels.h", "tile_ops.cuh", "mx_block.cuh"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    raise RuntimeError("nvcc not found")


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [
        os.path.join(ROOT, "include", h) for h in ("trimul.h", "atomattn.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, ptxas_verbose: bool = False) -> str:
    if not force and not _stale():
        return LIB
    os.makedirs(LIB_DIR, exist_ok=True)
    tmp = LIB + f".{os.getpid()}.tmp"
    cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
           "-Xcompiler", "-fPIC", "-shared", "-cudart", "static", "-ldl",
           "-I", os.path.join(ROOT, "include"), "-I", CSRC, "-o", tmp]
    if ptxas_verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, f) for f in SOURCES]
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True, ptxas_verbose="--verbose-ptxas" in sys.argv))

"""Build and call tests/csrc/fo_arith_check.cu: GPU checks of the identities
the step kernel's fast path relies on (its own device functions against the
IEEE operations they replace).  Test infrastructure only."""
from __future__ import annotations

import ctypes
import os
import subprocess

from bit_states_b200 import build as fobuild

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "csrc", "fo_arith_check.cu")
OUT = os.path.join(HERE, "_build", "libfo_arith_check.so")
DEPS = [SRC] + [os.path.join(fobuild.CSRC, f) for f in ("fo_codec.cuh", "fo_kernels.cuh")]

_lib = None


def build(force: bool = False) -> str:
    if not force and os.path.exists(OUT) and all(os.path.getmtime(d) <= os.path.getmtime(OUT) for d in DEPS):
        return OUT
    os.makedirs(os.path.dirname(OUT), exist_ok=True)
    tmp = OUT + f".tmp{os.getpid()}"
    cmd = [fobuild.nvcc(), *fobuild.NVCC_FLAGS, "-I", os.path.join(fobuild.ROOT, "include"),
           "-I", fobuild.CSRC, SRC, "-o", tmp]
    subprocess.run(cmd, check=True)
    os.replace(tmp, OUT)
    return OUT


def load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        lib.fo_arith_check.argtypes = [ctypes.c_int, ctypes.c_uint64, ctypes.c_uint64,
                                       ctypes.POINTER(ctypes.c_ulonglong), ctypes.POINTER(ctypes.c_uint32)]
        lib.fo_arith_check.restype = ctypes.c_int
        _lib = lib
    return _lib


def run(which: int, n: int = 0, seed: int = 0):
    """-> (counters[4], examples[16]); raises on a CUDA error."""
    cnt = (ctypes.c_ulonglong * 4)()
    ex = (ctypes.c_uint32 * 16)()
    rc = load().fo_arith_check(which, n, seed, cnt, ex)
    if rc != 0:
        raise RuntimeError(f"fo_arith_check({which}) failed with code {rc}")
    return list(cnt), list(ex)

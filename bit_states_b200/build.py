"""Build libfo.so (the C-ABI library with the sm_100a kernels) in-tree.

nvcc flags that keep the arithmetic exactly as written: no contraction into
FMA (-fmad=false), IEEE division and square root, denormals kept.  The host
side (binary64 scalars) is compiled without floating-point contraction too.
"""
from __future__ import annotations

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
SOURCES = [os.path.join(CSRC, "fo_api.cu")]
DEPS = SOURCES + [os.path.join(CSRC, f) for f in ("fo_codec.cuh", "fo_kernels.cuh")] + \
    [os.path.join(ROOT, "include", "fo.h")]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-lineinfo", "-O3", "-std=c++17",
    "-fmad=false", "-prec-div=true", "-prec-sqrt=true", "-ftz=false",
    "-Xcompiler", "-fPIC,-ffp-contract=off,-fvisibility=hidden",
    "-shared",
]


def lib_path() -> str:
    return os.path.join(HERE, "libfo.so")


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def build(force: bool = False, verbose: bool = False, out: str = "", defines=()) -> str:
    out = out or lib_path()
    if not force and os.path.exists(out):
        t = os.path.getmtime(out)
        if all(os.path.getmtime(d) <= t for d in DEPS):
            return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = [nvcc(), *NVCC_FLAGS, *[f"-D{d}" for d in defines], "-I", os.path.join(ROOT, "include"), "-I", CSRC,
           *SOURCES, "-o", tmp]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    import sys

    print(build(force=True, verbose="-v" in sys.argv))

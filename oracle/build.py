"""Compile the C oracle into ``oracle/libfo_oracle.so`` with gcc.

The flags keep binary32 semantics plain: no contraction of a*b+c into fma,
no fast-math, SSE2 arithmetic (the x86-64 default), no x87 excess precision.
"""
from __future__ import annotations

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "fo_oracle.c")

CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
          "-fexcess-precision=standard", "-fno-finite-math-only", "-pthread"]


def lib_path() -> str:
    return os.path.join(HERE, "libfo_oracle.so")


def build(force: bool = False, src: str = SRC, out: str = "") -> str:
    out = out or lib_path()
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src):
        return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", *CFLAGS, src, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(force=True))

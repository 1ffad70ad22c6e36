"""Device side of the workload generator: builds and binds workloads/libfo_gen.so
(CUDA), which produces the same bits as ``workloads.gen`` on the host."""
from __future__ import annotations

import ctypes
import os
import subprocess

from . import gen

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "csrc", "gen.cu")
LIB = os.path.join(HERE, "libfo_gen.so")

DIST = {"normal": 0, "normal_outliers": 1, "student_t3": 2}

_lib = None


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    nvcc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    tmp = LIB + f".tmp{os.getpid()}"
    subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-fmad=false",
                    "-prec-div=true", "-prec-sqrt=true", "-ftz=false", "-Xcompiler", "-fPIC",
                    "-shared", SRC, "-o", tmp], check=True)
    os.replace(tmp, LIB)
    return LIB


def _load():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB):
            build()
        lib = ctypes.CDLL(LIB)
        P, I, I64, U64, F = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_uint64, ctypes.c_float
        lib.fo_gen_f32.argtypes = [P, I64, I, U64, U64, F, F, F, P]
        lib.fo_gen_f32.restype = I
        lib.fo_gen_16.argtypes = [P, I64, I, U64, U64, F, F, F, I, P]
        lib.fo_gen_16.restype = I
        _lib = lib
    return _lib


def _stream(stream):
    import torch

    return (stream or torch.cuda.current_stream()).cuda_stream


def master_f32(wl, ti: int, out, stream=None):
    """Fill ``out`` (float32 CUDA tensor, numel of tensor ti) with its masters."""
    spec = wl.tensors[ti]
    if spec.init == "const":
        out.fill_(spec.value)
        return out
    key = gen.stream_key(wl.seed, ti, 0, gen.KIND_MASTER)
    rc = _load().fo_gen_f32(out.data_ptr(), out.numel(), 0, key, 0, float(gen.normal_scale(spec.value)),
                            0.0, 1.0, _stream(stream))
    if rc:
        raise RuntimeError(f"fo_gen_f32 failed: cuda error {rc}")
    return out


def grad_16(wl, ti: int, step: int, out, stream=None):
    """Fill ``out`` (int16 CUDA tensor) with the 16-bit gradient patterns of
    tensor ti at ``step``."""
    key = gen.stream_key(wl.seed, ti, step, gen.KIND_GRAD)
    key_o = gen.stream_key(wl.seed, ti, step, gen.KIND_OUTLIER)
    dist = DIST[wl.grad_dist]
    c = float(gen.normal_scale(wl.grad_scale))
    c1 = float(gen.normal_scale(1.0))
    rc = _load().fo_gen_16(out.data_ptr(), out.numel(), dist, key, key_o, c, c1,
                           float(wl.grad_scale), 1 if wl.grad_dtype == "fp16" else 0, _stream(stream))
    if rc:
        raise RuntimeError(f"fo_gen_16 failed: cuda error {rc}")
    return out

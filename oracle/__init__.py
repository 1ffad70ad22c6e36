"""CPU oracle for the FlashOptim-style compressed optimizer step.

TEST INFRASTRUCTURE ONLY: this package may be imported by ``tests/``, by
``__graft_entry__.smoke()`` and by the CPU-baseline leg of ``bench.py``, and
by nothing else.  It wraps ``fo_oracle.c`` (plain scalar C) through ctypes and
shares no code with the CUDA library in ``bit_states_b200``.

All array arguments are numpy arrays in host memory; 16-bit floats travel as
their ``uint16`` bit patterns.  dtype codes: 0 = bf16, 1 = fp16.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from .build import build, lib_path

_lib = None

BF16, FP16 = 0, 1


def bind(lib):
    """Declare the C signatures on a loaded copy of the oracle library."""
    P = ctypes.c_void_p
    I64 = ctypes.c_int64
    I = ctypes.c_int
    D = ctypes.c_double
    lib.oracle_adamw_step.argtypes = [P, P, P, P, P, P, P, I64, I, I, I, D, D, D, D, D, I64, I]
    lib.oracle_sgdm_step.argtypes = [P, P, P, P, P, I64, I, I, I, D, D, D, D, I, I64, I]
    lib.oracle_encode_master.argtypes = [P, P, P, I64, I, I, I]
    lib.oracle_decode_master.argtypes = [P, P, P, I64, I, I, I]
    lib.oracle_downcast.argtypes = [P, P, I64, I, I]
    lib.oracle_widen.argtypes = [P, P, I64, I]
    lib.oracle_scale_fp16.argtypes = [P, P, I64]
    lib.oracle_quantize_state.argtypes = [P, P, P, I64, I]
    lib.oracle_dequantize_state.argtypes = [P, P, P, I64, I]
    lib.oracle_quantize_fixed_scale.argtypes = [P, P, ctypes.c_uint16, I64, I]
    lib.oracle_adamw_scalars.argtypes = [D, D, D, D, D, I64, P]
    for name in ("oracle_adamw_step", "oracle_sgdm_step", "oracle_encode_master",
                 "oracle_decode_master", "oracle_downcast", "oracle_widen",
                 "oracle_scale_fp16", "oracle_quantize_state", "oracle_dequantize_state",
                 "oracle_quantize_fixed_scale", "oracle_adamw_scalars"):
        getattr(lib, name).restype = I
    return lib


def _load():
    global _lib
    if _lib is None:
        path = lib_path()
        if not os.path.exists(path):
            build()
        _lib = bind(ctypes.CDLL(path))
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str):
    if rc != 0:
        raise ValueError(f"oracle {what} rejected its arguments (rc={rc})")


def ecc_dtype(ecc_bits: int):
    return np.int8 if ecc_bits == 8 else np.int16


def n_groups(n: int) -> int:
    return (n + 31) // 32


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


def encode_master(x: np.ndarray, wdt: int = BF16, ecc_bits: int = 8, threads: int = 1):
    """f32 masters -> (downcast bits uint16, ECC codes)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    w = np.empty(x.shape, np.uint16)
    e = np.empty(x.shape, ecc_dtype(ecc_bits))
    _check(_load().oracle_encode_master(_p(x), _p(w), _p(e), x.size, wdt, ecc_bits, threads),
           "encode_master")
    return w, e


def decode_master(w: np.ndarray, e: np.ndarray, wdt: int = BF16, ecc_bits: int = 8,
                  threads: int = 1) -> np.ndarray:
    w = np.ascontiguousarray(w, dtype=np.uint16)
    e = np.ascontiguousarray(e, dtype=ecc_dtype(ecc_bits))
    assert w.shape == e.shape
    x = np.empty(w.shape, np.float32)
    _check(_load().oracle_decode_master(_p(w), _p(e), _p(x), w.size, wdt, ecc_bits, threads),
           "decode_master")
    return x


def downcast(x: np.ndarray, wdt: int = BF16, threads: int = 1) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    w = np.empty(x.shape, np.uint16)
    _check(_load().oracle_downcast(_p(x), _p(w), x.size, wdt, threads), "downcast")
    return w


def widen(w: np.ndarray, wdt: int = BF16) -> np.ndarray:
    w = np.ascontiguousarray(w, dtype=np.uint16)
    x = np.empty(w.shape, np.float32)
    _check(_load().oracle_widen(_p(w), _p(x), w.size, wdt), "widen")
    return x


def scale_fp16(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=np.float32)
    s = np.empty(a.shape, np.uint16)
    _check(_load().oracle_scale_fp16(_p(a), _p(s), a.size), "scale_fp16")
    return s


def quantize_state(z: np.ndarray, kind: int):
    """kind 0: momentum -> int8 codes; kind 1: sqrt(v) -> uint8 codes."""
    z = np.ascontiguousarray(z, dtype=np.float32)
    q = np.empty(z.shape, np.int8 if kind == 0 else np.uint8)
    s = np.empty(n_groups(z.size), np.uint16)
    _check(_load().oracle_quantize_state(_p(z), _p(q), _p(s), z.size, kind), "quantize_state")
    return q, s


def dequantize_state(q: np.ndarray, s: np.ndarray, kind: int) -> np.ndarray:
    """kind 0: momentum m; kind 1: variance v; kind 2: sqrt(v)."""
    q = np.ascontiguousarray(q)
    s = np.ascontiguousarray(s, dtype=np.uint16)
    assert s.size >= n_groups(q.size)
    z = np.empty(q.shape, np.float32)
    _check(_load().oracle_dequantize_state(_p(q), _p(s), _p(z), q.size, kind),
           "dequantize_state")
    return z


def quantize_fixed_scale(z: np.ndarray, S_bits: int, kind: int) -> np.ndarray:
    z = np.ascontiguousarray(z, dtype=np.float32)
    q = np.empty(z.shape, np.int8 if kind == 0 else np.uint8)
    _check(_load().oracle_quantize_fixed_scale(_p(z), _p(q), int(S_bits), z.size, kind),
           "quantize_fixed_scale")
    return q


def adamw_scalars(lr, beta1, beta2, eps, wd, t) -> np.ndarray:
    out = np.empty(8, np.float32)
    _load().oracle_adamw_scalars(lr, beta1, beta2, eps, wd, t, _p(out))
    return out


class State:
    """Compressed optimizer state of one tensor, in host memory."""

    def __init__(self, w, ecc, mq, ms, vq=None, vs=None):
        self.w, self.ecc, self.mq, self.ms, self.vq, self.vs = w, ecc, mq, ms, vq, vs

    @classmethod
    def zeros_like_master(cls, w, ecc, adam: bool = True):
        n = w.size
        ng = n_groups(n)
        mq = np.zeros(n, np.int8)
        ms = np.zeros(ng, np.uint16)
        vq = np.zeros(n, np.uint8) if adam else None
        vs = np.zeros(ng, np.uint16) if adam else None
        return cls(w.copy(), ecc.copy(), mq, ms, vq, vs)

    def copy(self):
        c = lambda a: None if a is None else a.copy()
        return State(c(self.w), c(self.ecc), c(self.mq), c(self.ms), c(self.vq), c(self.vs))


def adamw_step(st: State, grad: np.ndarray, *, lr, beta1, beta2, eps, weight_decay, step,
               wdt=BF16, gdt=BF16, ecc_bits=8, threads=1) -> None:
    """One AdamW step on ``st`` in place; ``grad`` holds 16-bit patterns."""
    grad = np.ascontiguousarray(grad, dtype=np.uint16)
    n = st.w.size
    assert grad.size == n and st.ecc.size == n and st.mq.size == n and st.vq.size == n
    rc = _load().oracle_adamw_step(_p(st.w), _p(st.ecc), _p(grad), _p(st.mq), _p(st.ms),
                                   _p(st.vq), _p(st.vs), n, wdt, gdt, ecc_bits, lr, beta1, beta2,
                                   eps, weight_decay, int(step), threads)
    _check(rc, "adamw_step")


def sgdm_step(st: State, grad: np.ndarray, *, lr, momentum, dampening=0.0, weight_decay=0.0,
              nesterov=False, step, wdt=FP16, gdt=FP16, ecc_bits=8, threads=1) -> None:
    """One SGD-momentum step on ``st`` in place (only the momentum state)."""
    grad = np.ascontiguousarray(grad, dtype=np.uint16)
    n = st.w.size
    assert grad.size == n and st.ecc.size == n and st.mq.size == n
    rc = _load().oracle_sgdm_step(_p(st.w), _p(st.ecc), _p(grad), _p(st.mq), _p(st.ms), n, wdt,
                                  gdt, ecc_bits, lr, momentum, dampening, weight_decay,
                                  int(bool(nesterov)), int(step), threads)
    _check(rc, "sgdm_step")

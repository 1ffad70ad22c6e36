"""ctypes binding of libfo (include/fo.h): argument marshalling only.

Every step of the optimizer runs in the CUDA kernels of libfo.so; this module
turns torch tensors into device pointers and the current CUDA stream into a
``cudaStream_t``.  It never computes on the host and has no fallback: if the
library is missing or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional, Sequence

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libfo.so")

FO_OK = 0
FO_DT_BF16 = 0
FO_DT_FP16 = 1
_DT = {"bf16": FO_DT_BF16, "fp16": FO_DT_FP16}


class FoError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        self.status = status
        super().__init__(f"{where}: {detail}")


class fo_tensor(ctypes.Structure):
    _fields_ = [("w", ctypes.c_void_p), ("ecc", ctypes.c_void_p), ("grad", ctypes.c_void_p),
                ("m_q", ctypes.c_void_p), ("m_scale", ctypes.c_void_p), ("v_q", ctypes.c_void_p),
                ("v_scale", ctypes.c_void_p), ("numel", ctypes.c_int64)]


class fo_adamw_hparams(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_double), ("beta1", ctypes.c_double), ("beta2", ctypes.c_double),
                ("eps", ctypes.c_double), ("weight_decay", ctypes.c_double), ("step", ctypes.c_int64)]


class fo_sgdm_hparams(ctypes.Structure):
    _fields_ = [("lr", ctypes.c_double), ("momentum", ctypes.c_double),
                ("dampening", ctypes.c_double), ("weight_decay", ctypes.c_double),
                ("nesterov", ctypes.c_int), ("step", ctypes.c_int64)]


class fo_format(ctypes.Structure):
    _fields_ = [("w_dtype", ctypes.c_int), ("grad_dtype", ctypes.c_int), ("ecc_bits", ctypes.c_int)]


EXPORTS = ("fo_adamw_step", "fo_sgdm_step", "fo_stream_copy", "fo_encode_master", "fo_decode_master",
           "fo_check_errors", "fo_status_string", "fo_last_error", "fo_version")

_lib = None


def load(path: str = LIB_PATH):
    """Load libfo.so (once).  Raises if it is missing: there is no fallback."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise FoError(-1, "libfo", f"{path} not built (run bit_states_b200/build.py)")
    lib = ctypes.CDLL(path)
    P, I, I64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64
    lib.fo_adamw_step.argtypes = [ctypes.POINTER(fo_tensor), I, fo_format,
                                  ctypes.POINTER(fo_adamw_hparams), P]
    lib.fo_sgdm_step.argtypes = [ctypes.POINTER(fo_tensor), I, fo_format,
                                 ctypes.POINTER(fo_sgdm_hparams), P]
    lib.fo_stream_copy.argtypes = [ctypes.POINTER(fo_tensor), I, fo_format, I, P]
    lib.fo_encode_master.argtypes = [P, P, P, I64, fo_format, P]
    lib.fo_decode_master.argtypes = [P, P, P, I64, fo_format, P]
    lib.fo_check_errors.argtypes = [P]
    for n in ("fo_adamw_step", "fo_sgdm_step", "fo_stream_copy", "fo_encode_master", "fo_decode_master",
              "fo_check_errors"):
        getattr(lib, n).restype = I
    lib.fo_status_string.argtypes = [I]
    lib.fo_status_string.restype = ctypes.c_char_p
    lib.fo_last_error.argtypes = []
    lib.fo_last_error.restype = ctypes.c_char_p
    lib.fo_version.argtypes = []
    lib.fo_version.restype = I
    _lib = lib
    return lib


def _check(rc: int, where: str):
    if rc != FO_OK:
        lib = load()
        raise FoError(rc, where, f"{lib.fo_status_string(rc).decode()}: {lib.fo_last_error().decode()}")


def make_format(w_dtype="bf16", grad_dtype="bf16", ecc_bits=8) -> fo_format:
    return fo_format(_DT[w_dtype], _DT[grad_dtype], int(ecc_bits))


def _stream_handle(stream) -> Optional[int]:
    if stream is None:
        import torch

        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _ptr(t) -> int:
    return 0 if t is None else t.data_ptr()


@dataclass
class TensorState:
    """Device buffers of one parameter tensor (torch tensors, caller-owned)."""
    w: object
    ecc: object
    m_q: object
    m_scale: object
    v_q: object = None
    v_scale: object = None

    @property
    def numel(self) -> int:
        return self.w.numel()

    def desc(self, grad) -> fo_tensor:
        assert grad.numel() == self.numel
        return fo_tensor(_ptr(self.w), _ptr(self.ecc), _ptr(grad), _ptr(self.m_q), _ptr(self.m_scale),
                         _ptr(self.v_q), _ptr(self.v_scale), self.numel)


def descriptors(states: Sequence[TensorState], grads: Sequence) -> ctypes.Array:
    arr = (fo_tensor * max(1, len(states)))()
    for i, (s, g) in enumerate(zip(states, grads)):
        arr[i] = s.desc(g)
    return arr


def fo_adamw_step(descs, n_tensors: int, fmt: fo_format, h: fo_adamw_hparams, stream=None):
    _check(load().fo_adamw_step(descs, n_tensors, fmt, ctypes.byref(h), _stream_handle(stream)),
           "fo_adamw_step")


def fo_sgdm_step(descs, n_tensors: int, fmt: fo_format, h: fo_sgdm_hparams, stream=None):
    _check(load().fo_sgdm_step(descs, n_tensors, fmt, ctypes.byref(h), _stream_handle(stream)),
           "fo_sgdm_step")


def fo_stream_copy(descs, n_tensors: int, fmt: fo_format, adamw_mix: bool = True, stream=None):
    """The step's byte traffic without its arithmetic (a bandwidth ceiling)."""
    _check(load().fo_stream_copy(descs, n_tensors, fmt, int(bool(adamw_mix)), _stream_handle(stream)),
           "fo_stream_copy")


def fo_encode_master(x32, w, ecc, n: int, fmt: fo_format, stream=None):
    _check(load().fo_encode_master(_ptr(x32), _ptr(w), _ptr(ecc), int(n), fmt, _stream_handle(stream)),
           "fo_encode_master")


def fo_decode_master(w, ecc, x32, n: int, fmt: fo_format, stream=None):
    _check(load().fo_decode_master(_ptr(w), _ptr(ecc), _ptr(x32), int(n), fmt, _stream_handle(stream)),
           "fo_decode_master")


def fo_check_errors(stream=None):
    """Wait for ``stream`` and raise if a step kernel gave up a bounded wait
    for a staged copy since the last check (its chunks were not stepped)."""
    _check(load().fo_check_errors(_stream_handle(stream)), "fo_check_errors")


def fo_version() -> int:
    return load().fo_version()

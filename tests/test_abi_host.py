"""Host-side tests of the C ABI (no GPU needed): the library loads, exports
every symbol that include/fo.h declares, and rejects bad arguments on the
host before any CUDA call, with a status and a one-line explanation."""
import ctypes
import os
import re

import pytest

from bit_states_b200 import build as fobuild
from bit_states_b200 import fo

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    fobuild.build()
    return fo.load()


def _declared():
    names = set()
    inc = os.path.join(ROOT, "include")
    for f in os.listdir(inc):
        if f.endswith(".h"):
            txt = open(os.path.join(inc, f)).read()
            names |= set(re.findall(r"FO_API\s+[\w\s\*]+?\b(fo_\w+)\s*\(", txt))
    return names


def test_exports_every_declared_symbol(lib):
    names = _declared()
    assert {"fo_adamw_step", "fo_sgdm_step", "fo_encode_master", "fo_decode_master"} <= names
    for n in names:
        assert hasattr(lib, n), n
    import subprocess

    out = subprocess.run(["nm", "-D", "--defined-only", fo.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r"\bT (fo_\w+)", out))
    assert names <= exported


def test_version_and_status_strings(lib):
    assert lib.fo_version() >= 100
    assert lib.fo_status_string(0) == b"FO_OK"
    assert lib.fo_status_string(5) == b"FO_ERR_CUDA"
    assert lib.fo_status_string(6) == b"FO_ERR_TIMEOUT"


def _hp(**kw):
    d = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01, step=1)
    d.update(kw)
    return fo.fo_adamw_hparams(d["lr"], d["beta1"], d["beta2"], d["eps"], d["weight_decay"], d["step"])


def _t(numel=64, base=0x10000000, **over):
    d = dict(w=base, ecc=base + 0x1000, grad=base + 0x2000, m_q=base + 0x3000, m_scale=base + 0x4000,
             v_q=base + 0x5000, v_scale=base + 0x6000, numel=numel)
    d.update(over)
    return fo.fo_tensor(d["w"], d["ecc"], d["grad"], d["m_q"], d["m_scale"], d["v_q"], d["v_scale"],
                        d["numel"])


def _call_adamw(lib, tensors, fmt=None, hp=None, n=None):
    arr = (fo.fo_tensor * max(1, len(tensors)))(*tensors)
    fmt = fmt or fo.make_format()
    hp = hp if hp is not None else _hp()
    return lib.fo_adamw_step(arr, len(tensors) if n is None else n, fmt, ctypes.byref(hp), None)


@pytest.mark.parametrize("case,status", [
    ("bad_wdt", 2), ("bad_ecc", 2), ("null_h", 1), ("step0", 1), ("beta1", 1), ("nan_lr", 1),
    ("neg_numel", 1), ("null_grad", 1), ("null_v", 1), ("odd_w", 3), ("odd_scale", 3),
    ("odd_ecc16", 3), ("neg_n", 1), ("too_many", 4), ("null_array", 1), ("huge_numel", 1),
])
def test_adamw_rejects_on_host(lib, case, status):
    t = [_t()]
    fmt, hp, n = None, None, None
    if case == "bad_wdt":
        fmt = fo.fo_format(7, 0, 8)
    elif case == "bad_ecc":
        fmt = fo.make_format(ecc_bits=12)
    elif case == "step0":
        hp = _hp(step=0)
    elif case == "beta1":
        hp = _hp(beta1=1.0)
    elif case == "nan_lr":
        hp = _hp(lr=float("nan"))
    elif case == "neg_numel":
        t = [_t(numel=-1)]
    elif case == "huge_numel":
        t = [_t(numel=(1 << 36) + 1)]
    elif case == "null_grad":
        t = [_t(grad=0)]
    elif case == "null_v":
        t = [_t(v_q=0)]
    elif case == "odd_w":
        t = [_t(w=0x10000001)]
    elif case == "odd_scale":
        t = [_t(m_scale=0x10004001)]
    elif case == "odd_ecc16":
        fmt = fo.make_format(ecc_bits=16)
        t = [_t(ecc=0x10001001)]
    elif case == "neg_n":
        n = -1
    elif case == "too_many":
        n = (1 << 20) + 1
    if case == "null_h":
        arr = (fo.fo_tensor * 1)(*t)
        rc = lib.fo_adamw_step(arr, 1, fo.make_format(), None, None)
    elif case == "null_array":
        rc = lib.fo_adamw_step(None, 3, fo.make_format(), ctypes.byref(_hp()), None)
    elif case == "too_many":
        rc = lib.fo_adamw_step(None, n, fo.make_format(), ctypes.byref(_hp()), None)
    else:
        rc = _call_adamw(lib, t, fmt, hp, n)
    assert rc == status, (case, rc, lib.fo_last_error())
    assert lib.fo_last_error() != b""


def test_empty_calls_are_noops(lib):
    # n_tensors == 0 and all-empty tensors return before touching CUDA
    assert _call_adamw(lib, [], n=0) == 0
    assert _call_adamw(lib, [_t(numel=0, w=0, ecc=0, grad=0, m_q=0, m_scale=0, v_q=0, v_scale=0)]) == 0
    assert lib.fo_encode_master(None, None, None, 0, fo.make_format(), None) == 0
    assert lib.fo_decode_master(None, None, None, 0, fo.make_format(), None) == 0
    assert lib.fo_last_error() == b""


def test_sgdm_and_codec_reject_on_host(lib):
    arr = (fo.fo_tensor * 1)(_t(v_q=0, v_scale=0))
    bad = fo.fo_sgdm_hparams(0.1, 1.5, 0.0, 0.0, 0, 1)
    assert lib.fo_sgdm_step(arr, 1, fo.make_format("fp16", "fp16"), ctypes.byref(bad), None) == 1
    bad = fo.fo_sgdm_hparams(0.1, 0.9, 0.0, 0.0, 0, 0)
    assert lib.fo_sgdm_step(arr, 1, fo.make_format("fp16", "fp16"), ctypes.byref(bad), None) == 1
    assert lib.fo_encode_master(None, None, None, 5, fo.make_format(), None) == 1
    assert lib.fo_encode_master(0x1002, 0x2000, 0x3000, 5, fo.make_format(), None) == 3
    assert lib.fo_decode_master(0x2001, 0x3000, 0x4000, 5, fo.make_format(), None) == 3
    assert lib.fo_decode_master(0x2000, 0x3000, 0x4000, -1, fo.make_format(), None) == 1
    assert lib.fo_encode_master(0x1000, 0x2000, 0x3000, 5, fo.fo_format(0, 0, 4), None) == 2


def test_binding_raises_without_library(tmp_path):
    saved = fo._lib
    fo._lib = None
    try:
        with pytest.raises(fo.FoError):
            fo.load(str(tmp_path / "missing.so"))
    finally:
        fo._lib = saved


def test_stream_copy_rejects_on_host(lib):
    arr = (fo.fo_tensor * 1)(_t())
    assert lib.fo_stream_copy(arr, 1, fo.fo_format(0, 0, 4), 1, None) == 2           # ECC width
    assert lib.fo_stream_copy(None, 3, fo.make_format(), 1, None) == 1              # NULL table
    odd = (fo.fo_tensor * 1)(_t(w=0x1001))
    assert lib.fo_stream_copy(odd, 1, fo.make_format(), 1, None) == 3               # alignment
    no_v = (fo.fo_tensor * 1)(_t(v_q=0, v_scale=0))
    assert lib.fo_stream_copy(no_v, 1, fo.make_format(), 1, None) == 1              # AdamW mix needs v
    assert lib.fo_stream_copy(arr, 0, fo.make_format(), 1, None) == 0               # no-op
    assert lib.fo_stream_copy((fo.fo_tensor * 1)(_t(numel=0, w=0, ecc=0, grad=0, m_q=0, m_scale=0, v_q=0,
                                                     v_scale=0)), 1, fo.make_format(), 0, None) == 0

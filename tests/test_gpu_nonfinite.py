"""GPU parity for non-finite inputs and saturated group scales.

The reading for non-finite values (the pages are silent; gradients kept in
backward precision, per Davis Blalock's FlashOptim release thread, overflow to
inf in fp16 training): a NaN downcasts to the positive quiet NaN of the format
(bf16 0x7FC0, fp16 0x7E00) with ECC 0, inf and NaN state values stay out of
their group's maximum and get code 0, and the rest is IEEE binary32.

Blocks of whole staged chunks (each exercising the kernel's fast path and its
checks) plus a ragged tail (the scalar path):
  * ordinary values;
  * +-inf and NaN gradients (several NaN payloads and both signs) at random
    elements;
  * NaN and inf weights in the input state;
  * gradients large enough that a group's largest |m'| or sqrt(v') exceeds
    65504, the largest fp16 scale (the scale saturates and codes must clamp to
    +-127 / 255; a fast path that only keeps the low byte of the code would
    wrap them);
  * fp16 weights at the largest finite value, pushed past 65520 (they round
    to inf).
Both optimizers, every weight / gradient dtype and both ECC widths; several
steps, including late steps where the bias corrections are close to one.
Every emitted byte must equal the oracle's.
"""
import numpy as np
import pytest
import torch

import oracle
from bit_states_b200 import fo

import gpu_util as U

pytestmark = pytest.mark.gpu

DEV = "cuda"
CHUNK = 1536  # a whole number of staged chunks of every launch geometry
F32 = np.float32
NAN_PATTERNS = np.array([0x7FC00000, 0xFFC00000, 0x7F800001, 0xFFBFFFFF, 0x7FFFFFFF], np.uint32)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    from bit_states_b200 import build as fobuild

    fobuild.build()
    fo.load()
    yield
    torch.cuda.synchronize()


NAN16 = {"bf16": np.array([0x7FC0, 0xFFC0, 0x7F81, 0xFFFF, 0x7FA5], np.uint16),
         "fp16": np.array([0x7E00, 0xFE00, 0x7C01, 0xFFFF, 0x7D55], np.uint16)}


def _to16(x32: np.ndarray, dt: str, r) -> np.ndarray:
    """16-bit gradient patterns: finite values and inf by the oracle's
    downcast, NaNs as assorted NaN patterns of both signs and payloads."""
    g = oracle.downcast(np.ascontiguousarray(x32, F32), 0 if dt == "bf16" else 1)
    k = np.nonzero(np.isnan(x32))[0]
    g[k] = NAN16[dt][r.integers(0, NAN16[dt].size, k.size)]
    return g


def _sprinkle(g: np.ndarray, r, frac: float) -> np.ndarray:
    g = g.copy()
    k = np.nonzero(r.random(g.size) < frac)[0]
    pick = r.integers(0, 3, k.size)
    nans = NAN_PATTERNS[r.integers(0, NAN_PATTERNS.size, k.size)].view(F32)
    g[k] = np.where(pick == 0, F32(np.inf), np.where(pick == 1, F32(-np.inf), nans))
    return g


def _blocks(rng, wdt, gdt, optimizer):
    gmax = 6.0e4 if gdt == "fp16" else 3.0e6
    blocks = []

    def ordinary(r):
        return (r.standard_normal(CHUNK) * 1e-3).astype(F32)

    def nx():
        return (rng.standard_normal(CHUNK) * 0.02).astype(F32)

    blocks.append(("ordinary", nx(), None, ordinary))
    blocks.append(("nonfinite grads", nx(), None, lambda r: _sprinkle(ordinary(r), r, 0.03)))
    blocks.append(("all-nonfinite group", nx(), None,
                   lambda r: np.where(np.arange(CHUNK) // 32 == 3, F32(np.inf), ordinary(r)).astype(F32)))
    wbad = np.zeros(CHUNK, np.uint16)
    wbad[::7] = 1  # marks: replaced by NaN / inf patterns below
    blocks.append(("nonfinite weights", nx(), wbad, ordinary))
    # huge finite gradients: scales saturate at 65504 (m' alone for SGD)
    blocks.append(("saturating grads", nx(), None,
                   lambda r: (r.standard_normal(CHUNK) * (gmax / 3)).clip(-gmax, gmax).astype(F32)))
    blocks.append(("few saturating", nx(), None,
                   lambda r: np.where(r.random(CHUNK) < 0.01, F32(gmax), ordinary(r)).astype(F32)))
    if wdt == "fp16":
        big = np.where(rng.random(CHUNK) < 0.5, F32(65504.0), F32(-65504.0)).astype(F32)
        blocks.append(("fp16 max weights", big, None,
                       lambda r, b=big: (-np.sign(b) * (1e4 if optimizer == "sgdm" else 1e-3)).astype(F32)))
    return blocks


def _setup(wdt, gdt, nbits, optimizer, seed):
    rng = np.random.default_rng(seed)
    blocks = _blocks(rng, wdt, gdt, optimizer)
    tail = 45
    x = np.concatenate([b[1] for b in blocks] + [(rng.standard_normal(tail) * 0.02).astype(F32)])
    n = x.size
    wcode = 0 if wdt == "bf16" else 1
    w, e = oracle.encode_master(x, wcode, nbits)
    off = 0
    for name, _, wbad, _ in blocks:
        if wbad is not None:
            k = np.nonzero(wbad)[0] + off
            pats = ([0xFFC1, 0x7F81, 0x7F80, 0xFF80] if wdt == "bf16" else [0xFE05, 0x7C01, 0x7C00, 0xFC00])
            w[k] = np.resize(np.array(pats, np.uint16), k.size)
        off += CHUNK
    adam = optimizer == "adamw"
    st = oracle.State.zeros_like_master(w, e, adam=adam)
    ng = (n + 31) // 32
    d = fo.TensorState(torch.from_numpy(w.view(np.int16).copy()).to(DEV), torch.from_numpy(e.copy()).to(DEV),
                       torch.zeros(n, dtype=torch.int8, device=DEV), torch.zeros(ng, dtype=torch.int16, device=DEV),
                       torch.zeros(n, dtype=torch.uint8, device=DEV) if adam else None,
                       torch.zeros(ng, dtype=torch.int16, device=DEV) if adam else None)
    return blocks, tail, n, st, d


def _grads(blocks, tail, r):
    return np.concatenate([b[3](r) for b in blocks] + [_sprinkle((r.standard_normal(tail) * 1e-3).astype(F32),
                                                                 r, 0.1)])


def _compare(d, st, t, adam):
    pairs = [("w", U.to_np_bytes(d.w), st.w.view(np.uint16)), ("ecc", d.ecc.cpu().numpy(), st.ecc),
             ("m_q", d.m_q.cpu().numpy(), st.mq), ("m_scale", U.to_np_bytes(d.m_scale), st.ms.view(np.uint16))]
    if adam:
        pairs += [("v_q", d.v_q.cpu().numpy(), st.vq), ("v_scale", U.to_np_bytes(d.v_scale), st.vs.view(np.uint16))]
    for name, got, exp in pairs:
        bad = np.nonzero(got.view(exp.dtype) != exp)[0]
        assert bad.size == 0, f"step {t} {name}: {bad.size} mismatches, first at {bad[:6]}: " \
                              f"got {got.view(exp.dtype)[bad[:6]]} expected {exp[bad[:6]]}"


FORMATS = [(w, g, nb) for w in ("bf16", "fp16") for g in ("bf16", "fp16") for nb in (8, 16)]


@pytest.mark.parametrize("t0", [1, 1000])
@pytest.mark.parametrize("wdt,gdt,nbits", FORMATS)
def test_adamw_nonfinite_and_saturating_every_byte(wdt, gdt, nbits, t0):
    blocks, tail, n, st, d = _setup(wdt, gdt, nbits, "adamw", 7 + nbits + t0)
    hp = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01)
    fmt = fo.make_format(wdt, gdt, nbits)
    gv = torch.zeros(n, dtype=torch.int16, device=DEV)
    wc, gc = (0 if wdt == "bf16" else 1), (0 if gdt == "bf16" else 1)
    for t in range(t0, t0 + 4):
        r = np.random.default_rng(100 * t + nbits)
        gb = _to16(_grads(blocks, tail, r), gdt, r)
        gv.copy_(torch.from_numpy(gb.view(np.int16)))
        fo.fo_adamw_step(fo.descriptors([d], [gv]), 1, fmt, fo.fo_adamw_hparams(**hp, step=t))
        oracle.adamw_step(st, gb, **hp, step=t, wdt=wc, gdt=gc, ecc_bits=nbits)
        torch.cuda.synchronize()
        _compare(d, st, t, True)


@pytest.mark.parametrize("nesterov", [False, True])
@pytest.mark.parametrize("wdt,gdt,nbits", FORMATS)
def test_sgdm_nonfinite_and_saturating_every_byte(wdt, gdt, nbits, nesterov):
    blocks, tail, n, st, d = _setup(wdt, gdt, nbits, "sgdm", 31 + nbits + 2 * nesterov)
    hp = dict(lr=0.1, momentum=0.9, dampening=0.0, weight_decay=1e-4, nesterov=nesterov)
    fmt = fo.make_format(wdt, gdt, nbits)
    gv = torch.zeros(n, dtype=torch.int16, device=DEV)
    wc, gc = (0 if wdt == "bf16" else 1), (0 if gdt == "bf16" else 1)
    for t in range(1, 5):
        r = np.random.default_rng(300 * t + nbits)
        gb = _to16(_grads(blocks, tail, r), gdt, r)
        gv.copy_(torch.from_numpy(gb.view(np.int16)))
        fo.fo_sgdm_step(fo.descriptors([d], [gv]), 1, fmt,
                        fo.fo_sgdm_hparams(hp["lr"], hp["momentum"], hp["dampening"], hp["weight_decay"],
                                           int(nesterov), t))
        oracle.sgdm_step(st, gb, **hp, step=t, wdt=wc, gdt=gc, ecc_bits=nbits)
        torch.cuda.synchronize()
        _compare(d, st, t, False)


@pytest.mark.parametrize("wdt,nbits", [("bf16", 8), ("bf16", 16), ("fp16", 8), ("fp16", 16)])
def test_encode_master_nan_is_canonical(wdt, nbits):
    rng = np.random.default_rng(9)
    n = 4096 + 5
    x = (rng.standard_normal(n) * 0.02).astype(F32)
    x[::5] = NAN_PATTERNS[rng.integers(0, NAN_PATTERNS.size, x[::5].size)].view(F32)
    x[1::11] = np.inf
    x[2::13] = -np.inf
    w, e = oracle.encode_master(x, 0 if wdt == "bf16" else 1, nbits)
    xd = torch.from_numpy(x).to(DEV)
    wd = torch.empty(n, dtype=torch.int16, device=DEV)
    ed = torch.empty(n, dtype=torch.int8 if nbits == 8 else torch.int16, device=DEV)
    fo.fo_encode_master(xd, wd, ed, n, fo.make_format(wdt, "bf16", nbits))
    torch.cuda.synchronize()
    assert np.array_equal(U.to_np_bytes(wd), w)
    assert np.array_equal(ed.cpu().numpy(), e)

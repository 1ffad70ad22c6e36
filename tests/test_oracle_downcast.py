"""Pins of the oracle's round-to-nearest-even downcast against library casts.

The downcast is the base weight x' of the weight split ("FlashOptim:
Breaking the Memory Wall ...", section "1. ULP-based Weight Splitting").
torch's float32 -> bfloat16 cast and numpy's float32 -> float16 cast both
round to nearest even, so they give the expected patterns independently of
the oracle.
"""
import numpy as np
import pytest
import torch

from conftest import threads

BF16, FP16 = 0, 1


def _lib_bf16(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _lib_fp16(x: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        return x.astype(np.float16).view(np.uint16)


def _is_nan_bits(b: np.ndarray, wdt: int) -> np.ndarray:
    if wdt == BF16:
        return ((b & 0x7F80) == 0x7F80) & ((b & 0x7F) != 0)
    return ((b & 0x7C00) == 0x7C00) & ((b & 0x3FF) != 0)


def _compare(orc, pats: np.ndarray, wdt: int):
    x = pats.view(np.float32)
    got = orc.downcast(x, wdt, threads=threads())
    exp = _lib_bf16(x) if wdt == BF16 else _lib_fp16(x)
    nan = np.isnan(x)
    # NaN: the libraries disagree on sign and payload (torch's bf16 cast gives
    # 0xFFFF, torch's fp16 cast and numpy keep sign and payload bits); the
    # reading fixes one positive quiet NaN with only the quiet bit set
    assert np.all(_is_nan_bits(got[nan], wdt))
    assert np.all(got[nan] == (0x7FC0 if wdt == BF16 else 0x7E00))
    bad = np.nonzero(got[~nan] != exp[~nan])[0]
    assert bad.size == 0, f"{bad.size} mismatches, first x={x[~nan][bad[:4]]}"


def _structured_patterns() -> np.ndarray:
    """Every 16-bit head with the low halves that decide bf16 rounding, and
    every exponent with the mantissa tails that decide fp16 rounding."""
    heads = np.arange(1 << 16, dtype=np.uint32) << 16
    lows = np.array([0, 1, 0x7FFF, 0x8000, 0x8001, 0xFFFF, 0x4000, 0xC000, 0x1234], np.uint32)
    a = (heads[:, None] | lows[None, :]).ravel()
    # fp16 rounding is decided by the low 13 bits of the f32 mantissa; for
    # fp16 subnormals by more.  Sweep every exponent with dense tails.
    exps = np.arange(256, dtype=np.uint32) << 23
    tails = np.concatenate([np.arange(0, 1 << 13, dtype=np.uint32),
                            np.arange(0, 1 << 23, 4099, dtype=np.uint32)])
    b = (exps[:, None] | tails[None, :]).ravel()
    b = np.concatenate([b, b | np.uint32(0x80000000)])
    rng = np.random.default_rng(1)
    c = rng.integers(0, 1 << 32, size=1 << 20, dtype=np.uint64).astype(np.uint32)
    return np.concatenate([a, b, c])


@pytest.mark.parametrize("wdt", [BF16, FP16])
def test_downcast_structured(orc, wdt):
    _compare(orc, _structured_patterns(), wdt)


@pytest.mark.parametrize("wdt", [BF16, FP16])
def test_downcast_special_values(orc, wdt):
    vals = np.array([0.0, -0.0, np.inf, -np.inf, 1.0, -1.0, 65504.0, 65519.99, 65520.0, 3.4e38,
                     3.3895e38, 1e-45, 5.96e-8, 2.98e-8, 2.9802322e-08, 1.1754944e-38], np.float32)
    _compare(orc, vals.view(np.uint32).copy(), wdt)


@pytest.mark.exhaustive
@pytest.mark.parametrize("wdt", [BF16, FP16])
def test_downcast_all_2_32(orc, wdt):
    step = 1 << 26
    for start in range(0, 1 << 32, step):
        pats = np.arange(start, start + step, dtype=np.uint64).astype(np.uint32)
        _compare(orc, pats, wdt)

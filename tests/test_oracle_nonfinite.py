"""Pins of the oracle's reading for non-finite values.

The pages are silent on inf and NaN.  Gradients kept in backward precision
(Davis Blalock's FlashOptim release thread, the post on gradients) overflow to
inf in fp16 mixed-precision training, so a step must still give a defined
result.  The reading: a NaN downcasts to the positive quiet NaN of the format
(bf16 0x7FC0, fp16 0x7E00) with ECC 0; inf and NaN state values are left out
of their group's maximum and stored as code 0; the rest is IEEE binary32
arithmetic.

What fixes the expected values independently of the oracle's handling of
non-finite numbers:
  * quantizing a group with some entries inf / NaN equals quantizing it with
    those entries replaced by zero (zero never raises a maximum and has code 0);
  * a step in which element k receives a non-finite gradient equals, on every
    byte outside element k's weight and ECC, a step in which element k has a
    zero gradient and zero state (its m' and v' are then zero: code 0, no
    contribution to the scale), while element k's weight is fixed by IEEE
    arithmetic: AdamW gives m'/den = inf/inf or NaN, so x'' is NaN; SGD with
    momentum from a zero state gives x'' = -lr * (+-inf) = -+inf;
  * an fp16 master pushed past 65520 rounds to inf (numpy's cast) with ECC 0;
    AdamW keeps it inf, SGD's coupled decay turns it into NaN (0 * inf).
"""
import numpy as np
import pytest

BF16, FP16 = 0, 1
QNAN = {BF16: 0x7FC0, FP16: 0x7E00}
INF = {BF16: 0x7F80, FP16: 0x7C00}
HP = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01)


def _bits16(x: np.ndarray, dt: int) -> np.ndarray:
    """16-bit patterns of f32 values (exactly representable) via the oracle's
    own widening checked against numpy / bit shifts."""
    x = np.asarray(x, np.float32)
    if dt == FP16:
        with np.errstate(over="ignore", invalid="ignore"):
            return x.astype(np.float16).view(np.uint16)
    return (x.view(np.uint32) >> 16).astype(np.uint16)


NONFINITE = np.array([np.inf, -np.inf, np.nan], np.float32)


@pytest.mark.parametrize("kind", [0, 1])
def test_nonfinite_state_values_stay_out_of_the_scale(orc, kind):
    oracle = orc
    rng = np.random.default_rng(5)
    n = 32 * 400 + 13
    z = (rng.standard_t(3, n) * 1e-3).astype(np.float32)
    if kind == 1:
        z = np.abs(z)
    hit = rng.random(n) < 0.05
    zz = z.copy()
    zz[hit] = rng.choice(NONFINITE if kind == 0 else np.array([np.inf, np.nan], np.float32), hit.sum())
    # a group made only of non-finite values has scale 0
    zz[32:64] = np.inf
    z[32:64] = 0.0
    q, s = oracle.quantize_state(zz, kind)
    z0 = np.where(np.isfinite(zz), zz, np.float32(0.0)).astype(np.float32)
    q0, s0 = oracle.quantize_state(z0, kind)
    assert np.array_equal(s, s0)
    assert np.array_equal(q, q0)
    assert np.all(q[hit] == 0)
    assert s[1] == 0
    # the scale is fp16 rounded up of the finite maximum (numpy's neighbours)
    A = np.array([np.max(np.abs(g[np.isfinite(g)]), initial=0.0) for g in np.split(
        np.pad(zz, (0, (-n) % 32)), (n + 31) // 32)], np.float64)
    S = s.view(np.float16).astype(np.float64)
    assert np.all(S >= A)
    below = np.nextafter(s.view(np.float16), np.float16(0)).astype(np.float64)
    assert np.all(below[A > 0] < A[A > 0])


def _state(oracle, n, wdt, nbits, adam, rng):
    x = (rng.standard_normal(n) * 0.02).astype(np.float32)
    w, e = oracle.encode_master(x, wdt, nbits)
    return oracle.State.zeros_like_master(w, e, adam=adam)


@pytest.mark.parametrize("nbits", [8, 16])
@pytest.mark.parametrize("wdt,gdt", [(BF16, BF16), (FP16, FP16), (BF16, FP16), (FP16, BF16)])
def test_adamw_nonfinite_gradient_poisons_only_its_element(orc, wdt, gdt, nbits):
    oracle = orc
    rng = np.random.default_rng(11 + wdt + 2 * gdt + nbits)
    n = 32 * 50 + 7
    st = _state(oracle, n, wdt, nbits, True, rng)
    # populate the state with a few ordinary steps first
    for t in (1, 2):
        g = _bits16((rng.standard_normal(n) * 1e-3).astype(np.float32), gdt)
        oracle.adamw_step(st, g, **HP, step=t, wdt=wdt, gdt=gdt, ecc_bits=nbits)
    k = np.sort(rng.choice(n, 40, replace=False))
    ref = st.copy()
    ref.mq[k] = 0
    ref.vq[k] = 0
    st.mq[k] = 0
    st.vq[k] = 0
    for t in (3, 4, 5):
        g32 = (rng.standard_normal(n) * 1e-3).astype(np.float32)
        gbad = g32.copy()
        gbad[k] = np.resize(NONFINITE, k.size)
        g32[k] = 0.0
        oracle.adamw_step(st, _bits16(gbad, gdt), **HP, step=t, wdt=wdt, gdt=gdt, ecc_bits=nbits)
        oracle.adamw_step(ref, _bits16(g32, gdt), **HP, step=t, wdt=wdt, gdt=gdt, ecc_bits=nbits)
        other = np.ones(n, bool)
        other[k] = False
        assert np.array_equal(st.w[other], ref.w[other])
        assert np.array_equal(st.ecc[other], ref.ecc[other])
        for a, b in ((st.mq, ref.mq), (st.vq, ref.vq), (st.ms, ref.ms), (st.vs, ref.vs)):
            assert np.array_equal(a, b)
        assert np.all(st.w[k] == QNAN[wdt])
        assert np.all(st.ecc[k] == 0)


@pytest.mark.parametrize("nesterov", [False, True])
@pytest.mark.parametrize("wdt,gdt", [(FP16, FP16), (BF16, BF16)])
def test_sgdm_nonfinite_gradient_poisons_only_its_element(orc, wdt, gdt, nesterov):
    oracle = orc
    rng = np.random.default_rng(21 + wdt + 2 * nesterov)
    n = 32 * 40 + 3
    st = _state(oracle, n, wdt, 8, False, rng)
    k = np.sort(rng.choice(n, 30, replace=False))
    ref = st.copy()
    h = dict(lr=0.1, momentum=0.9, dampening=0.0, weight_decay=0.0, nesterov=nesterov)
    g32 = (rng.standard_normal(n) * 1e-2).astype(np.float32)
    gbad = g32.copy()
    vals = np.resize(NONFINITE, k.size)
    gbad[k] = vals
    g32[k] = 0.0
    oracle.sgdm_step(st, _bits16(gbad, gdt), **h, step=1, wdt=wdt, gdt=gdt, ecc_bits=8)
    oracle.sgdm_step(ref, _bits16(g32, gdt), **h, step=1, wdt=wdt, gdt=gdt, ecc_bits=8)
    other = np.ones(n, bool)
    other[k] = False
    assert np.array_equal(st.w[other], ref.w[other])
    assert np.array_equal(st.ecc[other], ref.ecc[other])
    assert np.array_equal(st.mq, ref.mq) and np.array_equal(st.ms, ref.ms)
    # x'' = x - lr * (+-inf) = -+inf; NaN stays NaN (canonical pattern)
    exp = np.where(np.isnan(vals), QNAN[wdt], np.where(vals > 0, INF[wdt] | 0x8000, INF[wdt]))
    assert np.array_equal(st.w[k], exp.astype(np.uint16))
    assert np.all(st.ecc[k] == 0)


def test_fp16_master_overflow_rounds_to_inf_and_stays(orc):
    oracle = orc
    n = 64
    x = np.full(n, 65504.0, np.float32)
    x[1::2] = -65504.0
    w, e = oracle.encode_master(x, FP16, 8)
    st = oracle.State.zeros_like_master(w, e, adam=False)
    # lr = 1 and a gradient of -+100: x'' = x +- 100 exactly (fma with lr 1)
    g = np.where(x > 0, np.float32(-100.0), np.float32(100.0)).astype(np.float32)
    h = dict(lr=1.0, momentum=0.9, dampening=0.0, weight_decay=0.0, nesterov=False)
    oracle.sgdm_step(st, _bits16(g, FP16), **h, step=1, wdt=FP16, gdt=FP16, ecc_bits=8)
    with np.errstate(over="ignore"):
        exp = (x + np.where(x > 0, np.float32(100.0), np.float32(-100.0))).astype(np.float16).view(np.uint16)
    assert np.array_equal(st.w, exp)
    assert np.all((st.w & 0x7FFF) == 0x7C00)
    assert np.all(st.ecc == 0)
    # next step: the coupled decay forms fma(wd, x, g) with x = +-inf, which
    # is 0 * inf = NaN for wd = 0 (and inf - inf for wd > 0): IEEE gives NaN
    small = _bits16(np.full(n, 1e-3, np.float32), FP16)
    oracle.sgdm_step(st, small, **h, step=2, wdt=FP16, gdt=FP16, ecc_bits=8)
    assert np.all(st.w == QNAN[FP16])
    assert np.all(st.ecc == 0)
    # AdamW keeps an inf master: x (1 - lr wd) = inf and inf - step * q = inf
    w2, e2 = oracle.encode_master(x, FP16, 8)
    st2 = oracle.State.zeros_like_master(exp, e2 * 0, adam=True)
    oracle.adamw_step(st2, small, **HP, step=1, wdt=FP16, gdt=FP16, ecc_bits=8)
    assert np.array_equal(st2.w, exp)
    assert np.all(st2.ecc == 0)


def test_nan_masters_decode_and_reencode_canonically(orc):
    oracle = orc
    rng = np.random.default_rng(3)
    n = 96
    for wdt in (BF16, FP16):
        x = (rng.standard_normal(n) * 0.02).astype(np.float32)
        w, e = oracle.encode_master(x, wdt, 8)
        # NaN patterns of both signs with payloads
        w[::3] = 0xFFC1 if wdt == BF16 else 0xFE05
        w[1::3] = 0x7F81 if wdt == BF16 else 0x7C01
        st = oracle.State.zeros_like_master(w, e)
        g = _bits16((rng.standard_normal(n) * 1e-3).astype(np.float32), BF16)
        oracle.adamw_step(st, g, **HP, step=1, wdt=wdt, gdt=BF16, ecc_bits=8)
        assert np.all(st.w[::3] == QNAN[wdt]) and np.all(st.w[1::3] == QNAN[wdt])
        assert np.all(st.ecc[::3] == 0) and np.all(st.ecc[1::3] == 0)

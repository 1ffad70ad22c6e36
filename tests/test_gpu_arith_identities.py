"""GPU checks of the arithmetic identities behind the step kernel's fast path
(the kernel's own device functions, compiled with the library's flags, against
the IEEE operations of the exact path):

* the flush-to-zero approximate reciprocal / reciprocal square root equal the
  full forms wherever the result is normal (every positive normal input);
* the Newton-Raphson square root equals sqrt.rn on +0 and every binary32 in
  (0, 2^64), and is NaN from 2^64 up (so the slice is redone exactly);
* the Newton-Raphson quotient equals div.rn on 2^32 random pairs inside its
  stated range (divisor in [2^-60, 2^20), numerator 0 or |x| in [2^-80, 2^61));
* the approximate reciprocal is within 1 ulp of 1/d on [1, 2] (the bound the
  compander's tie margin is derived from), and the group-scale reciprocals
  equal 1/S and 255/S by div.rn for every finite fp16 scale S >= 0;
* (opt-in, FO_EXHAUSTIVE=1, about a minute) the Newton-Raphson quotient equals
  div.rn on every pair of significands (x, b in [1, 2): 2^46 pairs), and the
  approximate reciprocal (reciprocal square root) scales exactly by powers of
  two over the exponents the divider's range reaches: every correctly
  rounded step of the divider then commutes with the scaling while its
  intermediates stay normal, which extends the grid to the stated range;
* the bounded wait on an mbarrier gives up after its limit on a barrier that
  nothing completes (and returns at once on one that completed), so a staged
  copy that never lands cannot hang the step kernel;
* the fast ECC8 codec of 16-bit masters (bit arithmetic; for fp16 an exact
  fma at and below the smallest normal) equals the exact codec: decode of
  every finite 16-bit pattern with every code, encode of every binary32 below
  the fast path's limit (both signs).
"""
import pytest
import torch

import arith_check

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    arith_check.build()
    yield


def test_flush_to_zero_forms_equal_full_forms_on_normals():
    cnt, ex = arith_check.run(0)
    assert cnt[0] == 0, f"rcp differs on {cnt[0]} inputs, e.g. {[hex(v) for v in ex[:4]]}"
    assert cnt[1] == 0, f"rsqrt differs on {cnt[1]} inputs, e.g. {[hex(v) for v in ex[4:8]]}"


def test_newton_raphson_sqrt_exhaustive():
    cnt, ex = arith_check.run(1)
    assert cnt[0] == 0, f"sqrt differs on {cnt[0]} inputs, e.g. {[hex(v) for v in ex[:4]]}"
    assert cnt[1] == 0, f"not NaN on {cnt[1]} inputs >= 2^64, e.g. {[hex(v) for v in ex[4:8]]}"


@pytest.mark.parametrize("seed", [1, 2])
def test_newton_raphson_quotient_random_pairs(seed):
    cnt, ex = arith_check.run(2, n=1 << 31, seed=seed)
    assert cnt[0] == 0, f"quotient differs on {cnt[0]} pairs, e.g. {[hex(v) for v in ex[:4]]}"


def test_reciprocal_bound_and_scale_reciprocals():
    cnt, ex = arith_check.run(3)
    assert cnt[0] <= 1, f"rcp.approx off by {cnt[0]} ulp on [1, 2]"
    assert cnt[1] == 0, f"scale reciprocals differ for {cnt[1]} fp16 scales, e.g. {[hex(v) for v in ex[4:8]]}"


@pytest.mark.parametrize("which,name", [(4, "bf16"), (5, "fp16")])
def test_fast_ecc8_codec_exhaustive(which, name):
    cnt, ex = arith_check.run(which)
    assert cnt[0] == 0, f"{name} decode differs on {cnt[0]} (x', code) pairs, e.g. {[hex(v) for v in ex[:4]]}"
    assert cnt[1] == 0, f"{name} encode differs on {cnt[1]} inputs, e.g. {[hex(v) for v in ex[4:8]]}"


def test_approximations_scale_by_powers_of_two():
    cnt, ex = arith_check.run(7)
    assert cnt[0] == 0, f"rcp.approx does not scale on {cnt[0]} inputs, e.g. {[hex(v) for v in ex[:4]]}"
    assert cnt[1] == 0, f"rsqrt.approx does not scale on {cnt[1]} inputs, e.g. {[hex(v) for v in ex[4:8]]}"


@pytest.mark.exhaustive
def test_newton_raphson_quotient_every_significand_pair():
    """2^46 pairs in slices of 2^16 divisors (2^39 pairs, well under a second
    per launch)."""
    total, first = 0, None
    step = 1 << 16
    for b0 in range(0, 1 << 23, step):
        cnt, ex = arith_check.run(6, n=step, seed=b0)
        total += cnt[0]
        if cnt[0] and first is None:
            first = [hex(v) for v in ex[:4]]
    assert total == 0, f"quotient differs on {total} significand pairs, e.g. (x, b) = {first}"


def test_bounded_wait_gives_up_on_a_barrier_nothing_completes():
    limit = 20_000_000  # 20 ms
    cnt, ex = arith_check.run(8, n=limit)
    assert cnt[0] == 0, f"{cnt[0]} waits on a barrier nothing completes returned success"
    assert cnt[1] == 0, f"{cnt[1]} waits on a completed barrier gave up"
    assert limit <= cnt[3] <= cnt[2] < 1_000_000_000, f"waits lasted {cnt[3]} .. {cnt[2]} ns for a {limit} ns limit"

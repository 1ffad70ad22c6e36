"""Pins of the oracle's companded 8-bit optimizer states.

Source: "FlashOptim: Breaking the Memory Wall with 24-bit Weights and
Companded States", section "2. Companded Quantization" (momentum through a
softsign-like function, variance through a square root, both into 8-bit
codes with 256 bins), and Davis Blalock's release thread (8-bit linear
quantization with one 16-bit scale per 32 elements; companding is an
invertible preprocessing step).

What fixes the expected values independently of the oracle:
  * the momentum compander is twice torch's softsign (torch.nn.functional
    .softsign, binary64), the variance compander numpy's sqrt (binary64);
  * the scale rule (fp16 rounded toward +inf) is checked with numpy's fp16
    neighbours;
  * invertibility on the code grid, exhaustively over codes and scales;
  * "within one quantisation step" for heavy-tailed random data.
"""
import numpy as np
import torch

M, V, VSQRT = 0, 1, 2


def _fp16(bits):
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float64)


def test_scale_is_fp16_round_up(orc):
    rng = np.random.default_rng(0)
    a = np.concatenate([np.exp(rng.uniform(np.log(1e-9), np.log(7e4), 200000)),
                        [0.0, 6e-8, 5.960464477539063e-08, 6.103515625e-05, 1.0, 65504.0, 65504.5,
                         65520.0, 1e9, np.inf]]).astype(np.float32)
    s = orc.scale_fp16(a)
    v = _fp16(s)
    a64 = a.astype(np.float64)
    fin = a64 <= 65504.0
    assert np.all(v[fin] >= a64[fin])
    below = np.nextafter(s.view(np.float16)[fin], np.float16(0)).astype(np.float64)
    pos = a64[fin] > 0
    assert np.all(below[pos] < a64[fin][pos])
    assert np.all(v[a64 == 0] == 0)
    assert np.all(s[~fin] == 0x7BFF)  # saturated at 65504


def _softsign2(y):
    return 2.0 * torch.nn.functional.softsign(torch.from_numpy(np.asarray(y, np.float64))).numpy()


def test_momentum_compander_is_scaled_softsign(orc):
    rng = np.random.default_rng(1)
    n = 32 * 20000
    z = rng.standard_t(3, n).astype(np.float32) * np.float32(1e-3)
    q, s = orc.quantize_state(z, M)
    S = np.repeat(_fp16(s), 32)[:n]
    y = z.astype(np.float64) / S
    target = 127.0 * _softsign2(y)
    # the code is the nearest integer to 127 * phi(y); binary32 rounding of
    # the intermediate steps may only decide exact ties
    assert np.all(np.abs(q - target) <= 0.5 + 1e-4)
    # decoded values sit at the inverse compander of the code
    d = orc.dequantize_state(q, s, M).astype(np.float64)
    nz = S > 0
    assert np.allclose(127.0 * _softsign2(d[nz] / S[nz]), q[nz], atol=2e-4)
    # group maxima reach the full-scale code
    qa = np.abs(q.astype(np.int64)).reshape(-1, 32).max(axis=1)
    assert np.all(qa >= 126)


def test_variance_compander_is_sqrt(orc):
    rng = np.random.default_rng(2)
    n = 32 * 20000
    g = rng.standard_t(3, n) * 1e-4
    v = (g * g).astype(np.float32)
    sv = np.sqrt(v.astype(np.float64)).astype(np.float32)
    q, s = orc.quantize_state(sv, V)
    S = np.repeat(_fp16(s), 32)[:n]
    target = 255.0 * np.sqrt(v.astype(np.float64)) / S
    assert np.all(np.abs(q - target) <= 0.5 + 1e-4)
    d = orc.dequantize_state(q, s, V).astype(np.float64)
    assert np.allclose(np.sqrt(d) * 255.0 / np.where(S > 0, S, 1), q, atol=1e-3)


def test_compander_invertible_on_code_grid(orc):
    """For every code and every non-negative finite fp16 scale:
    quantize(dequantize(code, S), S) == code."""
    scales = np.arange(0, 0x7C00, dtype=np.uint16)          # +0 and all positive finite
    for kind, codes in ((M, np.arange(-127, 128, dtype=np.int8)),
                        (V, np.arange(0, 256, dtype=np.uint8))):
        bad = 0
        for S in scales[::1]:
            s_arr = np.full(1 + codes.size // 32, S, np.uint16)
            z = orc.dequantize_state(codes, s_arr, kind if kind == M else VSQRT)
            q = orc.quantize_fixed_scale(z, int(S), kind)
            exp = codes if S != 0 else np.zeros_like(codes)
            bad += int(np.count_nonzero(q != exp))
        assert bad == 0


def test_requantize_full_scale_group_is_fixed_point(orc):
    rng = np.random.default_rng(4)
    for kind in (M, V):
        for _ in range(200):
            if kind == M:
                q = rng.integers(-127, 128, 32).astype(np.int8)
                q[rng.integers(32)] = rng.choice([-127, 127])
            else:
                q = rng.integers(0, 256, 32).astype(np.uint8)
                q[rng.integers(32)] = 255
            S = np.array([rng.integers(1, 0x7C00)], np.uint16)
            z = orc.dequantize_state(q, S, M if kind == M else VSQRT)
            q2, s2 = orc.quantize_state(z, kind)
            assert np.array_equal(s2, S)
            assert np.array_equal(q2, q)


def test_within_one_quantisation_step(orc):
    rng = np.random.default_rng(5)
    n = 32 * 10000
    z = (rng.standard_t(2, n) * 1e-2).astype(np.float32)
    q, s = orc.quantize_state(z, M)
    qi = q.astype(np.int64)
    lo = orc.dequantize_state(np.clip(qi - 1, -127, 127).astype(np.int8), s, M)
    hi = orc.dequantize_state(np.clip(qi + 1, -127, 127).astype(np.int8), s, M)
    inner = np.abs(qi) < 127
    assert np.all((lo[inner] <= z[inner]) & (z[inner] <= hi[inner]))
    sv = np.abs(z)
    qv, sv_s = orc.quantize_state(sv, V)
    qvi = qv.astype(np.int64)
    lo = orc.dequantize_state(np.clip(qvi - 1, 0, 255).astype(np.uint8), sv_s, VSQRT)
    hi = orc.dequantize_state(np.clip(qvi + 1, 0, 255).astype(np.uint8), sv_s, VSQRT)
    assert np.all((lo <= sv) & (sv <= hi))


def test_zero_and_tail_groups(orc):
    z = np.zeros(45, np.float32)
    q, s = orc.quantize_state(z, M)
    assert np.all(q == 0) and np.all(s == 0) and s.size == 2
    z[40] = -3.0
    q, s = orc.quantize_state(z, M)
    assert s[0] == 0 and _fp16(s[1:])[0] == 3.0 and q[40] == -127
    assert np.all(np.delete(q, 40) == 0)


def test_companding_beats_linear_on_heavy_tails(orc):
    """The reason for companding: on heavy-tailed momentum the companded
    code reconstructs small entries far better than a linear 8-bit code
    with the same scale."""
    rng = np.random.default_rng(6)
    n = 32 * 20000
    z = (rng.standard_t(3, n) * 1e-3).astype(np.float32)
    q, s = orc.quantize_state(z, M)
    d = orc.dequantize_state(q, s, M).astype(np.float64)
    S = np.repeat(_fp16(s), 32)
    lin = np.clip(np.rint(z / S * 127), -127, 127) * S / 127
    small = np.abs(z) < np.median(np.abs(z))
    e_comp = np.abs(d - z)[small].mean()
    e_lin = np.abs(lin - z)[small].mean()
    assert e_comp < 0.6 * e_lin

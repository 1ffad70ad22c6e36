"""Pins of the oracle's ULP-normalised ECC (weight splitting).

Source: "FlashOptim: Breaking the Memory Wall with 24-bit Weights and
Companded States", section "1. ULP-based Weight Splitting" (the error between
the f32 master and its 16-bit version is normalised to the ULP interval and
quantized to an 8-bit correction, 24-bit effective precision), and Davis
Blalock's release thread (the f32 values rounding to one downcast value form
a fixed interval [val_min, val_max]; the ECC integer-quantizes where x32 lies
in it; 16-bit downcast + 8-bit ECC = 24-bit masters).

What fixes the expected values, independently of the oracle's binary64
interval arithmetic:
  * bf16: inside the preimage of a bf16 value the f32 grid is uniform with
    spacing u / 2^16, so the code is an integer function of the bit patterns:
    N=16 -> rho = |x|bits - |x'|bits (clamped), N=8 -> rho = round-half-even
    of that difference / 256.  Decoding is the inverse bit arithmetic.
  * every format: the decoded value must round back to x' (library cast),
    and rho must be the nearest code (brute force over the neighbouring codes).
  * encode(decode(x', rho)) = (x', rho) for every valid pair with N = 8.
"""
import numpy as np
import pytest
import torch

from conftest import threads

BF16, FP16 = 0, 1


def _bf16_of(xf: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(xf)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _fp16_of(xf: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        return xf.astype(np.float16).view(np.uint16)


def _bf16_patterns_with_offsets(seed=0, heads=None):
    """f32 patterns (w << 16) +- d (sign-magnitude) for all finite bf16 heads w
    and the offsets d that decide the 8-bit code: every tie 256k+128 and its
    neighbours, the clamp and preimage edges, plus random offsets."""
    if heads is None:
        heads = np.arange(1 << 16, dtype=np.int64)
    heads = heads[(heads & 0x7F80) != 0x7F80]
    k = np.arange(-128, 128, dtype=np.int64)
    offs = np.concatenate([(256 * k + 128)[:, None] + np.array([-1, 0, 1])[None, :]]).ravel()
    offs = np.concatenate([offs, [0, 1, -1, 32767, -32767, -32768, 32640, -32640, 32639, -32639]])
    offs = np.unique(offs)
    mag = (heads & 0x7FFF) << 16
    sgn = (heads & 0x8000) << 16
    m = mag[:, None] + offs[None, :]
    ok = (m >= 0) & (m < 0x7F800000)
    pats = (sgn[:, None] | m)[ok]
    rng = np.random.default_rng(seed)
    r = rng.integers(0, 0x7F800000, size=1 << 20, dtype=np.int64)
    r |= rng.integers(0, 2, size=r.size, dtype=np.int64) << 31
    return np.concatenate([pats, r]).astype(np.uint32)


def _bf16_closed_form(xbits: np.ndarray, w: np.ndarray, nbits: int):
    magx = (xbits & 0x7FFFFFFF).astype(np.int64)
    magw = (w.astype(np.int64) & 0x7FFF) << 16
    d = magx - magw
    if nbits == 16:
        rho = np.clip(d, -32767, 32767)
    else:
        rho = np.clip(np.rint(d / 256.0), -127, 127).astype(np.int64)
    rho[(w & 0x7F80) == 0x7F80] = 0
    return rho


def _bf16_decode_closed_form(w: np.ndarray, rho: np.ndarray, nbits: int) -> np.ndarray:
    w = w.astype(np.int64)
    unit = 256 if nbits == 8 else 1
    mag = ((w & 0x7FFF) << 16) + rho.astype(np.int64) * unit
    sgn = (w & 0x8000) << 16
    zero_in = ((w & 0x7FFF) == 0) & (rho < 0)
    # inward from +-0 the plain formula x' + s*rho*u/2^N crosses zero
    mag = np.where(zero_in, -mag, mag)
    sgn = np.where(zero_in, sgn ^ 0x80000000, sgn)
    out = (sgn | mag).astype(np.uint32)
    nonfin = (w & 0x7F80) == 0x7F80
    out[nonfin] = (w[nonfin] << 16).astype(np.uint32)
    return out


@pytest.mark.parametrize("nbits", [8, 16])
def test_bf16_encode_matches_integer_closed_form(orc, nbits):
    pats = _bf16_patterns_with_offsets()
    x = pats.view(np.float32)
    w, rho = orc.encode_master(x, BF16, nbits, threads=threads())
    assert np.array_equal(w, _bf16_of(x))
    exp = _bf16_closed_form(pats, w, nbits)
    bad = np.nonzero(rho.astype(np.int64) != exp)[0]
    assert bad.size == 0, f"{bad.size} mismatches; x bits {pats[bad[:4]]} got {rho[bad[:4]]} exp {exp[bad[:4]]}"


@pytest.mark.parametrize("nbits", [8, 16])
def test_bf16_decode_matches_closed_form_and_rounds_back(orc, nbits):
    pats = _bf16_patterns_with_offsets(seed=2)
    x = pats.view(np.float32)
    w, rho = orc.encode_master(x, BF16, nbits, threads=threads())
    dec = orc.decode_master(w, rho, BF16, nbits, threads=threads())
    assert np.array_equal(dec.view(np.uint32), _bf16_decode_closed_form(w, rho, nbits))
    # the reconstruction lies in the interval of f32 values that round to x'
    assert np.array_equal(_bf16_of(dec), w)
    # x that round to +-inf have no finite interval: x' = inf, rho = 0
    fin = (w & 0x7F80) != 0x7F80
    pats, dec, rho = pats[fin], dec[fin], rho[fin]
    # error bound: |x - dec| <= u / 2^(N+1) unclamped (u/2^N at the clamp);
    # in f32-bit units of the preimage grid (u / 2^16) that is 2^(15-N)
    err = np.abs(pats.astype(np.int64) - dec.view(np.uint32).astype(np.int64))
    lim = 1 << (16 - nbits - 1) if nbits == 8 else 0
    clamped = np.abs(rho.astype(np.int64)) == (1 << (nbits - 1)) - 1
    assert np.all(err[~clamped] <= lim)
    assert np.all(err[clamped] <= max(2 * lim, 1))
    if nbits == 16:
        # exact reconstruction except at the two clamped tie points
        assert np.count_nonzero(err) == np.count_nonzero(err[clamped])


def _fp16_inputs(seed=0):
    """For every finite fp16 value x': points across its whole preimage,
    including both rounding edges and the ties of the 8- and 16-bit codes."""
    h = np.arange(1 << 16, dtype=np.uint16)
    h = h[(h & 0x7C00) != 0x7C00]
    xp = h.view(np.float16).astype(np.float64)
    with np.errstate(over="ignore"):
        up = np.nextafter(h.view(np.float16), np.where(np.signbit(xp), np.float16(-np.inf), np.float16(np.inf))).astype(np.float64)
        dn = np.nextafter(h.view(np.float16), np.float16(0.0)).astype(np.float64)
    up = np.where(np.isfinite(up), up, xp + (xp - dn))
    hi = (up - xp) / 2.0           # signed half-distances to the rounding edges
    lo = (dn - xp) / 2.0
    fr = np.concatenate([np.linspace(-1.0, 1.0, 33), [1 - 2.0 ** -20, -(1 - 2.0 ** -20)],
                         (np.arange(-128, 129) + 0.5) / 128.0])
    rng = np.random.default_rng(seed)
    fr = np.concatenate([fr, rng.uniform(-1, 1, 32)])
    pos = np.where(fr[None, :] >= 0, fr[None, :] * hi[:, None], -fr[None, :] * lo[:, None])
    x = (xp[:, None] + pos).ravel()
    return x.astype(np.float32)


@pytest.mark.parametrize("nbits", [8, 16])
def test_fp16_code_is_nearest_and_rounds_back(orc, nbits):
    x = _fp16_inputs()
    w, rho = orc.encode_master(x, FP16, nbits, threads=threads())
    assert np.array_equal(w, _fp16_of(x))
    fin = (w & 0x7C00) != 0x7C00
    x, w, rho = x[fin], w[fin], rho[fin]
    dec = orc.decode_master(w, rho, FP16, nbits, threads=threads())
    # decode lands back in the preimage of x' (numpy's cast decides)
    assert np.array_equal(_fp16_of(dec), w)
    # brute force: no neighbouring code reconstructs x more closely
    lim = (1 << (nbits - 1)) - 1
    dt = rho.dtype
    e0 = np.abs(dec.astype(np.float64) - x.astype(np.float64))
    for step in (-1, 1):
        nb = np.clip(rho.astype(np.int64) + step, -lim, lim).astype(dt)
        dn = orc.decode_master(w, nb, FP16, nbits, threads=threads())
        en = np.abs(dn.astype(np.float64) - x.astype(np.float64))
        assert np.all(e0 <= en), f"nearer code exists for {np.count_nonzero(e0 > en)} inputs"
    # distance bound relative to the fp16 spacing on x's side of x'
    xp = w.view(np.float16).astype(np.float64)
    side_out = np.abs(x.astype(np.float64)) >= np.abs(xp)
    with np.errstate(over="ignore"):
        u_out = np.abs(np.nextafter(w.view(np.float16), np.copysign(np.float16(np.inf), w.view(np.float16))).astype(np.float64) - xp)
        u_in = np.abs(xp - np.nextafter(w.view(np.float16), np.float16(0)).astype(np.float64))
    u_in = np.where(xp == 0, u_out, u_in)
    u = np.where(side_out, u_out, u_in)
    okf = np.isfinite(u)
    bound = u / 2.0 ** (nbits + 1) + np.abs(x.astype(np.float64)) * 2.0 ** -24
    clamped = np.abs(rho.astype(np.int64)) == lim
    bound = np.where(clamped, 2 * bound, bound)
    assert np.all(e0[okf] <= bound[okf])


@pytest.mark.parametrize("wdt", [BF16, FP16])
def test_ecc8_idempotent_on_every_pair(orc, wdt):
    """encode(decode(x', rho)) == (x', rho) for all 2^16 x' and every 8-bit
    code rho in [-127, 127]; excluded are codes that encode never emits:
    rho != 0 on non-finite x', rho < 0 on +-0."""
    h = np.repeat(np.arange(1 << 16, dtype=np.uint16), 255)
    r = np.tile(np.arange(-127, 128, dtype=np.int8), 1 << 16)
    if wdt == BF16:
        nonfin = (h & 0x7F80) == 0x7F80
    else:
        nonfin = (h & 0x7C00) == 0x7C00
    zero = (h & 0x7FFF) == 0
    keep = ~(nonfin & (r != 0)) & ~(zero & (r < 0)) & ~nonfin
    h, r = h[keep], r[keep]
    dec = orc.decode_master(h, r, wdt, 8, threads=threads())
    w2, r2 = orc.encode_master(dec, wdt, 8, threads=threads())
    assert np.array_equal(w2, h)
    assert np.array_equal(r2, r)


def test_effective_precision_24_bits(orc):
    """bf16 + 8-bit ECC: the reconstruction error is at most one bf16 ULP
    / 2^8 (relative 2^-15, reached only at the clamped codes +-127) and at
    most ULP / 2^9 (relative 2^-16) elsewhere."""
    rng = np.random.default_rng(3)
    x = (rng.standard_normal(1 << 20) * 0.02).astype(np.float32)
    w, r = orc.encode_master(x, BF16, 8, threads=threads())
    d = orc.decode_master(w, r, BF16, 8, threads=threads())
    rel = np.abs(d.astype(np.float64) - x) / np.abs(x.astype(np.float64))
    assert rel.max() <= 2.0 ** -15
    assert rel[np.abs(r) < 127].max() <= 2.0 ** -16
    # plain bf16 alone: 2^-9 worst case; the code buys 8 more bits
    rel_bf16 = np.abs(torch.from_numpy(x).to(torch.bfloat16).float().numpy().astype(np.float64) - x) / np.abs(x)
    assert rel.max() * 2 ** 7 <= rel_bf16.max()


@pytest.mark.exhaustive
@pytest.mark.parametrize("nbits", [8, 16])
def test_bf16_all_2_32(orc, nbits):
    step = 1 << 26
    for start in range(0, 1 << 32, step):
        pats = np.arange(start, start + step, dtype=np.uint64).astype(np.uint32)
        x = pats.view(np.float32)
        fin = np.isfinite(x)
        pats, x = pats[fin], x[fin]
        w, rho = orc.encode_master(x, BF16, nbits, threads=threads())
        assert np.array_equal(rho.astype(np.int64), _bf16_closed_form(pats, w, nbits))
        dec = orc.decode_master(w, rho, BF16, nbits, threads=threads())
        assert np.array_equal(dec.view(np.uint32), _bf16_decode_closed_form(w, rho, nbits))
        fw = (w & 0x7F80) != 0x7F80
        assert np.array_equal(_bf16_of(dec[fw]), w[fw])

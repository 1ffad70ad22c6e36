"""Pins of the oracle's fused optimizer step against torch.optim in binary64.

Source: Davis Blalock's FlashOptim release thread (the optimizers compute
the same updates as the usual Adam / SGD while using less memory; gradients
stay in backward precision) and "FlashOptim: Breaking the Memory Wall with
24-bit Weights and Companded States" (AdamW, 16 -> 7 bytes per parameter).

The reference updates come from torch.optim.AdamW / torch.optim.SGD run in
float64 on the decoded masters; the compressed step may differ from them only
by the quantization of the stored state, never by a wrong term, sign or
index.
"""
import numpy as np
import pytest
import torch

from conftest import threads
from workloads import gen

BF16, FP16 = 0, 1
HP = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01)


def _grad_bits(g32, dt):
    return gen.to_16bit(g32, "bf16" if dt == BF16 else "fp16")


def _widen(orc, bits, dt):
    return orc.widen(bits, dt).astype(np.float64)


def _torch_adamw(x, grads, hp):
    p = torch.nn.Parameter(torch.from_numpy(x.astype(np.float64)))
    opt = torch.optim.AdamW([p], lr=hp["lr"], betas=(hp["beta1"], hp["beta2"]), eps=hp["eps"],
                            weight_decay=hp["weight_decay"], foreach=False)
    out = []
    for g in grads:
        p.grad = torch.from_numpy(g.astype(np.float64))
        opt.step()
        st = opt.state[p]
        out.append((p.detach().numpy().copy(), st["exp_avg"].numpy().copy(),
                    st["exp_avg_sq"].numpy().copy()))
    return out


def _setup(orc, n, seed, wdt=BF16, nbits=8, adam=True):
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal(n) * 0.02).astype(np.float32)
    w, e = orc.encode_master(x, wdt, nbits)
    return orc.State.zeros_like_master(w, e, adam=adam)


def test_adamw_step1_matches_torch(orc):
    n = 32 * 4096 + 13
    st = _setup(orc, n, 0)
    x0 = orc.decode_master(st.w, st.ecc, BF16, 8).astype(np.float64)
    rng = np.random.default_rng(1)
    gb = _grad_bits((rng.standard_normal(n) * 1e-3).astype(np.float32), BF16)
    g = _widen(orc, gb, BF16)
    orc.adamw_step(st, gb, **HP, step=1, threads=threads())
    xr, mr, vr = _torch_adamw(x0, [g], HP)[0]
    x1 = orc.decode_master(st.w, st.ecc, BF16, 8).astype(np.float64)
    # step-1 closed form: x(1 - lr wd) - lr g / (|g| + eps); deviations only
    # from binary32 rounding and the ECC (ULP/2^8 of x)
    assert np.all(np.abs(x1 - xr) <= np.abs(xr) * 2.0 ** -15 + 4 * 2.0 ** -24 * HP["lr"] + 1e-12)
    m = orc.dequantize_state(st.mq, st.ms, 0).astype(np.float64)
    v = orc.dequantize_state(st.vq, st.vs, 1).astype(np.float64)
    S_m = np.repeat(st.ms.view(np.float16).astype(np.float64), 32)[:n]
    S_v = np.repeat(st.vs.view(np.float16).astype(np.float64), 32)[:n]
    # one quantisation step of the companded code (largest step at full scale)
    assert np.all(np.abs(m - mr) <= S_m * (1.0 / 127) * 1.01)
    assert np.all(np.abs(np.sqrt(v) - np.sqrt(vr)) <= S_v / 255 * 0.51 + 1e-12)


@pytest.mark.parametrize("wdt,nbits,rel", [(BF16, 16, 2.0 ** -21), (FP16, 8, 2.0 ** -18), (FP16, 16, 2.0 ** -21)])
def test_adamw_step1_matches_torch_other_master_formats(orc, wdt, nbits, rel):
    """Step 1 against torch.optim.AdamW (binary64) for the other master
    formats: the decoded master after the step deviates from torch only by
    binary32 rounding of the update and by the ECC's resolution (u / 2^(N+1)
    of the 16-bit format: 2^-17 of |x| for fp16 + 8 bits, below binary32
    resolution for 16 bits), plus fp16's subnormal floor."""
    n = 32 * 2048 + 7
    st = _setup(orc, n, 10 + nbits + wdt, wdt=wdt, nbits=nbits)
    x0 = orc.decode_master(st.w, st.ecc, wdt, nbits).astype(np.float64)
    rng = np.random.default_rng(11)
    gb = _grad_bits((rng.standard_normal(n) * 1e-3).astype(np.float32), BF16)
    orc.adamw_step(st, gb, **HP, step=1, wdt=wdt, gdt=BF16, ecc_bits=nbits, threads=threads())
    xr = _torch_adamw(x0, [_widen(orc, gb, BF16)], HP)[0][0]
    x1 = orc.decode_master(st.w, st.ecc, wdt, nbits).astype(np.float64)
    tol = np.abs(xr) * rel + 4 * 2.0 ** -24 * HP["lr"] + 2.0 ** -32
    assert np.all(np.abs(x1 - xr) <= tol), np.max(np.abs(x1 - xr) / tol)
    # and the bound is not vacuous: the deviation is not zero everywhere
    assert np.any(x1 != xr)


def test_adamw_ten_steps_track_torch(orc):
    """Ten AdamW steps (the flat-group workload, reduced to 64K params) stay
    close to uncompressed binary64 AdamW: per step the median deviation is
    below 5% of lr, the 99.9th percentile below 25% of lr, and no parameter
    drifts by more than 2 lr.  The few largest deviations are entries whose
    gradient is ~1000x below their group's largest, so their 8-bit momentum
    and variance codes are 0 (their update then differs by about one lr).
    The thresholds are this project's choice: the pages claim the same
    updates qualitatively and print no tolerance."""
    n = 65536
    st = _setup(orc, n, 2)
    x0 = orc.decode_master(st.w, st.ecc, BF16, 8).astype(np.float64)
    rng = np.random.default_rng(3)
    gbs = [_grad_bits((rng.standard_normal(n) * 1e-3).astype(np.float32), BF16) for _ in range(10)]
    ref = _torch_adamw(x0, [_widen(orc, gb, BF16) for gb in gbs], HP)
    for k, gb in enumerate(gbs):
        orc.adamw_step(st, gb, **HP, step=k + 1, threads=threads())
        x = orc.decode_master(st.w, st.ecc, BF16, 8).astype(np.float64)
        dev = np.abs(x - ref[k][0]) / HP["lr"]
        assert np.median(dev) < 0.05, (k, np.median(dev))
        assert np.percentile(dev, 99.9) < 0.25, (k, np.percentile(dev, 99.9))
        assert dev.max() < 2.0, (k, dev.max())


def test_adamw_wrong_term_would_be_caught(orc):
    """A dropped bias correction changes step 1 by a factor ~3: the torch
    comparison above is sensitive to it (checked on the reference side)."""
    n = 4096
    st = _setup(orc, n, 4)
    x0 = orc.decode_master(st.w, st.ecc, BF16, 8).astype(np.float64)
    g = np.full(n, 1e-3)
    xr = _torch_adamw(x0, [g], HP)[0][0]
    no_bc = x0 * (1 - HP["lr"] * HP["weight_decay"]) - HP["lr"] * 0.1e-3 / (np.sqrt(0.001e-6) + 1e-8)
    assert np.min(np.abs(no_bc - xr)) > 1e-4


def test_zero_grad_zero_state(orc):
    n = 1000
    st = _setup(orc, n, 5)
    x0 = orc.decode_master(st.w, st.ecc, BF16, 8)
    orc.adamw_step(st, np.zeros(n, np.uint16), **HP, step=1)
    assert np.all(st.mq == 0) and np.all(st.ms == 0) and np.all(st.vq == 0) and np.all(st.vs == 0)
    x1 = orc.decode_master(st.w, st.ecc, BF16, 8)
    decay = np.float32(1.0 - HP["lr"] * HP["weight_decay"])
    w2, e2 = orc.encode_master(x0 * decay, BF16, 8)
    assert np.array_equal(st.w, w2) and np.array_equal(st.ecc, e2)
    assert np.allclose(x1, x0 * decay, rtol=2.0 ** -15, atol=0)


@pytest.mark.parametrize("wdt", [BF16, FP16])
def test_lr0_wd0_leaves_weights_bit_identical(orc, wdt):
    """With lr = 0 and no decay the update is exactly zero, so the weight
    split must re-encode to the same bytes (idempotence of the ECC)."""
    n = 32 * 1000 + 7
    st = _setup(orc, n, 6, wdt=wdt)
    w0, e0 = st.w.copy(), st.ecc.copy()
    rng = np.random.default_rng(7)
    for t in (1, 2, 3):
        gb = _grad_bits((rng.standard_normal(n) * 1e-3).astype(np.float32), BF16)
        orc.adamw_step(st, gb, lr=0.0, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.0, step=t,
                       wdt=wdt)
        assert np.array_equal(st.w, w0) and np.array_equal(st.ecc, e0)
    st2 = _setup(orc, n, 6, wdt=wdt, adam=False)
    gb = _grad_bits((rng.standard_normal(n) * 1e-2).astype(np.float32), FP16)
    orc.sgdm_step(st2, gb, lr=0.0, momentum=0.9, step=1, wdt=wdt, gdt=FP16)
    assert np.array_equal(st2.w, w0) and np.array_equal(st2.ecc, e0)


def _torch_sgd(x, grads, lr, mom, damp, wd, nesterov):
    p = torch.nn.Parameter(torch.from_numpy(x.astype(np.float64)))
    opt = torch.optim.SGD([p], lr=lr, momentum=mom, dampening=damp, weight_decay=wd,
                          nesterov=nesterov, foreach=False)
    out = []
    for g in grads:
        p.grad = torch.from_numpy(g.astype(np.float64))
        opt.step()
        out.append((p.detach().numpy().copy(), opt.state[p]["momentum_buffer"].numpy().copy()))
    return out


@pytest.mark.parametrize("damp,nesterov", [(0.0, False), (0.1, False), (0.0, True)])
def test_sgdm_matches_torch(orc, damp, nesterov):
    n = 32 * 2048 + 5
    st = _setup(orc, n, 8, wdt=FP16, adam=False)
    x0 = orc.decode_master(st.w, st.ecc, FP16, 8).astype(np.float64)
    rng = np.random.default_rng(9)
    gbs = [_grad_bits((rng.standard_normal(n) * 1e-2).astype(np.float32), FP16) for _ in range(2)]
    lr, mom, wd = 0.1, 0.9, 1e-4
    ref = _torch_sgd(x0, [_widen(orc, gb, FP16) for gb in gbs], lr, mom, damp, wd, nesterov)
    # step 1: buf = g + wd x exactly (up to binary32), x1 = x0 - lr * dir
    orc.sgdm_step(st, gbs[0], lr=lr, momentum=mom, dampening=damp, weight_decay=wd,
                  nesterov=nesterov, step=1, threads=threads())
    x1 = orc.decode_master(st.w, st.ecc, FP16, 8).astype(np.float64)
    b1 = orc.dequantize_state(st.mq, st.ms, 0).astype(np.float64)
    S = np.repeat(st.ms.view(np.float16).astype(np.float64), 32)[:n]
    # fp16 + 8-bit ECC: ULP(fp16)/2^8 relative 2^-18, plus binary32 rounding
    assert np.all(np.abs(x1 - ref[0][0]) <= np.abs(ref[0][0]) * 2.0 ** -17 + 1e-9)
    assert np.all(np.abs(b1 - ref[0][1]) <= S / 127 * 1.01)
    # step 2 from the stored (quantized) buffer: compare against torch run
    # from the same decoded state
    ref2 = _torch_sgd(x1, [], lr, mom, damp, wd, nesterov)
    p = torch.nn.Parameter(torch.from_numpy(x1.copy()))
    opt = torch.optim.SGD([p], lr=lr, momentum=mom, dampening=damp, weight_decay=wd,
                          nesterov=nesterov, foreach=False)
    opt.state[p]["momentum_buffer"] = torch.from_numpy(b1.copy())
    p.grad = torch.from_numpy(_widen(orc, gbs[1], FP16))
    opt.step()
    orc.sgdm_step(st, gbs[1], lr=lr, momentum=mom, dampening=damp, weight_decay=wd,
                  nesterov=nesterov, step=2, threads=threads())
    x2 = orc.decode_master(st.w, st.ecc, FP16, 8).astype(np.float64)
    xr2 = p.detach().numpy()
    assert np.all(np.abs(x2 - xr2) <= np.abs(xr2) * 2.0 ** -17 + 1e-8)
    del ref2


def test_threads_do_not_change_results(orc):
    n = 32 * 5000 + 31
    a = _setup(orc, n, 10)
    b = a.copy()
    rng = np.random.default_rng(11)
    gb = _grad_bits((rng.standard_normal(n) * 1e-3).astype(np.float32), BF16)
    orc.adamw_step(a, gb, **HP, step=1, threads=1)
    orc.adamw_step(b, gb, **HP, step=1, threads=7)
    for u, v in zip((a.w, a.ecc, a.mq, a.ms, a.vq, a.vs), (b.w, b.ecc, b.mq, b.ms, b.vq, b.vs)):
        assert np.array_equal(u, v)


def test_groups_are_independent(orc):
    """Stepping a tensor in pieces of whole groups gives the same bytes as
    stepping it at once (the basis of sampled parity at full size)."""
    n = 32 * 300 + 17
    a = _setup(orc, n, 12)
    rng = np.random.default_rng(13)
    gb = _grad_bits((rng.standard_normal(n) * 1e-3).astype(np.float32), BF16)
    b = a.copy()
    orc.adamw_step(a, gb, **HP, step=1)
    cut = 32 * 111
    for lo, hi in ((0, cut), (cut, n)):
        g0, g1 = lo // 32, (hi + 31) // 32
        part = orc.State(b.w[lo:hi].copy(), b.ecc[lo:hi].copy(), b.mq[lo:hi].copy(),
                         b.ms[g0:g1].copy(), b.vq[lo:hi].copy(), b.vs[g0:g1].copy())
        orc.adamw_step(part, gb[lo:hi], **HP, step=1)
        assert np.array_equal(part.w, a.w[lo:hi]) and np.array_equal(part.ecc, a.ecc[lo:hi])
        assert np.array_equal(part.mq, a.mq[lo:hi]) and np.array_equal(part.ms, a.ms[g0:g1])
        assert np.array_equal(part.vq, a.vq[lo:hi]) and np.array_equal(part.vs, a.vs[g0:g1])

"""GPU parity: every byte the CUDA path emits (downcast weights, ECC codes,
momentum / variance codes, fp16 scales) equals the CPU oracle's, on the same
seeded inputs.  All GPU work goes through the C ABI (libfo.so via ctypes).

Bar: bit-exact on every emitted byte (the method emits integer codes and
16-bit patterns only).  Non-finite values are not produced by these inputs.
"""
import numpy as np
import pytest
import torch

import oracle
from bit_states_b200 import fo
from workloads import gen, workload
from workloads import device as wdev
from workloads.shapes import TensorSpec, Workload, ADAMW_HP, SGDM_HP

import gpu_util as U

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    from bit_states_b200 import build as fobuild

    fobuild.build()
    wdev.build()
    fo.load()
    torch.cuda.init()
    yield
    torch.cuda.synchronize()


def _nthreads():
    import os

    return max(1, min(32, os.cpu_count() or 1))


# ---- generator -----------------------------------------------------------------

@pytest.mark.parametrize("name", ["gpt2-small-124M", "resnet50-25.6M", "llama3.1-8b"])
def test_device_generator_matches_host(name):
    wl = workload(name)
    rng = np.random.default_rng(0)
    for ti in rng.choice(len(wl.tensors), size=min(6, len(wl.tensors)), replace=False):
        n = wl.tensors[ti].numel
        n_dev = min(n, 1 << 22)
        x = torch.empty(n_dev, dtype=torch.float32, device=DEV)
        g = torch.empty(n_dev, dtype=torch.int16, device=DEV)
        # device generation is by global index, so generate a prefix
        spec = wl.tensors[ti]
        if spec.init != "const":
            wdev.master_f32(wl, ti, x)
        wdev.grad_16(wl, ti, 3, g)
        idx = rng.choice(n_dev, size=min(n_dev, 20000), replace=False)
        if spec.init != "const":
            assert np.array_equal(x.cpu().numpy()[idx].view(np.uint32),
                                  wl.master_values(ti, idx).view(np.uint32))
        assert np.array_equal(g.cpu().numpy()[idx].view(np.uint16), wl.grad_bits(ti, 3, idx))


# ---- master codec ---------------------------------------------------------------

def _codec_inputs(wdt):
    rng = np.random.default_rng(7)
    if wdt == "bf16":
        heads = np.arange(1 << 16, dtype=np.int64)
        heads = heads[(heads & 0x7F80) != 0x7F80]
        offs = np.unique(np.concatenate([256 * np.arange(-128, 128)[:, None] + 128 + np.array([-1, 0, 1])[None, :]]
                                        ).ravel().tolist() + [0, 1, -1, 32767, -32767, -32768])
        m = ((heads & 0x7FFF) << 16)[:, None] + offs[None, :]
        ok = (m >= 0) & (m < 0x7F800000)
        pats = (((heads & 0x8000) << 16)[:, None] | m)[ok].astype(np.uint32)
    else:
        e = np.arange(256, dtype=np.uint32) << 23
        tails = np.concatenate([np.arange(0, 1 << 13, dtype=np.uint32), rng.integers(0, 1 << 23, 4096).astype(np.uint32)])
        pats = (e[:, None] | tails[None, :]).ravel()
        pats = np.concatenate([pats, pats | np.uint32(0x80000000)])
    r = rng.integers(0, 1 << 32, size=1 << 22, dtype=np.uint64).astype(np.uint32)
    pats = np.concatenate([pats, r])
    x = pats.view(np.float32)
    return x[np.isfinite(x)]


@pytest.mark.parametrize("wdt", ["bf16", "fp16"])
@pytest.mark.parametrize("nbits", [8, 16])
def test_encode_decode_master_bit_exact(wdt, nbits):
    x = _codec_inputs(wdt)
    n = x.size
    fmt = fo.make_format(wdt, "bf16", nbits)
    xd = torch.from_numpy(x).to(DEV)
    w = torch.empty(n, dtype=torch.int16, device=DEV)
    e = torch.empty(n, dtype=torch.int8 if nbits == 8 else torch.int16, device=DEV)
    fo.fo_encode_master(xd, w, e, n, fmt)
    ow, oe = oracle.encode_master(x, U.DT[wdt], nbits, threads=_nthreads())
    gw = w.cpu().numpy().view(np.uint16)
    ge = e.cpu().numpy()
    assert np.count_nonzero(gw != ow) == 0
    assert np.count_nonzero(ge != oe) == 0
    # decode of every code of random heads (not just encode outputs)
    rng = np.random.default_rng(11)
    heads = rng.integers(0, 1 << 16, size=1 << 20, dtype=np.uint32).astype(np.uint16)
    lim = (1 << (nbits - 1)) - 1
    codes = rng.integers(-lim, lim + 1, size=heads.size).astype(oracle.ecc_dtype(nbits))
    od = oracle.decode_master(heads, codes, U.DT[wdt], nbits, threads=_nthreads())
    xo = torch.empty(heads.size, dtype=torch.float32, device=DEV)
    fo.fo_decode_master(torch.from_numpy(heads.view(np.int16)).to(DEV), torch.from_numpy(codes).to(DEV),
                        xo, heads.size, fmt)
    gd = xo.cpu().numpy()
    nan = np.isnan(od)
    assert np.array_equal(np.isnan(gd), nan)
    assert np.count_nonzero(gd.view(np.uint32)[~nan] != od.view(np.uint32)[~nan]) == 0


# ---- flat group, 10 steps, every byte ----------------------------------------------

def _run_full_compare(wl, steps, order=None, check_every=True, sample_above=None):
    """Every byte of every tensor against the oracle; tensors of more than
    `sample_above` elements on 256 sampled groups (first and last included)."""
    P = U.device_state(wl)
    G = U.GradArena(P)
    orcs = []
    rng = np.random.default_rng(23)
    for ti, t in enumerate(wl.tensors):
        ng = (t.numel + 31) // 32
        sampled = sample_above is not None and t.numel > sample_above
        groups = U.sample_groups(t.numel, 256, rng) if sampled else np.arange(ng)
        orcs.append(U.OracleSample(wl, ti, groups, threads=_nthreads()))
    for t in range(1, steps + 1):
        G.fill(wl, t)
        U.step(wl, P, G, t, order=order)
        for o in orcs:
            o.step(t)
        if check_every or t == steps:
            torch.cuda.synchronize()
            for ti, o in enumerate(orcs):
                exp = o.expected()
                got = U.gather_device(P, ti, exp)
                mm = U.mismatches(exp, got)
                assert all(v == 0 for v in mm.values()), (wl.name, ti, t, mm)
    return P


def test_flat_1m_ten_adamw_steps_every_byte():
    wl = workload("flat-1M")
    _run_full_compare(wl, 10)


# ---- ragged sizes, misaligned views, all formats ------------------------------------

RAGGED = [1, 2, 31, 32, 33, 255, 256, 257, 511, 512, 513, 767, 768, 769, 1000, 1023, 1024, 1025, 1536, 1537,
          2047, 2048, 2049, 2560, 2561, 3071, 3072, 3073, 4095, 4096, 65537]


def _ragged_workload(opt, wdt, gdt, nbits):
    ts = [TensorSpec(f"t{i}", (n,), "normal", 0.02 if i % 3 else 1.5) for i, n in enumerate(RAGGED)]
    hp = dict(ADAMW_HP) if opt == "adamw" else dict(SGDM_HP)
    return Workload(name=f"ragged-{opt}", tensors=ts, optimizer=opt, hparams=hp, w_dtype=wdt,
                    grad_dtype=gdt, ecc_bits=nbits, grad_dist="normal_outliers", grad_scale=1e-3, seed=5)


@pytest.mark.parametrize("opt", ["adamw", "sgdm"])
@pytest.mark.parametrize("wdt,gdt", [("bf16", "bf16"), ("fp16", "fp16"), ("bf16", "fp16"), ("fp16", "bf16")])
@pytest.mark.parametrize("nbits", [8, 16])
def test_ragged_multitensor_all_formats(opt, wdt, gdt, nbits):
    wl = _ragged_workload(opt, wdt, gdt, nbits)
    _run_full_compare(wl, 3)


# a tensor large enough that every warp of the persistent grid walks many
# chunks of it
LARGE = 3 << 25


@pytest.mark.parametrize("wdt,gdt", [("bf16", "bf16"), ("fp16", "fp16"), ("bf16", "fp16"), ("fp16", "bf16")])
def test_ragged_with_large_tensor(wdt, gdt):
    """The ragged list plus one tensor of 3 * 2^25 + 45 elements in the middle:
    every warp walks many chunks, across tensor boundaries (ragged tails,
    slice and chunk edges at 511 / 512 / 513, 1023 / 1024 / 1025 and
    1535 / 1536 / 1537); every byte of every
    ragged tensor and sampled groups of the large one against the oracle."""
    wl = _ragged_workload("adamw", wdt, gdt, 8)
    wl.tensors.insert(7, TensorSpec("fill", (LARGE + 45,), "normal", 0.02))
    _run_full_compare(wl, 2, sample_above=1 << 20)


@pytest.mark.parametrize("hp", [
    dict(lr=3e-4, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1),     # LLM-style betas
    dict(lr=1e-2, beta1=0.8, beta2=0.99, eps=1e-6, weight_decay=0.0),     # no decay: x (1 - lr wd) = x
    dict(lr=1e-3, beta1=0.0, beta2=0.999, eps=1e-12, weight_decay=0.01),  # no momentum averaging
])
def test_ragged_adamw_hyperparameter_sets(hp):
    wl = _ragged_workload("adamw", "bf16", "bf16", 8)
    wl.hparams = dict(hp)
    _run_full_compare(wl, 3)


@pytest.mark.parametrize("nesterov,damp", [(1, 0.0), (0, 0.25)])
def test_sgdm_variants(nesterov, damp):
    wl = _ragged_workload("sgdm", "fp16", "fp16", 8)
    wl.hparams.update(nesterov=nesterov, dampening=damp)
    _run_full_compare(wl, 3)


@pytest.mark.parametrize("nbits", [8, 16])
@pytest.mark.parametrize("s16,s8", [(1, 1), (2, 2), (3, 3), (8, 8), (16, 16), (8, 16), (24, 32), (16, 16 + 8)])
def test_misaligned_views_take_scalar_path(s16, s8, nbits):
    """Tensors whose arrays start off the 16-byte grid, or whose weights (and
    16-bit ECC codes) start off the 32-byte grid that their 256-bit stores
    need, take the scalar path; arrays on both grids take the staged path.
    Views into larger buffers: the 16-bit arrays are shifted by s16 elements,
    the 8-bit ones by s8.  Same bytes as the oracle either way, and canaries
    around every output stay intact."""
    n = 3000
    wl = _ragged_workload("adamw", "bf16", "bf16", nbits)
    wl.tensors = [TensorSpec("a", (n,), "normal", 0.02)]
    idx = np.arange(n)
    x = wl.master_values(0, idx)
    ow, oe = oracle.encode_master(x, 0, nbits)
    pad = 64
    mk = lambda dt, cnt: torch.full((cnt + 2 * pad,), 0x5A, dtype=dt, device=DEV)
    edt = torch.int8 if nbits == 8 else torch.int16
    w = mk(torch.int16, n); e = mk(edt, n); mq = mk(torch.int8, n); vq = mk(torch.uint8, n)
    ng = (n + 31) // 32
    ms = mk(torch.int16, ng); vs = mk(torch.int16, ng); g = mk(torch.int16, n)
    se = s8 if nbits == 8 else s16
    shifts = dict(w=s16, e=se, mq=s8, vq=s8, g=s16, ms=8, vs=8)
    views = {k: full[pad + shifts[k]:pad + shifts[k] + (ng if k in ("ms", "vs") else n)]
             for k, full in dict(w=w, e=e, mq=mq, vq=vq, g=g, ms=ms, vs=vs).items()}
    wv, ev, mqv, vqv, gv, msv, vsv = (views[k] for k in ("w", "e", "mq", "vq", "g", "ms", "vs"))
    wv.copy_(torch.from_numpy(ow.view(np.int16))); ev.copy_(torch.from_numpy(oe))
    mqv.zero_(); vqv.zero_(); msv.zero_(); vsv.zero_()
    st = oracle.State.zeros_like_master(ow, oe)
    before = {k: v.clone() for k, v in dict(w=w, e=e, mq=mq, vq=vq, ms=ms, vs=vs).items()}
    state = fo.TensorState(wv, ev, mqv, msv, vqv, vsv)
    for t in (1, 2):
        gb = wl.grad_bits(0, t, idx)
        gv.copy_(torch.from_numpy(gb.view(np.int16)))
        d = fo.descriptors([state], [gv])
        fo.fo_adamw_step(d, 1, fo.make_format("bf16", "bf16", nbits), U.hparams_adamw(wl, t))
        oracle.adamw_step(st, gb, **wl.hparams, step=t, ecc_bits=nbits)
    torch.cuda.synchronize()
    assert np.array_equal(U.to_np_bytes(wv), st.w)
    assert np.array_equal(ev.cpu().numpy(), st.ecc)
    assert np.array_equal(mqv.cpu().numpy(), st.mq)
    assert np.array_equal(vqv.cpu().numpy(), st.vq)
    assert np.array_equal(U.to_np_bytes(msv), st.ms)
    assert np.array_equal(U.to_np_bytes(vsv), st.vs)
    for k, full in dict(w=w, e=e, mq=mq, vq=vq, ms=ms, vs=vs).items():
        lo = pad + shifts[k]
        cnt = ng if k in ("ms", "vs") else n
        assert torch.equal(full[:lo], before[k][:lo]), k
        assert torch.equal(full[lo + cnt:], before[k][lo + cnt:]), k
    fo.fo_check_errors()


def test_empty_and_tiny_tensors_in_one_call():
    wl = _ragged_workload("adamw", "bf16", "bf16", 8)
    wl.tensors = [TensorSpec("one", (1,), "normal", 0.02), TensorSpec("seven", (7,), "normal", 0.02)]
    P = U.device_state(wl)
    G = U.GradArena(P)
    G.fill(wl, 1)
    empty = fo.TensorState(P.w[:0], P.ecc[:0], P.m_q[:0], P.m_scale[:0], P.v_q[:0], P.v_scale[:0])
    states = [empty, P.states[0], empty, P.states[1]]
    grads = [G.buf[:0], G.views[0], G.buf[:0], G.views[1]]
    d = fo.descriptors(states, grads)
    fo.fo_adamw_step(d, 4, fo.make_format(), U.hparams_adamw(wl, 1))
    torch.cuda.synchronize()
    for ti in range(2):
        o = U.OracleSample(wl, ti, np.arange(1))
        o.step(1)
        exp = o.expected()
        assert all(v == 0 for v in U.mismatches(exp, U.gather_device(P, ti, exp)).values())


@pytest.mark.parametrize("fill", [0, LARGE])
def test_many_tensors_split_across_launches(fill):
    """1000 tensors in one call: more than one launch's parameter block holds
    (384 descriptors), so the call is split into several launches (with a
    3 * 2^25-element tensor in the middle).
    Every byte of every tensor (sampled groups of the large one) against the
    oracle."""
    rng = np.random.default_rng(17)
    sizes = [int(v) for v in rng.integers(1, 2600, 1000)]
    for i in range(0, 1000, 97):
        sizes[i] = 1536 * int(rng.integers(1, 4))     # whole chunks: the staged path
    if fill:
        sizes[500] = fill
    wl = _ragged_workload("adamw", "bf16", "bf16", 8)
    wl.tensors = [TensorSpec(f"t{i}", (n,), "normal", 0.02) for i, n in enumerate(sizes)]
    _run_full_compare(wl, 2, sample_above=1 << 20)


# ---- gradient release == one multi-tensor launch -------------------------------------

def test_release_order_equals_multitensor_gpt2_shapes():
    wl = workload("gpt2-small-124M")
    A = U.device_state(wl)
    B = U.device_state(wl)
    G = U.GradArena(A)
    order = list(range(len(wl.tensors)))[::-1]
    for t in (1, 2, 3):
        G.fill(wl, t)
        U.step(wl, A, G, t)
        U.step(wl, B, G, t, order=order)
    torch.cuda.synchronize()
    for name in ("w", "ecc", "m_q", "m_scale", "v_q", "v_scale"):
        assert torch.equal(getattr(A, name), getattr(B, name)), name


# ---- full-size workloads in the benchmark's launch configuration ---------------------

def _sampled_check(wl, P, orcs, tag):
    torch.cuda.synchronize()
    bad = {}
    for ti, o in orcs.items():
        exp = o.expected()
        mm = U.mismatches(exp, U.gather_device(P, ti, exp))
        if any(mm.values()):
            bad[ti] = mm
    assert not bad, (wl.name, tag, bad)


def test_gpt2_small_101_steps_sampled():
    """GPT-2-small parameter list, 100 warm steps + 1 (the benchmark's
    workload of this size), one multi-tensor launch per step; the oracle
    replays the same seeded inputs for 2 sampled groups per tensor (plus the
    first and last group) over all 101 steps; bytes compared at 1, 100, 101."""
    wl = workload("gpt2-small-124M")
    P = U.device_state(wl)
    G = U.GradArena(P)
    rng = np.random.default_rng(1)
    orcs = {ti: U.OracleSample(wl, ti, U.sample_groups(t.numel, 2, rng)) for ti, t in enumerate(wl.tensors)}
    for t in range(1, wl.warm_steps + 2):
        G.fill(wl, t)
        U.step(wl, P, G, t)
        for o in orcs.values():
            o.step(t)
        if t in (1, 100, 101):
            _sampled_check(wl, P, orcs, f"step {t}")


def test_gpt2_small_sgdm_sampled():
    """The GPT-2-small list stepped by SGD-momentum (fp16 + 8-bit ECC, the
    profiling case for SGD-momentum at a size ten times the L2): 4 sampled
    groups per tensor (plus the first and last) against the oracle after
    steps 1 and 2."""
    wl = workload("gpt2-small-124M-sgdm")
    P = U.device_state(wl)
    G = U.GradArena(P)
    rng = np.random.default_rng(2)
    orcs = {ti: U.OracleSample(wl, ti, U.sample_groups(t.numel, 4, rng)) for ti, t in enumerate(wl.tensors)}
    for t in (1, 2):
        G.fill(wl, t)
        U.step(wl, P, G, t)
        for o in orcs.values():
            o.step(t)
        _sampled_check(wl, P, orcs, f"step {t}")


def test_resnet50_sgdm_every_byte():
    wl = workload("resnet50-25.6M")
    _run_full_compare(wl, 2)


@pytest.mark.parametrize("mode", ["multi", "release", "ecc16"])
def test_llama_8b_sampled(mode):
    """Llama-3.1-8B parameter list at full size (8.03e9 parameters): one
    multi-tensor launch (the benchmark's configuration), the 291 per-tensor
    calls in reverse layer order, and the 16-bit-ECC variant; sampled groups
    of every tensor against the oracle."""
    if mode == "ecc16":
        wl = workload("llama3.1-8b-ecc16")
    else:
        wl = workload("llama3.1-8b")
    P = U.device_state(wl)
    G = U.GradArena(P)
    G.fill(wl, 1)
    order = list(range(len(wl.tensors)))[::-1] if mode == "release" else None
    U.step(wl, P, G, 1, order=order)
    rng = np.random.default_rng(2)
    orcs = {ti: U.OracleSample(wl, ti, U.sample_groups(t.numel, 48, rng)) for ti, t in enumerate(wl.tensors)}
    for o in orcs.values():
        o.step(1)
    _sampled_check(wl, P, orcs, mode)
    del P, G
    torch.cuda.empty_cache()


# ---- exact rounding ties of the 8-bit codes ------------------------------------------

def _tie_groups(n_groups=96, seed=3):
    """bf16 gradients whose step-1 momentum / variance codes land exactly on
    a half-integer before rounding (127*c or sqrt(v)*k == q + 0.5), so that a
    code computed with one rounding fewer (a fused multiply-add) would differ.
    Found by a binary32 numpy search; element 0 of a group fixes its scale."""
    f = np.float32
    rng = np.random.default_rng(seed)
    allg = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    gv = (allg.astype(np.uint32) << 16).view(np.float32)
    ok = np.isfinite(gv) & (np.abs(gv) > 1e-12)
    groups = []
    for _ in range(n_groups * 400):
        G = f(rng.uniform(2e-4, 5e-3))
        Gb = gen.to_16bit(np.array([G], np.float32), "bf16")[0]
        G = np.array([Gb], np.uint16).astype(np.uint32) << 16
        G = G.view(np.float32)[0]
        cand = ok & (np.abs(gv) < abs(G))
        g = gv[cand]
        mn = (f(0.1) * g).astype(np.float32)
        A = abs(f(f(0.1) * G))
        S = oracle.scale_fp16(np.array([A], np.float32))[0]
        Sf = np.array([S], np.uint16).view(np.float16).astype(np.float32)[0]
        r = f(1) / Sf
        y = (mn * r).astype(np.float32)
        c = ((f(2) * y) / (f(1) + np.abs(y))).astype(np.float32)
        t = (f(127) * c).astype(np.float32)
        tie_m = (t - np.floor(t)) == f(0.5)
        vn = (f(1 - 0.999) * (g * g)).astype(np.float32)
        s = np.sqrt(vn)
        Av = np.sqrt(f(f(1 - 0.999) * (G * G)))
        Sv = oracle.scale_fp16(np.array([Av], np.float32))[0]
        Svf = np.array([Sv], np.uint16).view(np.float16).astype(np.float32)[0]
        tv = (s * (f(255) / Svf)).astype(np.float32)
        tie_v = (tv - np.floor(tv)) == f(0.5)
        pick = np.nonzero(tie_m | tie_v)[0]
        if pick.size < 1:
            continue
        sel = rng.choice(pick, size=min(31, pick.size), replace=False)
        fill = rng.choice(g.size, size=31 - sel.size, replace=False)
        grp = np.concatenate([[G], g[sel], g[fill]]).astype(np.float32)
        groups.append(grp)
        if len(groups) == n_groups:
            break
    assert len(groups) >= 16
    return np.concatenate(groups)


@pytest.mark.parametrize("shift", [0, 1])
def test_code_rounding_ties_bit_exact(shift):
    g32 = _tie_groups()
    n = g32.size
    gb = gen.to_16bit(g32, "bf16")
    rng = np.random.default_rng(9)
    x = (rng.standard_normal(n) * 0.02).astype(np.float32)
    w, e = oracle.encode_master(x, 0, 8)
    st = oracle.State.zeros_like_master(w, e)
    pad = 64
    ng = (n + 31) // 32
    bufs = [torch.zeros(n + pad, dtype=dt, device=DEV) for dt in (torch.int16, torch.int8, torch.int8, torch.uint8, torch.int16)]
    sc = [torch.zeros(ng + pad, dtype=torch.int16, device=DEV) for _ in range(2)]
    wv, ev, mqv, vqv, gv = (b[shift:shift + n] for b in bufs)
    wv.copy_(torch.from_numpy(w.view(np.int16)))
    ev.copy_(torch.from_numpy(e))
    gv.copy_(torch.from_numpy(gb.view(np.int16)))
    dst = fo.TensorState(wv, ev, mqv, sc[0][:ng], vqv, sc[1][:ng])
    hp = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01)
    fo.fo_adamw_step(fo.descriptors([dst], [gv]), 1, fo.make_format(), fo.fo_adamw_hparams(**hp, step=1))
    oracle.adamw_step(st, gb, **hp, step=1)
    torch.cuda.synchronize()
    assert np.array_equal(mqv.cpu().numpy(), st.mq)
    assert np.array_equal(vqv.cpu().numpy(), st.vq)
    assert np.array_equal(U.to_np_bytes(sc[0][:ng]), st.ms)
    assert np.array_equal(U.to_np_bytes(sc[1][:ng]), st.vs)
    assert np.array_equal(U.to_np_bytes(wv), st.w)
    assert np.array_equal(ev.cpu().numpy(), st.ecc)

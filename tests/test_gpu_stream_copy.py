"""fo_stream_copy (the bandwidth-ceiling pass that moves the step's bytes with
the step's staging and stores but no arithmetic) must leave every byte of
every array unchanged: staged chunks, ragged tails, misaligned views (with
canaries around them), both byte mixes and both ECC widths."""
import numpy as np
import pytest
import torch

from bit_states_b200 import fo
from workloads.shapes import TensorSpec, Workload, ADAMW_HP

import gpu_util as U

pytestmark = pytest.mark.gpu

DEV = "cuda"
SIZES = [1, 31, 33, 255, 257, 512, 513, 1000, 4097, 65537]


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    from bit_states_b200 import build as fobuild
    from workloads import device as wdev

    fobuild.build()
    wdev.build()
    fo.load()
    yield
    torch.cuda.synchronize()


def _snapshot(P):
    out = []
    for st in P.states:
        out.append({k: getattr(st, k).clone() for k in ("w", "ecc", "m_q", "m_scale", "v_q", "v_scale")
                    if getattr(st, k) is not None})
    return out


@pytest.mark.parametrize("adamw_mix", [True, False])
@pytest.mark.parametrize("nbits", [8, 16])
def test_stream_copy_leaves_every_byte(adamw_mix, nbits):
    ts = [TensorSpec(f"t{i}", (n,), "normal", 0.02) for i, n in enumerate(SIZES)]
    wl = Workload(name="copy", tensors=ts, optimizer="adamw", hparams=dict(ADAMW_HP), w_dtype="bf16",
                  grad_dtype="bf16", ecc_bits=nbits, seed=11)
    P = U.device_state(wl)
    G = U.GradArena(P)
    G.fill(wl, 1)
    # give the states non-trivial bytes with one real step first
    U.step(wl, P, G, 1)
    torch.cuda.synchronize()
    before = _snapshot(P)
    g_before = G.buf.clone()
    fmt = U.fmt_of(wl)
    d = fo.descriptors(P.states, G.views)
    for _ in range(3):
        fo.fo_stream_copy(d, len(P.states), fmt, adamw_mix)
    torch.cuda.synchronize()
    after = _snapshot(P)
    for i, (b, a) in enumerate(zip(before, after)):
        for k in b:
            assert torch.equal(b[k], a[k]), (i, k)
    assert torch.equal(g_before, G.buf)


@pytest.mark.parametrize("shift", [1, 3, 8])
def test_stream_copy_misaligned_views_and_canaries(shift):
    n, pad = 3000, 64
    ng = (n + 31) // 32
    rng = np.random.default_rng(shift)
    mk = lambda dt, cnt: torch.from_numpy(rng.integers(-100, 100, cnt + 2 * pad).astype(np.int64)).to(DEV).to(dt)
    w, e, mq, vq, g = mk(torch.int16, n), mk(torch.int8, n), mk(torch.int8, n), mk(torch.uint8, n), mk(torch.int16, n)
    ms, vs = mk(torch.int16, ng), mk(torch.int16, ng)
    s = shift
    views = dict(w=w[pad + s:pad + s + n], e=e[pad + s:pad + s + n], mq=mq[pad + s:pad + s + n],
                 vq=vq[pad + s:pad + s + n], g=g[pad + s:pad + s + n], ms=ms[pad + 1:pad + 1 + ng],
                 vs=vs[pad + 1:pad + 1 + ng])
    full = dict(w=w, e=e, mq=mq, vq=vq, g=g, ms=ms, vs=vs)
    before = {k: v.clone() for k, v in full.items()}
    st = fo.TensorState(views["w"], views["e"], views["mq"], views["ms"], views["vq"], views["vs"])
    fo.fo_stream_copy(fo.descriptors([st], [views["g"]]), 1, fo.make_format(), True)
    torch.cuda.synchronize()
    for k, t in full.items():
        assert torch.equal(t, before[k]), k

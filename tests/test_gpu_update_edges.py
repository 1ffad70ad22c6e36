"""GPU parity on constructed inputs at the edges of the AdamW fast path's
validity conditions (its Newton-Raphson square root and quotient, the
finite-range checks on the weights): zero and tiny weights, bf16 subnormal
and exactly zero gradients, gradients large enough to push the divisor above
2^20 or the first moment above 2^21, weights close to the bf16 maximum, and
hyper-parameters (eps below 2^-60, a step size below 2^-80, lr = 0)
under which the kernel must take its exact path everywhere.  Every emitted
byte must equal the oracle's after each of three steps.

The "AdamW" update is the one of "FlashOptim: Breaking the Memory Wall with
24-bit Weights and Companded States" (section "Method"), with the readings
the oracle states.  Inputs stay finite (no NaN payloads to compare).
"""
import numpy as np
import pytest
import torch

import oracle
from bit_states_b200 import fo
from workloads import gen

import gpu_util as U

pytestmark = pytest.mark.gpu

DEV = "cuda"
CHUNK = 1536  # whole staged chunks of the kernels (768 elements for AdamW with 8-bit ECC, 512 otherwise)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    from bit_states_b200 import build as fobuild

    fobuild.build()
    fo.load()
    yield
    torch.cuda.synchronize()


def _blocks(rng, wdt):
    """(weights, per-step gradient generator) for one block each."""
    f32 = np.float32
    big_w = 3.0e38 if wdt == "bf16" else 6.0e4

    def normal_w():
        return (rng.standard_normal(CHUNK) * 0.02).astype(f32)

    def normal_g(r):
        return (r.standard_normal(CHUNK) * 1e-3).astype(f32)

    blocks = []
    # ordinary block (fast path)
    blocks.append((normal_w(), normal_g))
    # zero weights (+0 and -0) with ordinary gradients
    w = np.zeros(CHUNK, f32)
    w[1::2] = -0.0
    blocks.append((w, normal_g))
    # zero weights with bf16-subnormal, zero and tiny gradients
    blocks.append((w.copy(), lambda r: np.where(r.random(CHUNK) < 0.3, f32(0.0),
                                               (r.standard_normal(CHUNK) * 1e-39)).astype(f32)))
    # tiny weights with ordinary gradients
    blocks.append(((rng.standard_normal(CHUNK) * 1e-30).astype(f32), normal_g))
    # gradients so large that sqrt(v') / sqrt(1 - b2^t) + eps exceeds 2^20
    blocks.append((normal_w(), lambda r: (r.standard_normal(CHUNK) * 3e6).astype(f32)))
    # gradients so large that |m'| exceeds 2^21
    blocks.append((normal_w(), lambda r: (r.standard_normal(CHUNK) * 1e8).astype(f32)))
    # mixed: a few huge entries among ordinary ones
    def mixed_g(r):
        g = normal_g(r)
        g[r.choice(CHUNK, 3, replace=False)] = f32(2e7)
        return g
    blocks.append((normal_w(), mixed_g))
    # weights near the largest finite 16-bit value
    blocks.append(((np.sign(rng.standard_normal(CHUNK)) * big_w * (1 - 0.01 * rng.random(CHUNK))).astype(f32),
                   normal_g))
    # exactly zero gradients on ordinary weights (zero first moment at step 1)
    blocks.append((normal_w(), lambda r: np.zeros(CHUNK, f32)))
    return blocks


HP_CASES = {
    "standard": dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01),
    "eps_1e-20": dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-20, weight_decay=0.01),
    "eps_1e-30_wd0": dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-30, weight_decay=0.0),
    "lr_1e-30": dict(lr=1e-30, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01),
    "lr_0": dict(lr=0.0, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01),
    "eps_1_beta1_0": dict(lr=1e-2, beta1=0.0, beta2=0.99, eps=1.0, weight_decay=0.1),
}


@pytest.mark.parametrize("nbits", [8, 16])
@pytest.mark.parametrize("wdt", ["bf16", "fp16"])
@pytest.mark.parametrize("hp_name", list(HP_CASES))
def test_update_edges_every_byte(wdt, hp_name, nbits):
    hp = HP_CASES[hp_name]
    rng = np.random.default_rng(20 + len(hp_name))
    blocks = _blocks(rng, wdt)
    tail = 77  # a ragged last chunk: the scalar path
    x = np.concatenate([b[0] for b in blocks] + [(rng.standard_normal(tail) * 0.02).astype(np.float32)])
    n = x.size
    wcode = 0 if wdt == "bf16" else 1
    w, e = oracle.encode_master(x, wcode, nbits)
    st = oracle.State.zeros_like_master(w, e)
    ng = (n + 31) // 32
    wv = torch.from_numpy(w.view(np.int16).copy()).to(DEV)
    ev = torch.from_numpy(e.copy()).to(DEV)  # int8 or int16 codes
    mqv = torch.zeros(n, dtype=torch.int8, device=DEV)
    vqv = torch.zeros(n, dtype=torch.uint8, device=DEV)
    msv = torch.zeros(ng, dtype=torch.int16, device=DEV)
    vsv = torch.zeros(ng, dtype=torch.int16, device=DEV)
    gv = torch.zeros(n, dtype=torch.int16, device=DEV)
    dst = fo.TensorState(wv, ev, mqv, msv, vqv, vsv)
    fmt = fo.make_format(wdt, "bf16", nbits)
    for t in range(1, 4):
        r = np.random.default_rng(1000 * t + len(hp_name))
        g32 = np.concatenate([b[1](r) for b in blocks] + [(r.standard_normal(tail) * 1e-3).astype(np.float32)])
        gb = gen.to_16bit(g32.astype(np.float32), "bf16")
        gv.copy_(torch.from_numpy(gb.view(np.int16)))
        fo.fo_adamw_step(fo.descriptors([dst], [gv]), 1, fmt, fo.fo_adamw_hparams(**hp, step=t))
        oracle.adamw_step(st, gb, **hp, step=t, wdt=wcode, gdt=0, ecc_bits=nbits)
        torch.cuda.synchronize()
        for name, got, exp in (("w", U.to_np_bytes(wv), st.w.view(np.uint16)),
                               ("ecc", ev.cpu().numpy(), st.ecc),
                               ("m_q", mqv.cpu().numpy(), st.mq),
                               ("v_q", vqv.cpu().numpy(), st.vq),
                               ("m_scale", U.to_np_bytes(msv), st.ms.view(np.uint16)),
                               ("v_scale", U.to_np_bytes(vsv), st.vs.view(np.uint16))):
            bad = np.nonzero(got.view(exp.dtype) != exp)[0]
            assert bad.size == 0, f"step {t} {name}: {bad.size} mismatches, first at {bad[:5]}"

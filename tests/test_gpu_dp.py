"""The data-parallel sharded step's CUDA path (communication stream, events,
NCCL collectives, the fused kernel on each bucket slice) on one GPU: a
world-size-1 NCCL group, so the collectives are copies and no rank waits on
another.  Every byte must equal the oracle stepping each tensor on its own
(the step is the FlashOptim-style AdamW / SGD-momentum of "FlashOptim:
Breaking the Memory Wall with 24-bit Weights and Companded States"), and one
fused multi-tensor call on the same tensors.  (Two or more GPUs are not
available here; the exchange between ranks is covered on CPU by
tests/test_dp_gloo.py.)"""
import socket

import numpy as np
import pytest
import torch

import oracle
from bit_states_b200 import fo
from bit_states_b200.dp import GROUP, DataParallelStep, FlatLayout, ShardedState
from workloads import gen


pytestmark = pytest.mark.gpu

NUMELS = [100, 4096 + 7, 1, 3000, 33, 70000, 2 * 768 * 40 + 5]
HP = {"adamw": dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01),
      "sgdm": dict(lr=0.1, momentum=0.9, dampening=0.0, weight_decay=1e-4, nesterov=False)}
DTYPE = {"adamw": "bf16", "sgdm": "fp16"}


@pytest.fixture(scope="module")
def pg():
    import torch.distributed as dist

    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    from bit_states_b200 import build as fobuild

    fobuild.build()
    fo.load()
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1)
    yield dist
    torch.cuda.synchronize()
    dist.destroy_process_group()


def _fresh(n, adam, dev):
    ng = (n + 31) // 32
    return fo.TensorState(torch.empty(n, dtype=torch.int16, device=dev), torch.empty(n, dtype=torch.int8, device=dev),
                          torch.zeros(n, dtype=torch.int8, device=dev), torch.zeros(ng, dtype=torch.int16, device=dev),
                          torch.zeros(n, dtype=torch.uint8, device=dev) if adam else None,
                          torch.zeros(ng, dtype=torch.int16, device=dev) if adam else None)


@pytest.mark.parametrize("optimizer", ["adamw", "sgdm"])
def test_dp_step_one_rank_equals_oracle_and_fused_step(pg, optimizer):
    dev = torch.device("cuda", 0)
    adam = optimizer == "adamw"
    dt = DTYPE[optimizer]
    dcode = 0 if dt == "bf16" else 1
    hp = HP[optimizer]
    layout = FlatLayout(NUMELS, 1, bucket_groups=512)
    st = ShardedState(layout, 0, dev, adam=adam)
    fmt = fo.make_format(dt, dt, 8)
    dp = DataParallelStep(st, fmt=fmt, hparams=hp, reduce_op="sum", grad_dtype=dt, w_dtype=dt,
                          optimizer=optimizer)
    xs = [gen.normal(gen.stream_key(0, ti, 0, gen.KIND_MASTER), np.arange(n), 0.02) for ti, n in enumerate(NUMELS)]
    ref = [_fresh(n, adam, dev) for n in NUMELS]
    orc = []
    x32 = torch.zeros(layout.numel, dtype=torch.float32, device=dev)
    for ti, (n, x) in enumerate(zip(NUMELS, xs)):
        xd = torch.from_numpy(x).to(dev)
        fo.fo_encode_master(xd, ref[ti].w, ref[ti].ecc, n, fmt)
        layout.tensor_view(x32, ti).copy_(xd)
        w, e = oracle.encode_master(x, dcode, 8)
        orc.append(oracle.State.zeros_like_master(w, e, adam=adam))
    st.encode_from(x32, fmt, w_dtype=dt)
    for t in (1, 2, 3):
        gb = [gen.to_16bit(gen.normal(gen.stream_key(0, ti, t, gen.KIND_GRAD), np.arange(n), 1e-3 if adam else 1e-2),
                           dt) for ti, n in enumerate(NUMELS)]
        gs = [torch.from_numpy(g.view(np.int16)).to(dev) for g in gb]
        flat = torch.zeros(layout.numel, dtype=torch.int16, device=dev)
        for ti, g in enumerate(gs):
            layout.tensor_view(flat, ti).copy_(g)
        dp.step(flat, t)
        if adam:
            fo.fo_adamw_step(fo.descriptors(ref, gs), len(ref), fmt, fo.fo_adamw_hparams(**hp, step=t))
            for o, g in zip(orc, gb):
                oracle.adamw_step(o, g, **hp, step=t, wdt=dcode, gdt=dcode, ecc_bits=8)
        else:
            fo.fo_sgdm_step(fo.descriptors(ref, gs), len(ref), fmt,
                            fo.fo_sgdm_hparams(hp["lr"], hp["momentum"], hp["dampening"], hp["weight_decay"],
                                               int(hp["nesterov"]), t))
            for o, g in zip(orc, gb):
                oracle.sgdm_step(o, g, **hp, step=t, wdt=dcode, gdt=dcode, ecc_bits=8)
        torch.cuda.synchronize()
        for ti, n in enumerate(NUMELS):
            o = layout.offsets[ti]
            ng = (n + 31) // 32
            go = o // GROUP
            got = {"w": st.w[o:o + n], "ecc": st.ecc[o:o + n], "m_q": st.m_q[o:o + n],
                   "m_scale": st.m_scale[go:go + ng]}
            exp = {"w": orc[ti].w, "ecc": orc[ti].ecc, "m_q": orc[ti].mq, "m_scale": orc[ti].ms}
            if adam:
                got.update(v_q=st.v_q[o:o + n], v_scale=st.v_scale[go:go + ng])
                exp.update(v_q=orc[ti].vq, v_scale=orc[ti].vs)
            for k, g in got.items():
                assert torch.equal(g, getattr(ref[ti], k)), (t, ti, k, "fused step")
                a = g.cpu().numpy()
                e = exp[k]
                bad = np.count_nonzero(a.view(np.uint8 if a.itemsize == 1 else np.uint16) !=
                                       e.view(np.uint8 if e.itemsize == 1 else np.uint16))
                assert bad == 0, (t, ti, k, f"{bad} bytes differ from the oracle")
            # the padding of the flat layout stays zero
            pad = st.w[o + n:o + ng * GROUP]
            assert torch.count_nonzero(pad) == 0, (t, ti, "padding")

"""The data-parallel sharded step's CUDA path (communication stream, events,
NCCL collectives, the fused kernel on each bucket slice) on one GPU: a
world-size-1 NCCL group, so the collectives are copies and no rank waits on
another.  Its bytes must equal one fused multi-tensor step on the same
tensors.  (Two or more GPUs are not available here; the exchange between ranks
is covered on CPU by tests/test_dp_gloo.py.)"""
import socket

import numpy as np
import pytest
import torch

from bit_states_b200 import fo
from bit_states_b200.dp import GROUP, DataParallelStep, FlatLayout, ShardedState
from workloads import gen


pytestmark = pytest.mark.gpu

NUMELS = [100, 4096 + 7, 1, 3000, 33, 70000]
HP = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01)


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


def test_dp_step_one_rank_equals_fused_step(pg):
    dev = torch.device("cuda", 0)
    layout = FlatLayout(NUMELS, 1, bucket_groups=512)
    st = ShardedState(layout, 0, dev)
    fmt = fo.make_format()
    dp = DataParallelStep(st, fmt=fmt, hparams=HP, reduce_op="sum")
    # reference: one tensor list stepped by one fused call
    xs = [gen.normal(gen.stream_key(0, ti, 0, gen.KIND_MASTER), np.arange(n), 0.02) for ti, n in enumerate(NUMELS)]
    ref = [fo.TensorState(torch.empty(n, dtype=torch.int16, device=dev), torch.empty(n, dtype=torch.int8, device=dev),
                          torch.zeros(n, dtype=torch.int8, device=dev),
                          torch.zeros((n + 31) // 32, dtype=torch.int16, device=dev),
                          torch.zeros(n, dtype=torch.uint8, device=dev),
                          torch.zeros((n + 31) // 32, dtype=torch.int16, device=dev)) for n in NUMELS]
    x32 = torch.zeros(layout.numel, dtype=torch.float32, device=dev)
    for ti, (n, x) in enumerate(zip(NUMELS, xs)):
        xd = torch.from_numpy(x).to(dev)
        fo.fo_encode_master(xd, ref[ti].w, ref[ti].ecc, n, fmt)
        layout.tensor_view(x32, ti).copy_(xd)
    st.encode_from(x32, fmt)
    for t in (1, 2, 3):
        gs = [torch.from_numpy(gen.to_16bit(gen.normal(gen.stream_key(0, ti, t, gen.KIND_GRAD), np.arange(n), 1e-3),
                                            "bf16").view(np.int16)).to(dev) for ti, n in enumerate(NUMELS)]
        flat = torch.zeros(layout.numel, dtype=torch.int16, device=dev)
        for ti, g in enumerate(gs):
            layout.tensor_view(flat, ti).copy_(g)
        dp.step(flat, t)
        fo.fo_adamw_step(fo.descriptors(ref, gs), len(ref), fmt, fo.fo_adamw_hparams(**HP, step=t))
    torch.cuda.synchronize()
    for ti, n in enumerate(NUMELS):
        o = layout.offsets[ti]
        ng = (n + 31) // 32
        go = o // GROUP
        assert torch.equal(st.w[o:o + n], ref[ti].w), ti
        assert torch.equal(st.ecc[o:o + n], ref[ti].ecc), ti
        assert torch.equal(st.m_q[o:o + n], ref[ti].m_q), ti
        assert torch.equal(st.v_q[o:o + n], ref[ti].v_q), ti
        assert torch.equal(st.m_scale[go:go + ng], ref[ti].m_scale), ti
        assert torch.equal(st.v_scale[go:go + ng], ref[ti].v_scale), ti

"""Data-parallel sharded step on CPU ranks (gloo, world size 2): gradients
reduce-scattered to the owners of their groups, each rank steps its slice of
every bucket, the updated downcast weights all-gathered.  The bytes (the
replicated x' on every rank, each rank's ECC / codes / scales) must equal one
process stepping every tensor with the summed gradients.  The step on a rank
is the oracle here (the GPU path passes the same slices to the fused kernel);
the layout, the bucket slicing and the collectives are the code under test."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from bit_states_b200.dp import GROUP, FlatLayout

NUMELS = [100, 4096 + 7, 1, 3000, 33, 2048]
HP = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01)
BUCKET_GROUPS = 40


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _masters(ti, n):
    from workloads import gen

    return gen.normal(gen.stream_key(0, ti, 0, gen.KIND_MASTER), np.arange(n), 0.02)


def _grads(rank, ti, t, n):
    from workloads import gen

    return gen.to_16bit(gen.normal(gen.stream_key(rank + 1, ti, t, gen.KIND_GRAD), np.arange(n), 1e-3), "bf16")


def _flat(layout, per_tensor, dtype):
    out = np.zeros(layout.numel, dtype)
    for ti, a in enumerate(per_tensor):
        o = layout.offsets[ti]
        out[o:o + a.size] = a
    return out


def _oracle_step_fn(state, grad, t, stream):
    import oracle

    st = oracle.State(state.w.numpy().view(np.uint16), state.ecc.numpy(), state.m_q.numpy(),
                      state.m_scale.numpy().view(np.uint16), state.v_q.numpy(),
                      state.v_scale.numpy().view(np.uint16))
    oracle.adamw_step(st, grad.numpy().view(np.uint16), **HP, step=t)


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist

    import oracle
    from bit_states_b200.dp import DataParallelStep, ShardedState

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        layout = FlatLayout(NUMELS, world, bucket_groups=BUCKET_GROUPS)
        st = ShardedState(layout, rank, "cpu")
        w, e = zip(*[oracle.encode_master(_masters(ti, n)) for ti, n in enumerate(NUMELS)])
        wf, ef = _flat(layout, w, np.uint16), _flat(layout, e, np.int8)
        st.w.copy_(torch.from_numpy(wf.view(np.int16)))
        for s0, s1, go in st.slices:
            st.ecc[go * GROUP:go * GROUP + (s1 - s0)] = torch.from_numpy(ef[s0:s1])
        dp = DataParallelStep(st, step_fn=_oracle_step_fn, reduce_op="sum")
        for t in (1, 2):
            g = _flat(layout, [_grads(rank, ti, t, n) for ti, n in enumerate(NUMELS)], np.uint16)
            dp.step(torch.from_numpy(g.view(np.int16)), t)
        q.put((rank, st.w.numpy().copy(), st.ecc.numpy().copy(), st.m_q.numpy().copy(),
               st.m_scale.numpy().copy(), st.v_q.numpy().copy(), st.v_scale.numpy().copy(),
               list(st.slices)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _bf16_sum(a, b):
    f = lambda u: (u.astype(np.uint32) << 16).view(np.float32)
    s = f(a) + f(b)                       # one binary32 addition (exact for two bf16 values)
    from workloads import gen

    return gen.to_16bit(s.astype(np.float32), "bf16")


def test_layout_buckets_cover_every_group_once():
    for world in (1, 2, 3, 8):
        L = FlatLayout(NUMELS, world, bucket_groups=BUCKET_GROUPS)
        owned = []
        for r in range(world):
            for b in L.buckets:
                g0, k = b.shard(world, r)
                owned.extend(range(g0, g0 + k))
        assert sorted(owned) == list(range(L.groups))
        assert all(b.groups % world == 0 for b in L.buckets)
        real = sum((n + 31) // 32 for n in NUMELS)
        assert real <= L.groups < real + len(L.buckets) * world


def test_two_rank_dp_step_equals_single_process():
    import oracle

    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(2):
        r = q.get(timeout=300)
        res[r[0]] = r[1:]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    layout = FlatLayout(NUMELS, 2, bucket_groups=BUCKET_GROUPS)
    # single-process reference: every tensor stepped with the summed gradients
    exp = []
    for ti, n in enumerate(NUMELS):
        w, e = oracle.encode_master(_masters(ti, n))
        st = oracle.State.zeros_like_master(w, e)
        for t in (1, 2):
            oracle.adamw_step(st, _bf16_sum(_grads(0, ti, t, n), _grads(1, ti, t, n)), **HP, step=t)
        exp.append(st)
    for rank in (0, 1):
        w, ecc, mq, ms, vq, vs, slices = res[rank]
        for ti, n in enumerate(NUMELS):
            o = layout.offsets[ti]
            assert np.array_equal(w[o:o + n].view(np.uint16), exp[ti].w), (rank, ti)
        # owned groups: map back to (tensor, group)
        for s0, s1, go in slices:
            for g in range(s0 // GROUP, s1 // GROUP):
                e0 = g * GROUP
                ti = max(i for i in range(len(NUMELS)) if layout.offsets[i] <= e0)
                lg = (e0 - layout.offsets[ti]) // GROUP
                n = NUMELS[ti]
                if lg * GROUP >= n:          # padding group
                    continue
                k = go + (g - s0 // GROUP)
                a, b = lg * GROUP, min(n, lg * GROUP + GROUP)
                L = b - a
                assert np.array_equal(ecc[k * GROUP:k * GROUP + L], exp[ti].ecc[a:b]), (rank, ti, lg)
                assert np.array_equal(mq[k * GROUP:k * GROUP + L], exp[ti].mq[a:b]), (rank, ti, lg)
                assert np.array_equal(vq[k * GROUP:k * GROUP + L], exp[ti].vq[a:b]), (rank, ti, lg)
                assert ms.view(np.uint16)[k] == exp[ti].ms[lg] and vs.view(np.uint16)[k] == exp[ti].vs[lg]


# ---- SGD-momentum, fp16 weights and gradients, three ranks ---------------------------

SGD_HP = dict(lr=0.1, momentum=0.9, dampening=0.0, weight_decay=1e-4, nesterov=False)


def _small_int_grads(rank, ti, t, n):
    """fp16 gradients k * 2^-12 with small integers k in [-8, 8]: the sum over
    three ranks is exact in fp16 in every order, so the collective's
    reduction order cannot change the reference."""
    from workloads import gen

    u = gen.normal(gen.stream_key(rank + 11, ti, t, gen.KIND_GRAD), np.arange(n), 1.0)
    k = np.clip(np.rint(3.0 * u), -8, 8).astype(np.int32)
    return k


def _to_fp16_bits(k):
    return (k.astype(np.float32) * np.float32(2.0 ** -12)).astype(np.float16).view(np.uint16)


def _oracle_sgdm_step_fn(state, grad, t, stream):
    import oracle

    st = oracle.State(state.w.numpy().view(np.uint16), state.ecc.numpy(), state.m_q.numpy(),
                      state.m_scale.numpy().view(np.uint16))
    oracle.sgdm_step(st, grad.numpy().view(np.uint16), **SGD_HP, step=t, wdt=oracle.FP16, gdt=oracle.FP16)


def _sgd_worker(rank, world, port, q):
    import torch
    import torch.distributed as dist

    import oracle
    from bit_states_b200.dp import DataParallelStep, ShardedState

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        layout = FlatLayout(NUMELS, world, bucket_groups=BUCKET_GROUPS)
        st = ShardedState(layout, rank, "cpu", adam=False)
        w, e = zip(*[oracle.encode_master(_masters(ti, n), oracle.FP16) for ti, n in enumerate(NUMELS)])
        wf, ef = _flat(layout, w, np.uint16), _flat(layout, e, np.int8)
        st.w.copy_(torch.from_numpy(wf.view(np.int16)))
        for s0, s1, go in st.slices:
            st.ecc[go * GROUP:go * GROUP + (s1 - s0)] = torch.from_numpy(ef[s0:s1])
        dp = DataParallelStep(st, step_fn=_oracle_sgdm_step_fn, reduce_op="sum", grad_dtype="fp16",
                              w_dtype="fp16", optimizer="sgdm")
        for t in (1, 2, 3):
            g = _flat(layout, [_to_fp16_bits(_small_int_grads(rank, ti, t, n)) for ti, n in enumerate(NUMELS)],
                      np.uint16)
            dp.step(torch.from_numpy(g.view(np.int16)), t)
        q.put((rank, st.w.numpy().copy(), st.ecc.numpy().copy(), st.m_q.numpy().copy(),
               st.m_scale.numpy().copy(), list(st.slices)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_three_rank_sgdm_fp16_equals_single_process():
    import oracle

    world = 3
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_sgd_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        r = q.get(timeout=300)
        res[r[0]] = r[1:]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    layout = FlatLayout(NUMELS, world, bucket_groups=BUCKET_GROUPS)
    exp = []
    for ti, n in enumerate(NUMELS):
        w, e = oracle.encode_master(_masters(ti, n), oracle.FP16)
        st = oracle.State.zeros_like_master(w, e, adam=False)
        for t in (1, 2, 3):
            ksum = sum(_small_int_grads(r, ti, t, n) for r in range(world))
            oracle.sgdm_step(st, _to_fp16_bits(ksum), **SGD_HP, step=t, wdt=oracle.FP16, gdt=oracle.FP16)
        exp.append(st)
    seen = 0
    for rank in range(world):
        w, ecc, mq, ms, slices = res[rank]
        for ti, n in enumerate(NUMELS):
            o = layout.offsets[ti]
            assert np.array_equal(w[o:o + n].view(np.uint16), exp[ti].w), (rank, ti)
        for s0, s1, go in slices:
            for g in range(s0 // GROUP, s1 // GROUP):
                e0 = g * GROUP
                ti = max(i for i in range(len(NUMELS)) if layout.offsets[i] <= e0)
                lg = (e0 - layout.offsets[ti]) // GROUP
                n = NUMELS[ti]
                if lg * GROUP >= n:
                    continue
                k = go + (g - s0 // GROUP)
                a, b = lg * GROUP, min(n, lg * GROUP + GROUP)
                L = b - a
                assert np.array_equal(ecc[k * GROUP:k * GROUP + L], exp[ti].ecc[a:b]), (rank, ti, lg)
                assert np.array_equal(mq[k * GROUP:k * GROUP + L], exp[ti].mq[a:b]), (rank, ti, lg)
                assert ms.view(np.uint16)[k] == exp[ti].ms[lg]
                seen += 1
    assert seen == sum((n + 31) // 32 for n in NUMELS)   # every real group owned by exactly one rank


def test_dp_step_rejects_mismatched_optimizer():
    import pytest

    from bit_states_b200.dp import DataParallelStep, ShardedState

    layout = FlatLayout(NUMELS, 1, bucket_groups=BUCKET_GROUPS)
    with pytest.raises(ValueError):
        DataParallelStep(ShardedState(layout, 0, "cpu", adam=True), step_fn=lambda *a: None, optimizer="sgdm")
    with pytest.raises(ValueError):
        DataParallelStep(ShardedState(layout, 0, "cpu", adam=False), step_fn=lambda *a: None)
    with pytest.raises(ValueError):
        DataParallelStep(ShardedState(layout, 0, "cpu"), step_fn=lambda *a: None, optimizer="lamb")


def test_layout_properties_random_lists():
    """Property test of the flat layout: for random parameter lists, world
    sizes and bucket sizes, every tensor starts on a group boundary and its
    groups lie inside the layout, buckets tile the groups in order with sizes
    that are multiples of the world size, and every rank's slices are equal,
    disjoint and together cover every group exactly once."""
    hypothesis = pytest.importorskip("hypothesis")
    given, settings, hs = hypothesis.given, hypothesis.settings, hypothesis.strategies

    @settings(max_examples=200, deadline=None)
    @given(hs.lists(hs.integers(0, 5000), min_size=1, max_size=12), hs.integers(1, 8), hs.integers(1, 300))
    def check(numels, world, bucket_groups):
        L = FlatLayout(numels, world, bucket_groups=bucket_groups)
        off = 0
        for o, n in zip(L.offsets, numels):
            assert o % GROUP == 0 and o == off
            off += (n + GROUP - 1) // GROUP * GROUP
        assert off <= L.numel == L.groups * GROUP
        g = 0
        for b in L.buckets:
            assert b.g0 == g and b.groups > 0 and b.groups % world == 0
            g += b.groups
        assert g == L.groups
        owned = np.zeros(L.groups, np.int32)
        for r in range(world):
            for b in L.buckets:
                g0, k = b.shard(world, r)
                assert k == b.groups // world and b.g0 <= g0 and g0 + k <= b.g0 + b.groups
                owned[g0:g0 + k] += 1
        assert np.all(owned == 1)
        # only the last bucket is rounded up to a multiple of the world size
        assert 0 <= L.groups - off // GROUP < world

    check()


# ---- the exchange and the steps alone (what bench.py times separately) ---------------

def _split_worker(rank, world, port, q):
    import torch
    import torch.distributed as dist

    import oracle
    from bit_states_b200.dp import DataParallelStep, ShardedState

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        layout = FlatLayout(NUMELS, world, bucket_groups=BUCKET_GROUPS)
        w, e = zip(*[oracle.encode_master(_masters(ti, n)) for ti, n in enumerate(NUMELS)])
        wf, ef = _flat(layout, w, np.uint16), _flat(layout, e, np.int8)
        states = []
        for _ in range(2):
            st = ShardedState(layout, rank, "cpu")
            st.w.copy_(torch.from_numpy(wf.view(np.int16)))
            for s0, s1, go in st.slices:
                st.ecc[go * GROUP:go * GROUP + (s1 - s0)] = torch.from_numpy(ef[s0:s1])
            states.append(st)
        a = DataParallelStep(states[0], step_fn=_oracle_step_fn, reduce_op="sum")
        b = DataParallelStep(states[1], step_fn=_oracle_step_fn, reduce_op="sum")
        g = torch.from_numpy(_flat(layout, [_grads(rank, ti, 1, n) for ti, n in enumerate(NUMELS)],
                                   np.uint16).view(np.int16))
        a.step(g, 1)
        w_before = states[1].w.clone()
        b.exchange(g)
        same_w = bool(torch.equal(states[1].w, w_before))
        same_grad = bool(torch.equal(a.gown, b.gown))
        b.step_only(1)
        sa, sb = states
        owned_w = all(torch.equal(sa.w[s0:s1], sb.w[s0:s1]) for s0, s1, go in sa.slices)
        codes = all(torch.equal(getattr(sa, k), getattr(sb, k)) for k in ("ecc", "m_q", "m_scale", "v_q", "v_scale"))
        q.put((rank, same_w, same_grad, owned_w, codes))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_exchange_alone_and_steps_alone_compose_to_the_step():
    """exchange() moves the reduced gradient shards and leaves x' as it was;
    step_only() on those shards then gives the owned bytes of step()."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_split_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=300) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, same_w, same_grad, owned_w, codes in res:
        assert same_w and same_grad and owned_w and codes, (rank, same_w, same_grad, owned_w, codes)

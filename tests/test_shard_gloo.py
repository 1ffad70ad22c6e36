"""Multi-rank host logic on CPU (gloo, world_size 2): the group-aligned
partition covers every group exactly once, and stepping each rank's shard
(here with the oracle, the GPU kernel uses the same descriptors) and
gathering gives the bytes of stepping the whole list at once."""
import os
import socket

import numpy as np
import torch.multiprocessing as mp

from bit_states_b200.shard import GROUP, shard_spans


def test_spans_cover_every_group_once():
    numels = [1, 31, 32, 33, 1000, 4096, 7, 65537, 0, 5]
    for world in (1, 2, 3, 4, 7, 8):
        seen = {}
        for r in range(world):
            for sp in shard_spans(numels, world, r):
                for g in range(sp.g0, sp.g1):
                    key = (sp.tensor, g)
                    assert key not in seen
                    seen[key] = r
                assert sp.e0 % GROUP == 0
        expect = {(ti, g) for ti, n in enumerate(numels) for g in range((n + 31) // 32)}
        assert set(seen) == expect
        sizes = [sum(sp.g1 - sp.g0 for sp in shard_spans(numels, world, r)) for r in range(world)]
        assert max(sizes) - min(sizes) <= 1


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, numels, q):
    import torch
    import torch.distributed as dist

    import oracle
    from workloads import gen

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        hp = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01)
        out = {}
        for sp in shard_spans(numels, world, rank):
            idx = np.arange(sp.e0, sp.e1)
            x = gen.normal(gen.stream_key(0, sp.tensor, 0, gen.KIND_MASTER), idx, 0.02)
            w, e = oracle.encode_master(x)
            st = oracle.State.zeros_like_master(w, e)
            for t in (1, 2):
                g = gen.to_16bit(gen.normal(gen.stream_key(0, sp.tensor, t, gen.KIND_GRAD), idx, 1e-3), "bf16")
                oracle.adamw_step(st, g, **hp, step=t)
            out[(sp.tensor, sp.g0)] = (st.w, st.ecc, st.mq, st.ms, st.vq, st.vs)
        allout = [None] * world
        dist.all_gather_object(allout, out)
        if rank == 0:
            merged = {}
            for d in allout:
                merged.update(d)
            q.put(merged)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_shards_equal_whole_list():
    numels = [100, 4096 + 7, 1, 3000]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, numels, q)) for r in range(2)]
    for p in procs:
        p.start()
    merged = q.get(timeout=180)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    import oracle
    from workloads import gen

    hp = dict(lr=1e-3, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.01)
    for ti, n in enumerate(numels):
        idx = np.arange(n)
        x = gen.normal(gen.stream_key(0, ti, 0, gen.KIND_MASTER), idx, 0.02)
        w, e = oracle.encode_master(x)
        st = oracle.State.zeros_like_master(w, e)
        for t in (1, 2):
            g = gen.to_16bit(gen.normal(gen.stream_key(0, ti, t, gen.KIND_GRAD), idx, 1e-3), "bf16")
            oracle.adamw_step(st, g, **hp, step=t)
        parts = sorted((g0, v) for (tj, g0), v in merged.items() if tj == ti)
        cat = lambda k: np.concatenate([v[k] for _, v in parts])
        assert np.array_equal(cat(0), st.w) and np.array_equal(cat(1), st.ecc)
        assert np.array_equal(cat(2), st.mq) and np.array_equal(cat(3), st.ms)
        assert np.array_equal(cat(4), st.vq) and np.array_equal(cat(5), st.vs)


def test_spans_properties_random_lists():
    """Property test of the partition: for random lists and world sizes every
    group is owned by exactly one rank, ranks own contiguous runs in list order
    with sizes differing by at most one group, and the sliced views of
    shard_states cover each span's elements and scales exactly."""
    import torch
    from hypothesis import given, settings
    from hypothesis import strategies as hs

    from bit_states_b200.fo import TensorState
    from bit_states_b200.shard import shard_states

    @settings(max_examples=200, deadline=None)
    @given(hs.lists(hs.integers(0, 3000), min_size=1, max_size=10), hs.integers(1, 9))
    def check(numels, world):
        flat_owner = []
        for r in range(world):
            spans = shard_spans(numels, world, r)
            for sp in spans:
                assert 0 <= sp.g0 < sp.g1 <= (sp.numel + GROUP - 1) // GROUP
                flat_owner.extend([(sp.tensor, g, r) for g in range(sp.g0, sp.g1)])
            states = [TensorState(torch.zeros(n, dtype=torch.int16), torch.zeros(n, dtype=torch.int8),
                                  torch.zeros(n, dtype=torch.int8), torch.zeros((n + 31) // 32, dtype=torch.int16),
                                  torch.zeros(n, dtype=torch.uint8), torch.zeros((n + 31) // 32, dtype=torch.int16))
                      for n in numels]
            grads = [torch.zeros(n, dtype=torch.int16) for n in numels]
            ss, gg = shard_states(states, grads, spans)
            for sp, st, g in zip(spans, ss, gg):
                assert st.w.numel() == st.ecc.numel() == st.m_q.numel() == st.v_q.numel() == g.numel() == sp.elems
                assert st.m_scale.numel() == st.v_scale.numel() == sp.g1 - sp.g0
                # the views start where the span starts (storage offsets, in elements)
                assert st.w.storage_offset() == sp.e0 and st.m_scale.storage_offset() == sp.g0
        # in list order: (tensor, group) keys ascending, owners non-decreasing
        keys = sorted(flat_owner)
        assert keys == sorted(set(keys))                  # each group once
        assert [(t, g) for t, g, _ in keys] == [(ti, g) for ti, n in enumerate(numels)
                                                for g in range((n + 31) // 32)]
        owners = [r for _, _, r in keys]
        assert owners == sorted(owners)
        sizes = [owners.count(r) for r in range(world)]
        assert max(sizes) - min(sizes) <= 1

    check()

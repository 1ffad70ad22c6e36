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

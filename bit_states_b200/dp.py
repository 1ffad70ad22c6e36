"""Data-parallel sharded step: the exchange that brackets the compressed step
when several ranks train one model.

Every group of 32 elements is independent in the step, so the optimizer state
(ECC codes, momentum / variance codes and scales) is partitioned across ranks
and never communicated; only the 16-bit tensors cross ranks:

  1. reduce-scatter of the 16-bit gradients: each rank receives the reduced
     gradient of the groups it owns (2 B per parameter in);
  2. the fused step on the owned groups (one flat descriptor per bucket);
  3. all-gather of the updated 16-bit downcast weights x' (2 B per parameter
     out), so that every rank holds the whole x' for its next forward pass.

Layout: the parameter list is laid out flat with every tensor padded to a
whole number of groups (the padding is zero and stays zero), then cut into
buckets of ``bucket_groups`` groups (a multiple of the world size); rank r owns
the r-th equal slice of every bucket.  A bucket's slice is one contiguous
array of whole groups, so it is stepped as one flat tensor: the codes and
scales of the real elements equal those of stepping each tensor on its own
(zeros never raise a group's absolute maximum).

On CUDA the collectives run on a communication stream in one fixed order (all
reduce-scatters, then all all-gathers), ordered against the step of each
bucket on the compute stream by events: a bucket is stepped as soon as its
reduce-scatter lands and gathered as soon as its step ends, so the exchange
overlaps the steps bucket by bucket.  The collectives are torch.distributed's
(NCCL on GPUs, gloo on CPUs); the step itself is ``step_fn`` (by default the
library's fused kernel).
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, List, Optional, Sequence

GROUP = 32


def _round_up(n: int, a: int) -> int:
    return (n + a - 1) // a * a


@dataclass(frozen=True)
class Bucket:
    g0: int          # first group of the bucket in the flat layout
    groups: int      # groups in the bucket (a multiple of the world size)

    def shard(self, world: int, rank: int):
        """(first group, group count) of rank ``rank``'s slice."""
        per = self.groups // world
        return self.g0 + rank * per, per


class FlatLayout:
    """Group-aligned flat layout of a parameter list, cut into buckets."""

    def __init__(self, numels: Sequence[int], world: int, bucket_groups: int = 1 << 16):
        if world < 1:
            raise ValueError("world must be >= 1")
        self.numels = [int(n) for n in numels]
        self.world = world
        self.offsets: List[int] = []      # element offset of each tensor in the flat buffer
        off = 0
        for n in self.numels:
            self.offsets.append(off)
            off += _round_up(n, GROUP)
        total_groups = off // GROUP
        bg = max(world, _round_up(int(bucket_groups), world))
        self.buckets: List[Bucket] = []
        g = 0
        while g < total_groups:
            k = min(bg, _round_up(total_groups - g, world))
            self.buckets.append(Bucket(g, k))
            g += k
        self.groups = g                   # total groups including the padding of the last bucket
        self.numel = g * GROUP            # elements of every flat buffer

    def tensor_view(self, flat, i: int):
        """The real elements of tensor i in a flat buffer."""
        o = self.offsets[i]
        return flat[o:o + self.numels[i]]


class ShardedState:
    """One rank's compressed state: the whole x' (replicated) plus the ECC
    codes, momentum / variance codes and scales of the groups it owns."""

    def __init__(self, layout: FlatLayout, rank: int, device, adam: bool = True, ecc_bits: int = 8):
        import torch

        self.layout, self.rank, self.adam, self.ecc_bits = layout, rank, adam, ecc_bits
        W = layout.world
        owned = sum(b.groups // W for b in layout.buckets)
        edt = torch.int8 if ecc_bits == 8 else torch.int16
        self.w = torch.zeros(layout.numel, dtype=torch.int16, device=device)   # x', replicated
        self.ecc = torch.zeros(owned * GROUP, dtype=edt, device=device)
        self.m_q = torch.zeros(owned * GROUP, dtype=torch.int8, device=device)
        self.m_scale = torch.zeros(owned, dtype=torch.int16, device=device)
        self.v_q = torch.zeros(owned * GROUP, dtype=torch.uint8, device=device) if adam else None
        self.v_scale = torch.zeros(owned, dtype=torch.int16, device=device) if adam else None
        # per bucket: (flat element range of the owned slice, offset into the owned arrays)
        self.slices = []
        o = 0
        for b in layout.buckets:
            g0, k = b.shard(W, rank)
            self.slices.append((g0 * GROUP, (g0 + k) * GROUP, o))
            o += k

    def encode_from(self, x32_flat, fmt, group=None, w_dtype: str = "bf16"):
        """Initialise from f32 masters in the flat layout (every rank passes
        the same values): each rank encodes the groups it owns (downcast and
        ECC), then the downcast weights are all-gathered."""
        import torch
        import torch.distributed as dist

        from . import fo

        wflat = self.w.view({"bf16": torch.bfloat16, "fp16": torch.float16}[w_dtype])
        for bi, b in enumerate(self.layout.buckets):
            s0, s1, go = self.slices[bi]
            n, o = s1 - s0, go * GROUP
            fo.fo_encode_master(x32_flat[s0:s1], self.w[s0:s1], self.ecc[o:o + n], n, fmt)
            e0 = b.g0 * GROUP
            dist.all_gather_into_tensor(wflat[e0:e0 + b.groups * GROUP], wflat[s0:s1], group=group)

    def bucket_state(self, bi: int):
        """TensorState of this rank's slice of bucket bi (one flat tensor)."""
        from .fo import TensorState

        e0, e1, go = self.slices[bi]
        n, ng = e1 - e0, (e1 - e0) // GROUP
        o = go * GROUP
        sl = lambda t, a, k: None if t is None else t[a:a + k]
        return TensorState(self.w[e0:e1], self.ecc[o:o + n], self.m_q[o:o + n], self.m_scale[go:go + ng],
                           sl(self.v_q, o, n), sl(self.v_scale, go, ng))


def _descriptor_cache():
    """Descriptors of (state, grad) pairs built once: a bucket's slices do not
    move between steps, so each step reuses its ctypes descriptor."""
    from . import fo

    cache = {}

    def get(state, grad):
        key = (state.w.data_ptr(), state.ecc.data_ptr(), grad.data_ptr(), state.numel)
        d = cache.get(key)
        if d is None:
            d = cache[key] = fo.descriptors([state], [grad])
        return d

    return get


def _adamw_step_fn(fmt, hp):
    from . import fo

    desc = _descriptor_cache()

    def step(state, grad, t, stream):
        h = fo.fo_adamw_hparams(hp["lr"], hp["beta1"], hp["beta2"], hp["eps"], hp["weight_decay"], t)
        fo.fo_adamw_step(desc(state, grad), 1, fmt, h, stream)

    return step


def _sgdm_step_fn(fmt, hp):
    from . import fo

    desc = _descriptor_cache()

    def step(state, grad, t, stream):
        h = fo.fo_sgdm_hparams(hp["lr"], hp["momentum"], hp.get("dampening", 0.0), hp.get("weight_decay", 0.0),
                               int(bool(hp.get("nesterov", False))), t)
        fo.fo_sgdm_step(desc(state, grad), 1, fmt, h, stream)

    return step


class DataParallelStep:
    """Reduce-scatter -> fused step on the owned groups -> all-gather of x',
    bucket by bucket.

    ``step_fn(state, grad_shard, t, stream)`` steps one bucket slice in place
    (default: the library's fused step for ``optimizer``, "adamw" or "sgdm",
    with ``hparams``; SGD-momentum needs a state built with ``adam=False``).
    ``reduce_op`` is "sum" or "avg" (the average needs a backend that
    provides it, such as NCCL)."""

    def __init__(self, state: ShardedState, group=None, step_fn: Optional[Callable] = None,
                 fmt=None, hparams=None, reduce_op: str = "sum", grad_dtype: str = "bf16",
                 w_dtype: str = "bf16", optimizer: str = "adamw"):
        import torch
        import torch.distributed as dist

        self.state = state
        # collectives see the 16-bit patterns as their floating-point type: the
        # reduction adds gradients, the all-gather only moves bytes
        tdt = {"bf16": torch.bfloat16, "fp16": torch.float16}
        self.gdt, self.wdt = tdt[grad_dtype], tdt[w_dtype]
        self.group = group
        self.layout = state.layout
        if optimizer not in ("adamw", "sgdm"):
            raise ValueError("optimizer must be 'adamw' or 'sgdm'")
        if (optimizer == "adamw") != state.adam:
            raise ValueError("the state's variance arrays do not match the optimizer")
        if step_fn is None:
            from . import fo

            fmt = fmt or fo.make_format(w_dtype, grad_dtype, state.ecc_bits)
            step_fn = (_adamw_step_fn if optimizer == "adamw" else _sgdm_step_fn)(fmt, hparams)
        self.step_fn = step_fn
        self.op = {"sum": dist.ReduceOp.SUM, "avg": dist.ReduceOp.AVG}[reduce_op]
        dev = state.w.device
        self.cuda = dev.type == "cuda"
        self.comm = torch.cuda.Stream(device=dev) if self.cuda else None
        # this rank's reduced gradient, laid out like its owned state arrays
        self.gown = torch.zeros(state.m_q.numel(), dtype=torch.int16, device=dev)
        self._buckets = None

    def _parts(self):
        st, L = self.state, self.layout
        parts = []
        for bi, b in enumerate(L.buckets):
            e0 = b.g0 * GROUP
            s0, s1, go = st.slices[bi]
            parts.append((e0, e0 + b.groups * GROUP, s0, s1, go * GROUP, (s1 - s0)))
        return parts

    def exchange(self, grads_flat):
        """The collectives of one step without the step itself: every bucket's
        reduce-scatter into this rank's gradient shard, then every bucket's
        all-gather of x' (unchanged), on the communication stream.  Used to
        time the exchange alone; the state is left as it was."""
        import torch
        import torch.distributed as dist

        gflat = grads_flat.view(self.gdt)
        wflat = self.state.w.view(self.wdt)
        parts = self._parts()
        if not self.cuda:
            for e0, e1, s0, s1, o, n in parts:
                dist.reduce_scatter_tensor(self.gown[o:o + n].view(self.gdt), gflat[e0:e1], op=self.op,
                                           group=self.group)
                dist.all_gather_into_tensor(wflat[e0:e1], wflat[s0:s1].clone(), group=self.group)
            return
        cur = torch.cuda.current_stream()
        self.comm.wait_stream(cur)
        with torch.cuda.stream(self.comm):
            for e0, e1, s0, s1, o, n in parts:
                dist.reduce_scatter_tensor(self.gown[o:o + n].view(self.gdt), gflat[e0:e1], op=self.op,
                                           group=self.group)
            for e0, e1, s0, s1, o, n in parts:
                dist.all_gather_into_tensor(wflat[e0:e1], wflat[s0:s1], group=self.group)
        cur.wait_stream(self.comm)

    def _bucket(self, bi: int):
        """(state of this rank's slice of bucket bi, its gradient shard), views
        built once."""
        if self._buckets is None:
            self._buckets = [(self.state.bucket_state(i), self.gown[o:o + n])
                             for i, (e0, e1, s0, s1, o, n) in enumerate(self._parts())]
        return self._buckets[bi]

    def step_only(self, t: int, stream=None):
        """The fused step of every owned bucket slice on the gradient shard of
        the last exchange, without collectives (to time the steps alone)."""
        for bi in range(len(self.layout.buckets)):
            self.step_fn(*self._bucket(bi), t, stream)

    def step(self, grads_flat, t: int):
        """grads_flat: this rank's whole 16-bit gradient in the flat layout
        (int16 bit patterns, layout.numel elements, padding zero).

        Collectives go in one fixed order on one stream (every rank issues the
        same sequence): all reduce-scatters, then the all-gathers, each
        all-gather waiting for the step of its bucket; each bucket's step waits
        for its reduce-scatter.  The steps therefore overlap the remaining
        reduce-scatters and the earlier buckets' all-gathers."""
        import torch
        import torch.distributed as dist

        st = self.state
        gflat = grads_flat.view(self.gdt)
        wflat = st.w.view(self.wdt)
        parts = self._parts()
        if not self.cuda:
            for bi, (e0, e1, s0, s1, o, n) in enumerate(parts):
                dist.reduce_scatter_tensor(self.gown[o:o + n].view(self.gdt), gflat[e0:e1], op=self.op,
                                           group=self.group)
                self.step_fn(*self._bucket(bi), t, None)
                dist.all_gather_into_tensor(wflat[e0:e1], wflat[s0:s1].clone(), group=self.group)
            return
        cur = torch.cuda.current_stream()
        self.comm.wait_stream(cur)  # the gradients are complete
        rs_done, step_done = [], []
        with torch.cuda.stream(self.comm):
            for e0, e1, s0, s1, o, n in parts:
                dist.reduce_scatter_tensor(self.gown[o:o + n].view(self.gdt), gflat[e0:e1], op=self.op,
                                           group=self.group)
                ev = torch.cuda.Event()
                ev.record(self.comm)
                rs_done.append(ev)
        for bi, (e0, e1, s0, s1, o, n) in enumerate(parts):
            cur.wait_event(rs_done[bi])
            self.step_fn(*self._bucket(bi), t, cur)
            ev = torch.cuda.Event()
            ev.record(cur)
            step_done.append(ev)
        with torch.cuda.stream(self.comm):
            for bi, (e0, e1, s0, s1, o, n) in enumerate(parts):
                self.comm.wait_event(step_done[bi])
                # in place: this rank's slice already sits at its offset of the output
                dist.all_gather_into_tensor(wflat[e0:e1], wflat[s0:s1], group=self.group)
        cur.wait_stream(self.comm)

"""Partition of a parameter list across ranks in whole 32-element groups.

Every group of 32 consecutive elements of a tensor is independent in the
compressed step (its scales and codes depend on that group alone), so a
parameter list shards across data-parallel ranks with no exchange inside the
step: rank r steps the groups it owns, through ordinary descriptors that point
into the middle of each tensor at a group boundary (weights, ECC and codes at
element 32*g0, scales at entry g0).  Which rank owns what is computed here on
the host; the arrays themselves stay where the caller allocated them.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Sequence

GROUP = 32


@dataclass(frozen=True)
class Span:
    tensor: int       # index in the parameter list
    g0: int           # first group (inclusive)
    g1: int           # last group (exclusive)
    numel: int        # elements of the tensor

    @property
    def e0(self) -> int:
        return self.g0 * GROUP

    @property
    def e1(self) -> int:
        return min(self.g1 * GROUP, self.numel)

    @property
    def elems(self) -> int:
        return max(0, self.e1 - self.e0)


def shard_spans(numels: Sequence[int], world: int, rank: int) -> List[Span]:
    """Contiguous, balanced split of all groups of the list (in list order)
    into ``world`` parts; returns rank ``rank``'s part as per-tensor spans.
    Every group belongs to exactly one rank; a rank's part may cut tensors."""
    if world < 1 or not (0 <= rank < world):
        raise ValueError("bad world / rank")
    groups = [(int(n) + GROUP - 1) // GROUP for n in numels]
    total = sum(groups)
    lo = total * rank // world
    hi = total * (rank + 1) // world
    out: List[Span] = []
    base = 0
    for ti, (ng, n) in enumerate(zip(groups, numels)):
        a, b = max(lo, base), min(hi, base + ng)
        if a < b:
            out.append(Span(ti, a - base, b - base, int(n)))
        base += ng
    return out


def shard_states(states, grads, spans: Sequence[Span]):
    """Slice TensorState objects (torch views) to a rank's spans."""
    from .fo import TensorState

    out_s, out_g = [], []
    for sp in spans:
        st, g = states[sp.tensor], grads[sp.tensor]
        e0, e1, g0, g1 = sp.e0, sp.e1, sp.g0, min(sp.g1, (sp.numel + GROUP - 1) // GROUP)
        sl = lambda t, a, b: None if t is None else t[a:b]
        out_s.append(TensorState(st.w[e0:e1], st.ecc[e0:e1], st.m_q[e0:e1], st.m_scale[g0:g1],
                                 sl(st.v_q, e0, e1), sl(st.v_scale, g0, g1)))
        out_g.append(g[e0:e1])
    return out_s, out_g

"""Helpers of the GPU parity tests: build a workload's compressed state on the
device through the C ABI, run steps, and compute the oracle's expected bytes
for sampled groups from the same seeded inputs (never from the GPU)."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from bit_states_b200 import fo
from bit_states_b200.state import CompressedParams
from workloads import device as wdev

DT = {"bf16": 0, "fp16": 1}


def device_state(wl, dev="cuda"):
    P = CompressedParams([t.numel for t in wl.tensors], dev, adam=(wl.optimizer == "adamw"),
                         ecc_bits=wl.ecc_bits, w_dtype=wl.w_dtype)
    big = max(t.numel for t in wl.tensors)
    buf = torch.empty(big, dtype=torch.float32, device=dev)
    for ti, t in enumerate(wl.tensors):
        x = buf[:t.numel]
        wdev.master_f32(wl, ti, x)
        P.encode_from(ti, x)
    del buf
    return P


class GradArena:
    """One int16 arena holding every tensor's 16-bit gradient, laid out like
    the state arena (512-element aligned slices)."""

    def __init__(self, P: CompressedParams, dev="cuda"):
        self.P = P
        self.buf = torch.empty(P.total, dtype=torch.int16, device=dev)
        self.views = [self.buf[o:o + n] for o, n in zip(P.offsets, P.numels)]

    def fill(self, wl, step):
        for ti, v in enumerate(self.views):
            wdev.grad_16(wl, ti, step, v)


def hparams_adamw(wl, t):
    h = wl.hparams
    return fo.fo_adamw_hparams(h["lr"], h["beta1"], h["beta2"], h["eps"], h["weight_decay"], t)


def hparams_sgdm(wl, t):
    h = wl.hparams
    return fo.fo_sgdm_hparams(h["lr"], h["momentum"], h["dampening"], h["weight_decay"],
                              int(h["nesterov"]), t)


def fmt_of(wl):
    return fo.make_format(wl.w_dtype, wl.grad_dtype, wl.ecc_bits)


def step(wl, P, grads, t, order=None, stream=None):
    """One step of the whole list: a single multi-tensor call, or one call per
    tensor in ``order`` (gradient release)."""
    fmt = fmt_of(wl)
    if order is None:
        d = fo.descriptors(P.states, grads.views)
        if wl.optimizer == "adamw":
            fo.fo_adamw_step(d, len(P.states), fmt, hparams_adamw(wl, t), stream)
        else:
            fo.fo_sgdm_step(d, len(P.states), fmt, hparams_sgdm(wl, t), stream)
    else:
        for ti in order:
            d = fo.descriptors([P.states[ti]], [grads.views[ti]])
            if wl.optimizer == "adamw":
                fo.fo_adamw_step(d, 1, fmt, hparams_adamw(wl, t), stream)
            else:
                fo.fo_sgdm_step(d, 1, fmt, hparams_sgdm(wl, t), stream)


# ---- sampled oracle ---------------------------------------------------------

def sample_groups(n, k, rng):
    ng = (n + 31) // 32
    if ng <= k:
        return np.arange(ng)
    g = rng.choice(ng, size=k, replace=False)
    g = np.union1d(g, [0, ng - 1])          # always the first and the (maybe partial) last group
    return np.sort(g)


def group_elems(n, groups):
    g = np.asarray(groups, np.int64)
    idx = (32 * g[:, None] + np.arange(32, dtype=np.int64)[None, :]).ravel()
    return idx[idx < n]


class OracleSample:
    """The oracle's state for a set of groups of one tensor, stepped from
    the seeded inputs.  Full groups form one oracle array; a partial last
    group (if sampled) is stepped as its own array."""

    def __init__(self, wl, ti, groups, threads=1):
        self.wl, self.ti, self.threads = wl, ti, threads
        n = wl.tensors[ti].numel
        self.n = n
        self.groups = np.asarray(groups)
        full = self.groups[32 * self.groups + 32 <= n]
        tail = self.groups[32 * self.groups + 32 > n]
        self.parts = []
        for gs in (full, tail):
            if gs.size == 0:
                continue
            idx = group_elems(n, gs)
            x = wl.master_values(ti, idx)
            w, e = oracle.encode_master(x, DT[wl.w_dtype], wl.ecc_bits)
            st = oracle.State.zeros_like_master(w, e, adam=(wl.optimizer == "adamw"))
            self.parts.append((gs, idx, st))

    def step(self, t):
        for gs, idx, st in self.parts:
            g = self.wl.grad_bits(self.ti, t, idx)
            if self.wl.optimizer == "adamw":
                oracle.adamw_step(st, g, **self.wl.hparams, step=t, wdt=DT[self.wl.w_dtype],
                                  gdt=DT[self.wl.grad_dtype], ecc_bits=self.wl.ecc_bits,
                                  threads=self.threads)
            else:
                h = dict(self.wl.hparams)
                oracle.sgdm_step(st, g, lr=h["lr"], momentum=h["momentum"], dampening=h["dampening"],
                                 weight_decay=h["weight_decay"], nesterov=bool(h["nesterov"]), step=t,
                                 wdt=DT[self.wl.w_dtype], gdt=DT[self.wl.grad_dtype],
                                 ecc_bits=self.wl.ecc_bits, threads=self.threads)

    def expected(self):
        """dict field -> (element or group indices, expected values)"""
        out = {}
        for gs, idx, st in self.parts:
            for name, arr, ix in (("w", st.w, idx), ("ecc", st.ecc, idx), ("m_q", st.mq, idx),
                                  ("m_scale", st.ms, gs), ("v_q", st.vq, idx), ("v_scale", st.vs, gs)):
                if arr is None:
                    continue
                a, b = out.get(name, (np.zeros(0, np.int64), None))
                out[name] = (np.concatenate([a, ix]),
                             arr.view(np.uint8 if arr.itemsize == 1 else np.uint16) if b is None else
                             np.concatenate([b, arr.view(np.uint8 if arr.itemsize == 1 else np.uint16)]))
        return out


def gather_device(P, ti, exp):
    st = P.states[ti]
    got = {}
    for name, (ix, _) in exp.items():
        t = getattr(st, name)
        sel = t[torch.from_numpy(ix).to(t.device)].cpu().numpy()
        got[name] = sel.view(np.uint8 if sel.itemsize == 1 else np.uint16)
    return got


def mismatches(exp, got):
    return {k: int(np.count_nonzero(exp[k][1] != got[k])) for k in exp}


def to_np_bytes(t):
    a = t.cpu().numpy()
    return a.view(np.uint8 if a.itemsize == 1 else np.uint16)

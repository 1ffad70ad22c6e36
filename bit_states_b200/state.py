"""Compressed optimizer state of a parameter list, in device memory.

Buffers are allocated with torch (plumbing only) as one arena per stream of
bytes: downcast weights, ECC codes, momentum codes + scales, variance codes +
scales.  Each tensor's slice starts on a multiple of 512 elements (its
scales on a multiple of 16 groups), so every array of every tensor starts on
a 16-byte boundary, as the kernels' staged path needs.  All
arithmetic (encode, step, decode) runs in libfo's kernels.
"""
from __future__ import annotations

from typing import List, Sequence

from . import fo

ALIGN_ELEMS = 512


def _round_up(n: int, a: int) -> int:
    return (n + a - 1) // a * a


class CompressedParams:
    """Arena of the compressed state of ``numels`` parameters."""

    def __init__(self, numels: Sequence[int], device, adam: bool = True, ecc_bits: int = 8,
                 w_dtype: str = "bf16"):
        import torch

        self.numels = [int(n) for n in numels]
        self.adam = adam
        self.ecc_bits = ecc_bits
        self.w_dtype = w_dtype
        self.offsets: List[int] = []
        self.goffsets: List[int] = []
        off = goff = 0
        for n in self.numels:
            self.offsets.append(off)
            self.goffsets.append(goff)
            off += _round_up(max(n, 1), ALIGN_ELEMS)
            goff += _round_up((n + 31) // 32, 16)
        self.total = off
        self.gtotal = goff
        edt = torch.int8 if ecc_bits == 8 else torch.int16
        self.w = torch.zeros(self.total, dtype=torch.int16, device=device)
        self.ecc = torch.zeros(self.total, dtype=edt, device=device)
        self.m_q = torch.zeros(self.total, dtype=torch.int8, device=device)
        self.m_scale = torch.zeros(self.gtotal, dtype=torch.int16, device=device)
        if adam:
            self.v_q = torch.zeros(self.total, dtype=torch.uint8, device=device)
            self.v_scale = torch.zeros(self.gtotal, dtype=torch.int16, device=device)
        else:
            self.v_q = self.v_scale = None
        self.states = [self._state(i) for i in range(len(self.numels))]

    def _state(self, i: int) -> fo.TensorState:
        o, g, n = self.offsets[i], self.goffsets[i], self.numels[i]
        ng = (n + 31) // 32
        sl = lambda t, a, k: None if t is None else t[a:a + k]
        return fo.TensorState(self.w[o:o + n], self.ecc[o:o + n], self.m_q[o:o + n],
                              self.m_scale[g:g + ng], sl(self.v_q, o, n), sl(self.v_scale, g, ng))

    @property
    def format_bits(self) -> int:
        return self.ecc_bits

    def nbytes(self) -> int:
        t = self.w.nbytes + self.ecc.nbytes + self.m_q.nbytes + self.m_scale.nbytes
        if self.adam:
            t += self.v_q.nbytes + self.v_scale.nbytes
        return t

    def state_dict(self) -> dict:
        """Checkpoint: the compressed arrays (the masters are their downcast +
        ECC, so nothing is lost) and the layout they were allocated with."""
        d = {"numels": list(self.numels), "adam": self.adam, "ecc_bits": self.ecc_bits, "w_dtype": self.w_dtype,
             "w": self.w, "ecc": self.ecc, "m_q": self.m_q, "m_scale": self.m_scale}
        if self.adam:
            d["v_q"], d["v_scale"] = self.v_q, self.v_scale
        return d

    def load_state_dict(self, d: dict) -> None:
        """Resume from state_dict(): the same parameter list and format."""
        if (list(d["numels"]) != self.numels or bool(d["adam"]) != self.adam or int(d["ecc_bits"]) != self.ecc_bits
                or d["w_dtype"] != self.w_dtype):
            raise ValueError("checkpoint was taken with another parameter list or format")
        for k in ("w", "ecc", "m_q", "m_scale") + (("v_q", "v_scale") if self.adam else ()):
            getattr(self, k).copy_(d[k])

    def encode_from(self, i: int, x32, stream=None):
        """Split f32 masters of tensor i into downcast + ECC (device kernel)."""
        st = self.states[i]
        fmt = fo.make_format(self.w_dtype, "bf16", self.ecc_bits)
        fo.fo_encode_master(x32, st.w, st.ecc, st.numel, fmt, stream)

    def decode_to(self, i: int, out32, stream=None):
        st = self.states[i]
        fmt = fo.make_format(self.w_dtype, "bf16", self.ecc_bits)
        fo.fo_decode_master(st.w, st.ecc, out32, st.numel, fmt, stream)


class CompressedAdamW:
    """AdamW over a parameter list with bf16/fp16 + ECC masters and 8-bit
    companded states; ``step`` is one fused kernel launch for the whole list
    (or one per call when used for gradient release).  A checkpoint is the
    parameters' state_dict() plus this optimizer's step count ``t``."""

    def __init__(self, params: CompressedParams, lr=1e-3, betas=(0.9, 0.999), eps=1e-8,
                 weight_decay=0.01, grad_dtype="bf16"):
        assert params.adam
        self.p = params
        self.hp = dict(lr=lr, beta1=betas[0], beta2=betas[1], eps=eps, weight_decay=weight_decay)
        self.t = 0
        self.fmt = fo.make_format(params.w_dtype, grad_dtype, params.ecc_bits)

    def hparams(self, t: int) -> fo.fo_adamw_hparams:
        h = self.hp
        return fo.fo_adamw_hparams(h["lr"], h["beta1"], h["beta2"], h["eps"], h["weight_decay"], t)

    def step(self, grads, stream=None):
        self.t += 1
        descs = fo.descriptors(self.p.states, grads)
        fo.fo_adamw_step(descs, len(self.p.states), self.fmt, self.hparams(self.t), stream)

    def start_release(self) -> int:
        """Gradient release: begin one optimizer step whose tensors are then
        stepped one by one with step_tensor (all with this step count)."""
        self.t += 1
        return self.t

    def step_tensor(self, i: int, grad, t: int = None, stream=None):
        """Gradient release: step tensor i alone (its gradient may be freed
        once the work on the stream has finished), with step count t (by
        default the one start_release began)."""
        if t is None:
            if self.t < 1:
                raise ValueError("call start_release() before step_tensor()")
            t = self.t
        descs = fo.descriptors([self.p.states[i]], [grad])
        fo.fo_adamw_step(descs, 1, self.fmt, self.hparams(t), stream)

    def state_dict(self) -> dict:
        """The optimizer's part of a checkpoint: the step count (bias
        corrections depend on it) and the hyper-parameters; the compressed
        arrays are CompressedParams.state_dict()."""
        return {"t": self.t, "hparams": dict(self.hp)}

    def load_state_dict(self, d: dict) -> None:
        self.t = int(d["t"])
        self.hp.update(d["hparams"])


class CompressedSGDM:
    """SGD with momentum over a parameter list with fp16/bf16 + ECC masters and
    an 8-bit companded momentum; ``step`` is one fused kernel launch."""

    def __init__(self, params: CompressedParams, lr=0.1, momentum=0.9, dampening=0.0,
                 weight_decay=0.0, nesterov=False, grad_dtype="fp16"):
        self.p = params
        self.hp = dict(lr=lr, momentum=momentum, dampening=dampening, weight_decay=weight_decay,
                       nesterov=int(bool(nesterov)))
        self.t = 0
        self.fmt = fo.make_format(params.w_dtype, grad_dtype, params.ecc_bits)

    def hparams(self, t: int) -> fo.fo_sgdm_hparams:
        h = self.hp
        return fo.fo_sgdm_hparams(h["lr"], h["momentum"], h["dampening"], h["weight_decay"],
                                  h["nesterov"], t)

    def step(self, grads, stream=None):
        self.t += 1
        descs = fo.descriptors(self.p.states, grads)
        fo.fo_sgdm_step(descs, len(self.p.states), self.fmt, self.hparams(self.t), stream)

    def state_dict(self) -> dict:
        """The optimizer's part of a checkpoint: the step count (the first
        step copies the gradient into the momentum) and the hyper-parameters."""
        return {"t": self.t, "hparams": dict(self.hp)}

    def load_state_dict(self, d: dict) -> None:
        self.t = int(d["t"])
        self.hp.update(d["hparams"])

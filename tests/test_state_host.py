"""Host logic of the torch-side helpers (no GPU): the arena layout that the
kernels' staged path relies on (every array of every tensor on a 16-byte
boundary) and the argument marshalling of CompressedAdamW / CompressedSGDM
(descriptors, format, hyper-parameters, step count).  The library's entry
points are replaced by recorders; CPU tensors stand in for device memory."""
import pytest
import torch

from bit_states_b200 import fo
from bit_states_b200.state import CompressedAdamW, CompressedParams, CompressedSGDM

NUMELS = [1, 31, 33, 511, 513, 768, 1000, 4097, 65537]


@pytest.mark.parametrize("adam,ecc_bits", [(True, 8), (True, 16), (False, 8)])
def test_arena_arrays_are_16_byte_aligned_and_disjoint(adam, ecc_bits):
    P = CompressedParams(NUMELS, "cpu", adam=adam, ecc_bits=ecc_bits)
    arrays = ["w", "ecc", "m_q", "m_scale"] + (["v_q", "v_scale"] if adam else [])
    for name in arrays:
        spans = []
        for st, n in zip(P.states, NUMELS):
            a = getattr(st, name)
            k = n if name in ("w", "ecc", "m_q", "v_q") else (n + 31) // 32
            assert a.numel() == k
            assert a.data_ptr() % 16 == 0, (name, n)
            spans.append((a.data_ptr(), a.data_ptr() + a.numel() * a.element_size()))
        spans.sort()
        assert all(e0 <= s1 for (_, e0), (s1, _) in zip(spans, spans[1:])), name
    if not adam:
        assert all(st.v_q is None and st.v_scale is None for st in P.states)
    per = 2 + ecc_bits // 8 + 1 + (1 if adam else 0)
    assert P.nbytes() == P.total * per + P.gtotal * 2 * (2 if adam else 1)


class _Recorder:
    def __init__(self):
        self.calls = []

    def __call__(self, descs, n, fmt, h, stream=None):
        self.calls.append(([descs[i] for i in range(n)], n, (fmt.w_dtype, fmt.grad_dtype, fmt.ecc_bits),
                           {f: getattr(h, f) for f, _ in h._fields_}, stream))


def _grads(P, dtype=torch.int16):
    return [torch.zeros(n, dtype=dtype) for n in P.numels]


def test_adamw_wrapper_marshalling(monkeypatch):
    rec = _Recorder()
    monkeypatch.setattr(fo, "fo_adamw_step", rec)
    P = CompressedParams(NUMELS, "cpu", adam=True, ecc_bits=8, w_dtype="fp16")
    opt = CompressedAdamW(P, lr=3e-4, betas=(0.8, 0.95), eps=1e-6, weight_decay=0.1, grad_dtype="bf16")
    g = _grads(P)
    opt.step(g)
    opt.step(g)
    opt.step_tensor(4, g[4], t=7)
    assert len(rec.calls) == 3
    for k, (descs, n, fmt, h, _) in enumerate(rec.calls[:2]):
        assert n == len(NUMELS)
        assert fmt == (1, 0, 8)                       # fp16 weights, bf16 gradients, 8-bit ECC
        assert h == dict(lr=3e-4, beta1=0.8, beta2=0.95, eps=1e-6, weight_decay=0.1, step=k + 1)
        for d, st, gi in zip(descs, P.states, g):
            assert (d.w, d.ecc, d.grad, d.m_q, d.m_scale, d.v_q, d.v_scale, d.numel) == (
                st.w.data_ptr(), st.ecc.data_ptr(), gi.data_ptr(), st.m_q.data_ptr(), st.m_scale.data_ptr(),
                st.v_q.data_ptr(), st.v_scale.data_ptr(), st.numel)
    descs, n, _, h, _ = rec.calls[2]
    assert n == 1 and h["step"] == 7 and descs[0].numel == NUMELS[4] and descs[0].w == P.states[4].w.data_ptr()
    assert opt.t == 2


def test_sgdm_wrapper_marshalling(monkeypatch):
    rec = _Recorder()
    monkeypatch.setattr(fo, "fo_sgdm_step", rec)
    P = CompressedParams(NUMELS, "cpu", adam=False, ecc_bits=8, w_dtype="fp16")
    opt = CompressedSGDM(P, lr=0.05, momentum=0.9, dampening=0.1, weight_decay=1e-4, nesterov=True)
    opt.step(_grads(P))
    descs, n, fmt, h, _ = rec.calls[0]
    assert n == len(NUMELS) and fmt == (1, 1, 8)
    assert h == dict(lr=0.05, momentum=0.9, dampening=0.1, weight_decay=1e-4, nesterov=1, step=1)
    assert all(d.v_q is None and d.v_scale is None for d in descs)   # NULL: SGD-momentum has no variance


def test_adamw_wrapper_needs_variance_arrays():
    P = CompressedParams(NUMELS, "cpu", adam=False)
    with pytest.raises(AssertionError):
        CompressedAdamW(P)

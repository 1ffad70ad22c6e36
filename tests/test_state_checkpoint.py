"""Checkpoint / resume of the compressed state (host logic, CPU tensors; no
kernel runs): state_dict() captures every compressed array and the layout,
load_state_dict() restores them byte for byte into a fresh arena and refuses a
checkpoint of another parameter list or format."""
import io

import pytest
import torch

from bit_states_b200.state import CompressedParams


def _filled(numels, **kw):
    P = CompressedParams(numels, "cpu", **kw)
    g = torch.Generator().manual_seed(3)
    for k in ("w", "ecc", "m_q", "m_scale", "v_q", "v_scale"):
        t = getattr(P, k)
        if t is not None:
            t.copy_(torch.randint(-100, 100, t.shape, generator=g).to(t.dtype))
    return P


@pytest.mark.parametrize("adam,ecc_bits", [(True, 8), (True, 16), (False, 8)])
def test_round_trip_through_torch_save(adam, ecc_bits):
    numels = [1, 33, 4096, 1000, 70000]
    P = _filled(numels, adam=adam, ecc_bits=ecc_bits)
    buf = io.BytesIO()
    torch.save(P.state_dict(), buf)
    buf.seek(0)
    Q = CompressedParams(numels, "cpu", adam=adam, ecc_bits=ecc_bits)
    Q.load_state_dict(torch.load(buf))
    for k in ("w", "ecc", "m_q", "m_scale") + (("v_q", "v_scale") if adam else ()):
        assert torch.equal(getattr(P, k), getattr(Q, k)), k
    # per-tensor views see the restored bytes
    for a, b in zip(P.states, Q.states):
        assert torch.equal(a.w, b.w) and torch.equal(a.m_scale, b.m_scale)


def test_refuses_another_layout():
    P = _filled([10, 20])
    with pytest.raises(ValueError):
        CompressedParams([10, 21], "cpu").load_state_dict(P.state_dict())
    with pytest.raises(ValueError):
        CompressedParams([10, 20], "cpu", ecc_bits=16).load_state_dict(P.state_dict())

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


def test_optimizer_step_count_and_hyperparameters_checkpoint():
    """The optimizers' part of a checkpoint is the step count t (AdamW's bias
    corrections and SGD's first-step rule depend on it) and the
    hyper-parameters; resuming restores both."""
    from bit_states_b200.state import CompressedAdamW, CompressedSGDM

    P = CompressedParams([100, 33], "cpu")
    opt = CompressedAdamW(P, lr=3e-4, betas=(0.9, 0.95), weight_decay=0.1)
    opt.t = 17
    d = opt.state_dict()
    buf = io.BytesIO()
    torch.save(d, buf)
    buf.seek(0)
    fresh = CompressedAdamW(P)
    fresh.load_state_dict(torch.load(buf))
    assert fresh.t == 17 and fresh.hp == opt.hp
    h = fresh.hparams(fresh.t + 1)
    assert h.step == 18 and abs(h.beta2 - 0.95) < 1e-15 and abs(h.lr - 3e-4) < 1e-15
    S = CompressedParams([64], "cpu", adam=False, w_dtype="fp16")
    sgd = CompressedSGDM(S, lr=0.05, momentum=0.8, nesterov=True)
    sgd.t = 3
    s2 = CompressedSGDM(S)
    s2.load_state_dict(sgd.state_dict())
    assert s2.t == 3 and s2.hp == sgd.hp


def test_release_step_count_is_explicit():
    """Gradient release: start_release() advances the step count once per
    iteration and every per-tensor call of that iteration uses it; a
    per-tensor call before any start_release() is refused."""
    from bit_states_b200.state import CompressedAdamW

    P = CompressedParams([10], "cpu")
    opt = CompressedAdamW(P)
    with pytest.raises(ValueError):
        opt.step_tensor(0, torch.zeros(10, dtype=torch.int16))
    assert opt.start_release() == 1 and opt.start_release() == 2 and opt.t == 2

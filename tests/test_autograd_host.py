"""The autograd wrapper's plumbing on the CPU: the library calls are replaced by fakes that record
what they receive and write recognisable values, so the test checks which tensors reach the kernels
(the forward's output and log-sum-exp reach the backward, tau as a float) and that each gradient
comes back on the argument it belongs to (and only when asked for)."""
import torch

from learned_token_pruning_tg_b200 import autograd as ag
from learned_token_pruning_tg_b200 import tokengate as tg


def install_fakes(monkeypatch, calls):
    monkeypatch.setattr(tg, "new_workspace", lambda *a, **k: torch.zeros(16, dtype=torch.uint8))

    def fwd(q, k, v, out, ws, s_kept=None, gain=None, tau=1.0, lse=None, stream=None):
        calls["fwd"] = dict(tau=tau, s=s_kept, g=gain)
        out.copy_(q)
        lse.fill_(7.0)
        return out

    def bwd(q, k, v, out, dout, lse, dq, dk, dv, ws, s_kept=None, gain=None, tau=1.0, ds=None, dg=None, dtau=None,
            stream=None):
        calls["bwd"] = dict(out=out.clone(), dout=dout.clone(), lse=lse.clone(), tau=tau, ds=ds, dg=dg, dtau=dtau)
        dq.fill_(1.0)
        dk.fill_(2.0)
        dv.fill_(3.0)
        for t, val in ((ds, 4.0), (dg, 5.0), (dtau, 6.0)):
            if t is not None:
                t.fill_(val)
        return dq, dk, dv

    monkeypatch.setattr(tg, "tg_gated_attention", fwd)
    monkeypatch.setattr(tg, "tg_gated_attention_backward", bwd)


def inputs(K=5, Hq=4, Hkv=2, d_h=64):
    g = torch.Generator().manual_seed(0)
    q = torch.randn(K, Hq, d_h, generator=g).to(torch.bfloat16).requires_grad_()
    k = torch.randn(K, Hkv, d_h, generator=g).to(torch.bfloat16).requires_grad_()
    v = torch.randn(K, Hkv, d_h, generator=g).to(torch.bfloat16).requires_grad_()
    s = torch.randn(K, generator=g).requires_grad_()
    gain = torch.rand(Hq, generator=g).requires_grad_()
    return q, k, v, s, gain


def test_every_gradient_lands_on_its_argument(monkeypatch):
    calls = {}
    install_fakes(monkeypatch, calls)
    q, k, v, s, gain = inputs()
    tau = torch.tensor(1.25, requires_grad=True)
    out = ag.gated_attention(q, k, v, s, gain, tau)
    assert torch.equal(out, q.detach())
    (out.float() * 2.0).sum().backward()
    assert calls["fwd"]["tau"] == 1.25 and calls["bwd"]["tau"] == 1.25
    assert torch.equal(calls["bwd"]["out"], q.detach()) and torch.all(calls["bwd"]["lse"] == 7.0)
    assert torch.all(calls["bwd"]["dout"] == 2.0) and calls["bwd"]["dout"].dtype == torch.bfloat16
    for t, val in ((q, 1.0), (k, 2.0), (v, 3.0), (s, 4.0), (gain, 5.0)):
        assert torch.all(t.grad == val)
    assert tau.grad.shape == () and tau.grad.item() == 6.0


def test_gradients_only_when_asked(monkeypatch):
    calls = {}
    install_fakes(monkeypatch, calls)
    q, k, v, s, gain = inputs()
    s.requires_grad_(False)
    out = ag.gated_attention(q, k, v, s, gain, 0.9)      # tau a plain float: no gradient for it
    out.float().sum().backward()
    assert calls["bwd"]["ds"] is None and calls["bwd"]["dtau"] is None and calls["bwd"]["dg"] is not None
    assert s.grad is None and torch.all(gain.grad == 5.0)
    q2, k2, v2, _, _ = inputs()
    out = ag.gated_attention(q2, k2, v2)                   # no bias at all
    out.float().sum().backward()
    assert calls["fwd"]["s"] is None and calls["fwd"]["g"] is None
    assert torch.all(q2.grad == 1.0)


def test_tau_gradient_takes_tau_shape_and_device(monkeypatch):
    calls = {}
    install_fakes(monkeypatch, calls)
    q, k, v, s, gain = inputs()
    tau = torch.tensor([1.1], requires_grad=True)            # one element, shape [1]
    ag.gated_attention(q, k, v, s, gain, tau).float().sum().backward()
    assert tau.grad.shape == (1,) and tau.grad.item() == 6.0


def test_backward_limits_fail_in_the_forward(monkeypatch):
    import pytest
    calls = {}
    install_fakes(monkeypatch, calls)
    g = torch.Generator().manual_seed(1)
    q = torch.randn(5, 16, 64, generator=g).to(torch.bfloat16).requires_grad_()
    k = torch.randn(5, 1, 64, generator=g).to(torch.bfloat16).requires_grad_()   # Hq / Hkv = 16 > 8
    with pytest.raises(ValueError, match="Hq / Hkv"):
        ag.gated_attention(q, k, k.detach().clone())
    q96 = torch.randn(5, 4, 96, generator=g).to(torch.bfloat16).requires_grad_()
    k96 = torch.randn(5, 2, 96, generator=g).to(torch.bfloat16)
    with pytest.raises(ValueError, match="d_h"):
        ag.gated_attention(q96, k96, k96)
    # without a graph to build, the forward alone has the forward's own limits
    out = ag.gated_attention(q.detach(), k.detach(), k.detach())
    assert "fwd" in calls and out.shape == q.shape


def test_status_check_raises_on_a_set_bit(monkeypatch):
    import pytest
    calls = {}
    install_fakes(monkeypatch, calls)
    monkeypatch.setattr(tg, "tg_device_status", lambda ws, stream=None: tg.TG_STATUS_ATTENTION_TIMEOUT)
    q, k, v, s, gain = inputs()
    with pytest.raises(tg.TokenGateError):
        ag.gated_attention(q, k, v, s, gain, 1.0, check_status=True)
    monkeypatch.setattr(tg, "tg_device_status", lambda ws, stream=None: 0)
    ag.gated_attention(q, k, v, s, gain, 1.0, check_status=True).float().sum().backward()
    assert torch.all(q.grad == 1.0)

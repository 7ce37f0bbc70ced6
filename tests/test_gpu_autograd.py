"""The differentiable op (learned_token_pruning_tg_b200.autograd.gated_attention) on the GPU: its
gradients are the direct backward call's, bit for bit (same kernels, same inputs), and therefore
match the oracle's backward within the backward's tolerance.

The wrapper's plumbing is also checked on the CPU with fake kernels (tests/test_autograd_host.py).
"""
import numpy as np
import pytest
import torch

from learned_token_pruning_tg_b200 import autograd as ag
from learned_token_pruning_tg_b200 import synth
from tests.test_gpu_attention_backward import compare, run_gpu, want_grads

pytestmark = pytest.mark.gpu


def test_autograd_equals_direct_backward_and_oracle():
    d = synth.qkv(333, 8, 4, 128, seed=41)
    dout = synth.grad_out(333, 8, 128, seed=42)
    q, k, v = (t.cuda().requires_grad_() for t in (d.q, d.k, d.v))
    s, g = d.s.cuda().requires_grad_(), d.gain.cuda().requires_grad_()
    tau = torch.tensor(d.tau, device="cuda", requires_grad=True)
    out = ag.gated_attention(q, k, v, s, g, tau)
    out.backward(dout.cuda())
    got = {"dq": q.grad.float().cpu().numpy(), "dk": k.grad.float().cpu().numpy(), "dv": v.grad.float().cpu().numpy(),
           "ds": s.grad.cpu().numpy(), "dg": g.grad.cpu().numpy(), "dtau": float(tau.grad.item())}
    direct = run_gpu(d, dout)
    for key in ("dq", "dk", "dv", "ds", "dg"):
        assert np.array_equal(got[key], direct[key]), key
    compare(got, want_grads(d, dout))

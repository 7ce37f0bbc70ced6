"""GPU parity of tg_gated_attention_backward against the oracle's backward.

The GPU backward is called the way training calls it: after the GPU forward,
with that forward's bf16 output and log-sum-exp.  The oracle runs on the same
bf16 inputs (exact fp32 widenings) and computes everything in fp64 from the
definition, including the forward it needs.

Tolerance (derived from the kernels' arithmetic): the products are exact bf16 x
bf16 with fp32 accumulation; P and dS are rounded to bf16 (relative error
2^-9 per element) before the dV, dK and dQ products, D = dO . O uses the
forward's bf16 O (relative 2^-9), and dq, dk, dv are returned in bf16 (half
an ulp, 2^-9 of the value).  Each gradient is a sum over up to K terms of both
signs, so an element's error is bounded by 2^-9 times the sum of the absolute
terms rather than by its own size; with random-sign terms the sum of absolute
values stays within ~8x the largest output, so the tests hold every
tensor to max |gpu - oracle| <= 2^-9 * 8 ~= 1.6e-2 of its largest magnitude,
and the scalar / fp32 outputs (ds, dg, dtau, which are summed in fp32 from
unrounded dS) to 1e-2 relative to their own scale.
"""
import numpy as np
import pytest
import torch

import oracle
from learned_token_pruning_tg_b200 import synth
from learned_token_pruning_tg_b200 import tokengate as tg
from tests import oracle_pool
from tests.guards import guarded

pytestmark = pytest.mark.gpu

TOL = 2.0 ** -9 * 8      # of each tensor's largest magnitude


def run_gpu(d, dout, use_bias=True):
    """Forward then backward on the GPU; returns numpy copies of every gradient."""
    K, Hq, d_h = d.q.shape
    Hkv = d.k.shape[1]
    q, k, v = d.q.cuda(), d.k.cuda(), d.v.cuda()
    s = d.s.cuda() if use_bias else None
    g = d.gain.cuda() if use_bias else None
    ws_f = tg.new_workspace(K, Hkv * d_h, op=tg.TG_OP_ATTENTION)
    out = torch.empty(K, Hq, d_h, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(Hq, K, dtype=torch.float32, device="cuda")
    tg.tg_gated_attention(q, k, v, out, ws_f, s_kept=s, gain=g, tau=d.tau, lse=lse)
    ws = tg.new_workspace(K, Hq, Hkv, op=tg.TG_OP_ATTENTION_BACKWARD)
    dq, cq = guarded((K, Hq, d_h), torch.bfloat16)
    dk, ck = guarded((K, Hkv, d_h), torch.bfloat16)
    dv, cv = guarded((K, Hkv, d_h), torch.bfloat16)
    ds, cs = guarded((K,), torch.float32)
    dg, cg = guarded((Hq,), torch.float32)
    dtau, ct = guarded((1,), torch.float32)
    for t in (dq, dk, dv, ds, dg, dtau):
        t.fill_(float("nan"))    # every element must be written
    tg.tg_gated_attention_backward(q, k, v, out, dout.cuda(), lse, dq, dk, dv, ws, s_kept=s, gain=g, tau=d.tau,
                                   ds=ds, dg=dg, dtau=dtau)
    torch.cuda.synchronize()
    for c in (cq, ck, cv, cs, cg, ct):
        c()
    assert tg.tg_device_status(ws) == 0 and tg.tg_device_status(ws_f) == 0
    return {"dq": dq.float().cpu().numpy(), "dk": dk.float().cpu().numpy(), "dv": dv.float().cpu().numpy(),
            "ds": ds.cpu().numpy(), "dg": dg.cpu().numpy(), "dtau": float(dtau.item())}


def want_grads(d, dout, use_bias=True, pool=False):
    q, k, v, do = (t.float().numpy() for t in (d.q, d.k, d.v, dout))
    s = d.s.numpy() if use_bias else None
    g = d.gain.numpy() if use_bias else None
    if pool:
        return oracle_pool.gated_attention_backward(q, k, v, do, s=s, g=g, tau=d.tau)
    return oracle.gated_attention_backward(q, k, v, do, s=s, g=g, tau=d.tau)


def compare(got, want, report=None):
    # each error is relative to the tensor's own largest magnitude, floored at 1e-3 of the largest
    # gradient element overall (a gradient that vanishes mathematically -- every one but dv at K = 1 --
    # is then held to rounding noise on that scale)
    floor = 1e-3 * max(float(np.max(np.abs(want[key]))) for key in ("dq", "dk", "dv"))
    errs = {}
    for key in ("dq", "dk", "dv", "ds", "dg"):
        a, b = got[key], want[key]
        assert np.all(np.isfinite(a)), key
        scale = max(float(np.max(np.abs(b))), floor)
        errs[key] = float(np.max(np.abs(a - b))) / scale
    errs["dtau"] = abs(got["dtau"] - want["dtau"]) / max(abs(want["dtau"]), floor)
    if report is not None:
        report.update(errs)
    for key in ("dq", "dk", "dv"):
        assert errs[key] <= TOL, (key, errs)
    for key in ("ds", "dg", "dtau"):
        assert errs[key] <= 1e-2, (key, errs)
    return errs


@pytest.mark.parametrize("K,Hq,Hkv,d_h", [
    (1, 2, 1, 128),          # a single token: every gradient but dv vanishes
    (200, 4, 2, 64),         # two tiles, ragged tail
    (333, 8, 8, 128),        # G = 1, three tiles
    (300, 16, 2, 64),        # G = 8
    (600, 8, 2, 128),        # G = 4, five tiles
])
def test_backward_parity_small(K, Hq, Hkv, d_h):
    d = synth.qkv(K, Hq, Hkv, d_h, seed=K + Hq + d_h)
    dout = synth.grad_out(K, Hq, d_h, seed=K + 1)
    got = run_gpu(d, dout)
    compare(got, want_grads(d, dout))


def test_backward_without_bias():
    d = synth.qkv(400, 8, 4, 128, seed=17)
    dout = synth.grad_out(400, 8, 128, seed=18)
    got = run_gpu(d, dout, use_bias=False)
    assert np.all(got["ds"] == 0.0) and np.all(got["dg"] == 0.0)
    want = want_grads(d, dout, use_bias=False)
    compare(got, want)


def test_backward_repeatable_bit_exact():
    d = synth.qkv(700, 8, 4, 128, seed=21)
    dout = synth.grad_out(700, 8, 128, seed=22)
    a = run_gpu(d, dout)
    for _ in range(2):
        b = run_gpu(d, dout)
        for key in ("dq", "dk", "dv", "ds", "dg"):
            assert np.array_equal(a[key], b[key]), key
        assert a["dtau"] == b["dtau"]


def test_backward_full_workload_128k():
    """The 128k workload's attention above the gate: K = 4608 kept tokens (4096 document tokens and
    the 512-token question), Qwen3-1.7B heads, 3% heavy rows; every gradient element checked."""
    d = synth.qkv(4608, 16, 8, 128, seed=4608, heavy_frac=0.03)
    dout = synth.grad_out(4608, 16, 128, seed=4609)
    got = run_gpu(d, dout)
    errs = compare(got, want_grads(d, dout, pool=True), report={})
    print("backward 128k normalised errors:", errs)

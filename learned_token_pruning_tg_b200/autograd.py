"""Token-gated attention as a differentiable torch op (the gradient path the gate trains through).

TokenGate gives each kept token's score a bias on the attention logits above the gate precisely so
that the scorer gets gradients, together with a learned per-head gain and temperature
(aiproducthub.cn article, paragraph 事件详情; aisight.pl article, section Jak to działa; chathome.org
article, section トークンゲート付きアテンションとは).  `gated_attention(q, k, v, s_kept, gain, tau)`
runs tg_gated_attention forward and tg_gated_attention_backward for the gradients of q, k, v, the
kept scores, the gains and the temperature.  Argument marshalling only: both directions are the
library's kernels; torch allocates the outputs and the workspaces.

The kernels' waits are bounded: a wait that runs out leaves a bit in the call's status word instead
of hanging.  With check_status=True (or TOKENGATE_CHECK_STATUS=1 in the environment) each call reads
that word back -- one synchronisation per call -- and raises on a set bit; otherwise a timeout shows
only as wrong values.
"""
from __future__ import annotations

import os
from typing import Optional, Union

import torch

from . import tokengate as tg

# limits of tg_gated_attention_backward, checked when the forward records a graph
_BWD_MAX_GROUP = 8
_BWD_HEAD_DIMS = (64, 128)


def _check_backward_limits(q, k, v):
    K, Hq, d_h = q.shape
    Hkv = k.shape[1]
    if d_h not in _BWD_HEAD_DIMS:
        raise ValueError(f"the backward supports d_h in {_BWD_HEAD_DIMS}, got {d_h}")
    if Hq % Hkv or Hq // Hkv > _BWD_MAX_GROUP:
        raise ValueError(f"the backward supports Hq / Hkv <= {_BWD_MAX_GROUP}, got {Hq} / {Hkv}")
    for t, name in ((q, "q"), (k, "k"), (v, "v")):
        if t.dim() != 3 or t.stride(2) != 1 or t.stride(1) != d_h or (K > 1 and t.stride(0) % 8):
            raise ValueError(f"{name}: heads must be dense and the token stride a multiple of 8")


def _raise_on_status(ws, what: str):
    bits = tg.tg_device_status(ws)
    if bits:
        raise tg.TokenGateError(what, tg.TG_ERR_TIMEOUT if bits & 0x3F else tg.TG_ERR_RANGE)


class GatedAttentionFunction(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, s_kept, gain, tau, check_status=False):
        K, Hq, d_h = q.shape
        Hkv = k.shape[1]
        if any(ctx.needs_input_grad[:6]):
            _check_backward_limits(q, k, v)   # fail here, not at .backward() after the graph is built
        tau_f = float(tau)
        out = torch.empty(K, Hq, d_h, dtype=torch.bfloat16, device=q.device)
        lse = torch.empty(Hq, K, dtype=torch.float32, device=q.device)
        ws = tg.new_workspace(K, Hkv * d_h, op=tg.TG_OP_ATTENTION, device=q.device)
        tg.tg_gated_attention(q, k, v, out, ws, s_kept=s_kept, gain=gain, tau=tau_f, lse=lse)
        if check_status:
            _raise_on_status(ws, "tg_gated_attention")
        ctx.save_for_backward(q, k, v, s_kept, gain, out, lse)
        ctx.tau = tau_f
        ctx.tau_is_tensor = isinstance(tau, torch.Tensor)
        if ctx.tau_is_tensor:
            ctx.tau_shape, ctx.tau_device, ctx.tau_dtype = tau.shape, tau.device, tau.dtype
        ctx.check_status = check_status
        return out

    @staticmethod
    def backward(ctx, dout):
        q, k, v, s_kept, gain, out, lse = ctx.saved_tensors
        K, Hq, d_h = q.shape
        Hkv = k.shape[1]
        dout = dout.to(torch.bfloat16).contiguous()
        dq = torch.empty(K, Hq, d_h, dtype=torch.bfloat16, device=q.device)
        dk = torch.empty(K, Hkv, d_h, dtype=torch.bfloat16, device=q.device)
        dv = torch.empty(K, Hkv, d_h, dtype=torch.bfloat16, device=q.device)
        need_s, need_g, need_tau = ctx.needs_input_grad[3], ctx.needs_input_grad[4], ctx.needs_input_grad[5]
        ds = torch.empty(K, dtype=torch.float32, device=q.device) if need_s else None
        dg = torch.empty(Hq, dtype=torch.float32, device=q.device) if need_g else None
        dtau = torch.empty(1, dtype=torch.float32, device=q.device) if need_tau else None
        ws = tg.new_workspace(K, Hq, Hkv, op=tg.TG_OP_ATTENTION_BACKWARD, device=q.device)
        tg.tg_gated_attention_backward(q, k, v, out, dout, lse, dq, dk, dv, ws, s_kept=s_kept, gain=gain,
                                       tau=ctx.tau, ds=ds, dg=dg, dtau=dtau)
        if ctx.check_status:
            _raise_on_status(ws, "tg_gated_attention_backward")
        dtau_out = None
        if need_tau and ctx.tau_is_tensor:
            # the gradient takes tau's own shape, device and dtype ([] or [1], CPU or GPU)
            dtau_out = dtau.reshape(ctx.tau_shape).to(device=ctx.tau_device, dtype=ctx.tau_dtype)
        return dq, dk, dv, ds, dg, dtau_out, None


def gated_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, s_kept: Optional[torch.Tensor] = None,
                    gain: Optional[torch.Tensor] = None, tau: Union[float, torch.Tensor] = 1.0,
                    check_status: Optional[bool] = None) -> torch.Tensor:
    """out [K, Hq, d_h] bf16 of token-gated causal GQA attention over the K kept tokens (q [K, Hq, d_h],
    k and v [K, Hkv, d_h] bf16, s_kept [K] and gain [Hq] fp32 or None, tau > 0 a float or a tensor of
    one element); differentiable with respect to every tensor argument.  check_status: read each call's
    status word back and raise on a timeout or a value out of range (default: the environment variable
    TOKENGATE_CHECK_STATUS)."""
    if check_status is None:
        check_status = os.environ.get("TOKENGATE_CHECK_STATUS", "0") not in ("", "0")
    return GatedAttentionFunction.apply(q, k, v, s_kept, gain, tau, bool(check_status))

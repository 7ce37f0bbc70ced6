"""Token-gated attention as a differentiable torch op (the gradient path the gate trains through).

TokenGate gives each kept token's score a bias on the attention logits above the gate precisely so
that the scorer gets gradients, together with a learned per-head gain and temperature
(aiproducthub.cn article, paragraph 事件详情; aisight.pl article, section Jak to działa; chathome.org
article, section トークンゲート付きアテンションとは).  `gated_attention(q, k, v, s_kept, gain, tau)`
runs tg_gated_attention forward and tg_gated_attention_backward for the gradients of q, k, v, the
kept scores, the gains and the temperature.  Argument marshalling only: both directions are the
library's kernels; torch allocates the outputs and the workspaces.
"""
from __future__ import annotations

from typing import Optional, Union

import torch

from . import tokengate as tg


class GatedAttentionFunction(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, s_kept, gain, tau):
        K, Hq, d_h = q.shape
        Hkv = k.shape[1]
        tau_f = float(tau)
        out = torch.empty(K, Hq, d_h, dtype=torch.bfloat16, device=q.device)
        lse = torch.empty(Hq, K, dtype=torch.float32, device=q.device)
        ws = tg.new_workspace(K, Hkv * d_h, op=tg.TG_OP_ATTENTION, device=q.device)
        tg.tg_gated_attention(q, k, v, out, ws, s_kept=s_kept, gain=gain, tau=tau_f, lse=lse)
        ctx.save_for_backward(q, k, v, s_kept, gain, out, lse)
        ctx.tau = tau_f
        ctx.tau_is_tensor = isinstance(tau, torch.Tensor)
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
        dtau_out = dtau.reshape(()) if (need_tau and ctx.tau_is_tensor) else None
        return dq, dk, dv, ds, dg, dtau_out


def gated_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, s_kept: Optional[torch.Tensor] = None,
                    gain: Optional[torch.Tensor] = None, tau: Union[float, torch.Tensor] = 1.0) -> torch.Tensor:
    """out [K, Hq, d_h] bf16 of token-gated causal GQA attention over the K kept tokens (q [K, Hq, d_h],
    k and v [K, Hkv, d_h] bf16, s_kept [K] and gain [Hq] fp32 or None, tau > 0 a float or a 0-dim
    tensor); differentiable with respect to every tensor argument."""
    return GatedAttentionFunction.apply(q, k, v, s_kept, gain, tau)

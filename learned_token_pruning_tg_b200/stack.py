"""A pruned prefill through a whole decoder stack (the gate layer inside a model).

TokenGate (aiproducthub.cn article, paragraph 事件详情; chathome.org article,
section TokenGate の学習可能なトークンプルーニングの仕組み): a gate after layer
L's attention scores every token from its residual, the best document tokens
are kept (the question always is), and every layer above L sees only the kept
tokens, each kept key carrying its score as a logit bias (scaled by a per-head
gain, with a per-layer temperature).

Decoder layers are Qwen3-1.7B-shaped: pre-norm RMSNorm, GQA attention with
rotate-half RoPE at the original positions, SwiGLU MLP, residual adds.
  layers 0..L-1   dense over all N tokens
  layer L         dense attention over N; gate on its post-attention residual;
                  top-K select; gather of the kept rows, their positions and
                  scores; then layer L's MLP on the K kept rows (the MLP is
                  per token, so this equals running it on N and gathering)
  layers L+1..    over the K kept rows, token-gated attention
Attention (dense layers: K = N, no bias, tau = 1, i.e. plain causal attention),
the Q/K/V projection with RoPE (tg_project_rope, which also writes V's fp16
copy for the attention), the gate, the select and the gather run in
libtokengate; RMSNorm, the output and MLP projections, SwiGLU and the residual
adds are torch (cuBLAS) glue.  The same
object runs the unpruned stack (every layer dense over N) for comparison.
Weights are random (seeded, drawn on the device): there are no trained weights.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Dict, List, Optional

import torch

from . import tokengate as tg


@dataclass(frozen=True)
class StackConfig:
    name: str
    N: int
    doc_begin: int
    doc_end: int
    n_layers: int
    gate_layer: int        # L: the gate scores the residual after this layer's attention
    d: int
    d_ff: int
    Hq: int
    Hkv: int
    d_h: int
    d_g: int
    k_doc: int
    seed: int
    eps: float = 1e-6
    rope_base: float = 1e6

    @property
    def K(self) -> int:
        n_doc = self.doc_end - self.doc_begin
        return min(self.k_doc, n_doc) + (self.N - n_doc)


# 28 Qwen3-1.7B-shaped layers at 64k, gate after layer 13, 8192 document tokens kept.
STACK64K = StackConfig("qwen3-1.7b-stack-64k", N=65536, doc_begin=0, doc_end=65024, n_layers=28, gate_layer=13,
                       d=2048, d_ff=6144, Hq=16, Hkv=8, d_h=128, d_g=256, k_doc=8192, seed=64)
# A small stack for tests.
STACK_TINY = StackConfig("stack-tiny", N=1024, doc_begin=0, doc_end=960, n_layers=4, gate_layer=1, d=256, d_ff=512,
                         Hq=4, Hkv=2, d_h=64, d_g=64, k_doc=192, seed=5)


@dataclass
class LayerWeights:
    ln1: torch.Tensor      # [d] bf16
    Wqkv: torch.Tensor     # [(Hq + 2 Hkv) d_h, d] bf16
    Wo: torch.Tensor       # [d, Hq d_h] bf16
    ln2: torch.Tensor      # [d] bf16
    Wgu: torch.Tensor      # [2 d_ff, d] bf16: SwiGLU gate rows, then up rows
    Wd: torch.Tensor       # [d, d_ff] bf16
    gain: torch.Tensor     # [Hq] fp32 (layers above L)
    tau: float             # (layers above L)


@dataclass
class StackWeights:
    layers: List[LayerWeights]
    W1: torch.Tensor       # gate MLP [d_g, d] bf16
    w2: torch.Tensor       # [d_g] fp32


def random_weights(cfg: StackConfig, device) -> StackWeights:
    """W ~ N(0, 1/fan_in) in bf16, RMSNorm weights 1 + 0.1 N(0, 1), gains ~ U(0, 2), temperatures
    ~ U(0.8, 1.5); drawn on the device from one seeded generator."""
    g = torch.Generator(device=device)
    g.manual_seed(cfg.seed)
    bf = torch.bfloat16

    def w(rows, cols):
        return (torch.randn(rows, cols, generator=g, device=device) / cols ** 0.5).to(bf)

    def ln():
        return (1.0 + 0.1 * torch.randn(cfg.d, generator=g, device=device)).to(bf)

    layers = []
    for _ in range(cfg.n_layers):
        layers.append(LayerWeights(
            ln1=ln(), Wqkv=w((cfg.Hq + 2 * cfg.Hkv) * cfg.d_h, cfg.d), Wo=w(cfg.d, cfg.Hq * cfg.d_h), ln2=ln(),
            Wgu=w(2 * cfg.d_ff, cfg.d), Wd=w(cfg.d, cfg.d_ff),
            gain=2.0 * torch.rand(cfg.Hq, generator=g, device=device),
            tau=float(0.8 + 0.7 * torch.rand(1, generator=g, device=device).item())))
    W1 = w(cfg.d_g, cfg.d)
    w2 = torch.randn(cfg.d_g, generator=g, device=device) / cfg.d_g ** 0.5
    return StackWeights(layers=layers, W1=W1, w2=w2)


def random_embeddings(cfg: StackConfig, device) -> torch.Tensor:
    g = torch.Generator(device=device)
    g.manual_seed(cfg.seed + 1)
    return torch.randn(cfg.N, cfg.d, generator=g, device=device).to(torch.bfloat16)


def rms_norm(x: torch.Tensor, weight: torch.Tensor, eps: float) -> torch.Tensor:
    xf = x.float()
    return (xf * torch.rsqrt(xf.pow(2).mean(-1, keepdim=True) + eps) * weight.float()).to(torch.bfloat16)


class PrunedPrefillStack:
    """Runs the stack; `run(x, prune=True)` prunes at the gate layer, `prune=False` keeps every
    token in every layer.  `capture` (a layer index) keeps that layer's attention inputs."""

    def __init__(self, cfg: StackConfig, weights: StackWeights, device="cuda"):
        self.cfg, self.wts = cfg, weights
        self.dev = torch.device(device)
        self.ws_gate = tg.new_workspace(cfg.N, cfg.d, cfg.d_g, op=tg.TG_OP_GATE, device=self.dev)
        self.ws_attn = tg.new_workspace(0, cfg.Hkv * cfg.d_h, op=tg.TG_OP_ATTENTION, device=self.dev)
        self.ws_proj = tg.new_workspace(cfg.N, cfg.d_h, op=tg.TG_OP_PROJECT, device=self.dev)
        self.v16 = torch.empty(cfg.N, cfg.Hkv * cfg.d_h, dtype=torch.float16, device=self.dev)
        self.captured: Dict[str, torch.Tensor] = {}
        self.kept: Optional[torch.Tensor] = None
        self.scores: Optional[torch.Tensor] = None
        # per layer (k, v, s): the KV cache a prefill leaves for decoding; s is the kept keys' scores
        # (their logit bias) in the layers above L, None below
        self.kv: List[tuple] = []

    def _attention(self, li: int, x: torch.Tensor, pos: torch.Tensor, s_kept, gated: bool, capture: bool,
                   keep_kv: bool):
        c, lw = self.cfg, self.wts.layers[li]
        n = x.shape[0]
        qkv = torch.empty(n, (c.Hq + 2 * c.Hkv) * c.d_h, dtype=torch.bfloat16, device=self.dev)
        v16 = self.v16[:n]
        tg.tg_project_rope(rms_norm(x, lw.ln1, c.eps), lw.Wqkv, pos, qkv, self.ws_proj, c.Hq, c.Hkv, c.d_h,
                           base=c.rope_base, v16=v16)
        q = qkv[:, : c.Hq * c.d_h].view(n, c.Hq, c.d_h)
        k = qkv[:, c.Hq * c.d_h: (c.Hq + c.Hkv) * c.d_h].view(n, c.Hkv, c.d_h)
        v = qkv[:, (c.Hq + c.Hkv) * c.d_h:].view(n, c.Hkv, c.d_h)
        if keep_kv:
            self.kv.append((k.clone(), v.clone(), s_kept if gated else None))
        out = torch.empty(n, c.Hq, c.d_h, dtype=torch.bfloat16, device=self.dev)
        if gated:
            tg.tg_gated_attention_f16v(q, k, v16, out, self.ws_attn, s_kept=s_kept, gain=lw.gain, tau=lw.tau)
        else:
            tg.tg_gated_attention_f16v(q, k, v16, out, self.ws_attn, tau=1.0)
        if capture:
            self.captured = {"q": q.clone(), "k": k.clone(), "v": v.clone(), "out": out.clone(),
                             "s": None if s_kept is None else s_kept.clone(), "gain": lw.gain.clone(),
                             "tau": torch.tensor(lw.tau if gated else 1.0)}
        return x + torch.matmul(out.view(n, c.Hq * c.d_h), lw.Wo.t())

    def _mlp(self, li: int, x: torch.Tensor) -> torch.Tensor:
        c, lw = self.cfg, self.wts.layers[li]
        gu = torch.matmul(rms_norm(x, lw.ln2, c.eps), lw.Wgu.t())
        a = torch.nn.functional.silu(gu[:, : c.d_ff].float()) * gu[:, c.d_ff:].float()
        return x + torch.matmul(a.to(torch.bfloat16), lw.Wd.t())

    def run(self, x: torch.Tensor, prune: bool = True, capture: Optional[int] = None,
            keep_kv: bool = False) -> torch.Tensor:
        """x: [N, d] bf16 embeddings on the device.  Returns the final hidden states of the kept tokens
        ([K, d] when pruning, [N, d] otherwise); self.kept holds the kept indices when pruning, and
        self.kv each layer's post-RoPE K and V (and the kept scores above L) when keep_kv."""
        c = self.cfg
        self.kv = []
        pos = torch.arange(c.N, dtype=torch.int32, device=self.dev)
        s_kept = None
        for li in range(c.n_layers):
            gated = prune and li > c.gate_layer
            x = self._attention(li, x, pos, s_kept, gated, capture == li, keep_kv)
            if prune and li == c.gate_layer:
                # the gate on layer L's post-attention residual, then top-K and the gather
                self.scores = torch.empty(c.N, dtype=torch.float32, device=self.dev)
                tg.tg_gate_score_for_select(x, self.wts.W1, self.wts.w2, self.scores, self.ws_gate, c.doc_begin,
                                            c.doc_end, eps=c.eps)
                self.kept = torch.empty(c.K, dtype=torch.int32, device=self.dev)
                tg.tg_topk_select_after_gate(self.scores, c.doc_begin, c.doc_end, c.k_doc, self.kept, self.ws_gate)
                xk = torch.empty(c.K, c.d, dtype=torch.bfloat16, device=self.dev)
                pk = torch.empty(c.K, dtype=torch.int32, device=self.dev)
                s_kept = torch.empty(c.K, dtype=torch.float32, device=self.dev)
                tg.tg_gather_compact(x, self.kept, xk, pk, pos_in=pos, scores=self.scores, s_out=s_kept)
                x, pos = xk, pk
            x = self._mlp(li, x)
        return x

    def kv_bytes(self) -> int:
        return sum(k.numel() * k.element_size() + v.numel() * v.element_size() +
                   (0 if sc is None else sc.numel() * 4) for k, v, sc in self.kv)

    def device_status(self) -> int:
        return (tg.tg_device_status(self.ws_gate) | tg.tg_device_status(self.ws_attn) |
                tg.tg_device_status(self.ws_proj))

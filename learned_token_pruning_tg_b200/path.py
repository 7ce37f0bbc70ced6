"""One TokenGate gate layer's prefill hot path, as a user calls it.

Layers below the gate run over all N tokens; at the gate layer every token is
scored, the best document tokens are kept (the question always is), the kept
rows are compacted, and the attention of the next layer runs over the K kept
tokens with the token-gated logit bias (TokenGate pages: aiproducthub.cn
article, paragraph 事件详情; chathome.org article, sections TokenGate の学習可能な
トークンプルーニングの仕組み and トークンゲート付きアテンションとは).

Steps, in order, all on the caller's current CUDA stream:
  gate     tg_gate_score_for_select libtokengate (tcgen05 GEMM + fused epilogue, which also
                                    counts the select's first radix pass)
  select   tg_topk_select_after_gate libtokengate (radix select from that count)
  gather   tg_gather_compact        libtokengate (bulk row copy; also the kept rows'
                                    positions and scores)
  proj     tg_project_rope          libtokengate (tcgen05 GEMM of the kept rows with
                                    RoPE and V's fp16 copy in its epilogue)
  attn     tg_gated_attention_f16v  libtokengate (tcgen05 flash attention)
With gather_into_projection=True the compaction instead happens on the way into
the projection: the select also writes the kept scores
(tg_topk_select_after_gate_kept_scores) and the projection's operand tiles are
the kept rows of h fetched by TMA gather4 copies (tg_project_rope_gather), so
no compacted copy is written (stages "gate", "select", "proj", "attn").  It is
not the default: on a B200 the gathered projection took 181 us at the 128k
workload against 9 + 72 us for the copy and the dense projection (four rows of
128 bytes per copy instruction, issued again for every one of the 16 column
tiles).  With fused_projection=False the projection is a library GEMM
(torch.matmul, cuBLAS) over the compacted rows followed by tg_rope_apply, and
the attention converts V itself (tg_gated_attention); stages "gather", "qkv",
"rope", "attn".
torch allocates every buffer once (plumbing); the kept count K is known on the
host, so nothing synchronizes inside a step.
"""
from __future__ import annotations

from typing import Callable, Optional

import torch

from . import tokengate as tg

STAGES_GATHER_FUSED = ("gate", "select", "proj", "attn")
STAGES_FUSED = ("gate", "select", "gather", "proj", "attn")
STAGES_UNFUSED = ("gate", "select", "gather", "qkv", "rope", "attn")
STAGES = STAGES_FUSED


def nvtx_marks() -> Callable[[str], None]:
    """A `mark` hook for GatedPrefillLayer.run that wraps each step in an NVTX range named
    "tg:<step>" (so a profiler can select one step, e.g. ncu --nvtx --nvtx-include "tg:attn/")."""
    open_range = [False]

    def mark(name: str) -> None:
        if open_range[0]:
            torch.cuda.nvtx.range_pop()
        open_range[0] = name != "end"
        if open_range[0]:
            torch.cuda.nvtx.range_push("tg:" + name)

    return mark


class GatedPrefillLayer:
    def __init__(self, N: int, doc_begin: int, doc_end: int, k_doc: int, W1: torch.Tensor, w2: torch.Tensor,
                 Wqkv: torch.Tensor, Hq: int, Hkv: int, d_h: int, gain: torch.Tensor, tau: float,
                 b1: Optional[torch.Tensor] = None, b2: float = 0.0, rms_weight: Optional[torch.Tensor] = None,
                 eps: float = 1e-6, rope_base: float = 1e6, device="cuda", fused_projection: bool = True,
                 gather_into_projection: bool = False):
        self.N, self.doc_begin, self.doc_end, self.k_doc = N, doc_begin, doc_end, k_doc
        self.K = tg.tg_kept_count(N, doc_begin, doc_end, k_doc)
        if self.K < 0:
            raise ValueError("bad document span or budget")
        dev = torch.device(device)
        self.d_g, self.d = W1.shape
        self.Hq, self.Hkv, self.d_h = Hq, Hkv, d_h
        self.W1 = W1.to(dev, torch.bfloat16).contiguous()
        self.w2 = w2.to(dev, torch.float32).contiguous()
        self.b1 = None if b1 is None else b1.to(dev, torch.float32).contiguous()
        self.b2 = float(b2)
        self.rms_weight = None if rms_weight is None else rms_weight.to(dev, torch.bfloat16).contiguous()
        self.eps, self.rope_base, self.tau = eps, rope_base, float(tau)
        self.fused = fused_projection
        self.gather_fused = fused_projection and gather_into_projection
        self.stages = (STAGES_GATHER_FUSED if self.gather_fused else STAGES_FUSED) if fused_projection else STAGES_UNFUSED
        self.Wqkv = Wqkv.to(dev, torch.bfloat16).contiguous()             # [(Hq + 2 Hkv) d_h, d]
        self.WqkvT = None if fused_projection else self.Wqkv.t().contiguous()
        self.gain = gain.to(dev, torch.float32).contiguous()
        K, d = self.K, self.d
        self.ws = tg.new_workspace(N, d, self.d_g, op=tg.TG_OP_GATE, device=dev)  # gate and select
        if fused_projection:
            self.ws_proj = tg.new_workspace(K, d_h, op=tg.TG_OP_PROJECT, device=dev)
            self.ws_attn = tg.new_workspace(0, Hkv * d_h, op=tg.TG_OP_ATTENTION, device=dev)
            self.v16 = torch.empty(K, Hkv * d_h, dtype=torch.float16, device=dev)
        else:
            self.ws_proj = None
            self.ws_attn = tg.new_workspace(K, Hkv * d_h, op=tg.TG_OP_ATTENTION, device=dev)
            self.v16 = None
        self.scores = torch.empty(N, dtype=torch.float32, device=dev)
        self.kept = torch.empty(max(K, 1), dtype=torch.int32, device=dev)
        # the compacted rows exist only when a separate step writes them
        self.h_kept = None if self.gather_fused else torch.empty(K, d, dtype=torch.bfloat16, device=dev)
        self.pos = torch.empty(max(K, 1), dtype=torch.int32, device=dev)
        self.s_kept = torch.empty(max(K, 1), dtype=torch.float32, device=dev)
        self.qkv = torch.empty(K, (Hq + 2 * Hkv) * d_h, dtype=torch.bfloat16, device=dev)
        self.q = self.qkv[:, : Hq * d_h].view(K, Hq, d_h)
        self.k = self.qkv[:, Hq * d_h: (Hq + Hkv) * d_h].view(K, Hkv, d_h)
        self.v = self.qkv[:, (Hq + Hkv) * d_h:].view(K, Hkv, d_h)
        self.out = torch.empty(K, Hq, d_h, dtype=torch.bfloat16, device=dev)

    def stage_calls(self, h: torch.Tensor):
        """{step name: a call running that step alone on the layer's buffers}, in path order.  Each
        step reads only what the steps before it wrote, so after one full pass any step may be run
        again by itself (the benchmark times each step this way)."""
        K = self.K

        def gate():
            # also counts the select's first radix pass in the workspace (the select below starts from it)
            tg.tg_gate_score_for_select(h, self.W1, self.w2, self.scores, self.ws, self.doc_begin, self.doc_end,
                                        b1=self.b1, b2=self.b2, rms_weight=self.rms_weight, eps=self.eps)

        def select():
            if self.gather_fused:
                tg.tg_topk_select_after_gate_kept_scores(self.scores, self.doc_begin, self.doc_end, self.k_doc,
                                                         self.kept[:K], self.s_kept[:K], self.ws)
            else:
                tg.tg_topk_select_after_gate(self.scores, self.doc_begin, self.doc_end, self.k_doc, self.kept[:K],
                                             self.ws)

        def gather():
            tg.tg_gather_compact(h, self.kept[:K], self.h_kept, self.pos[:K], scores=self.scores,
                                 s_out=self.s_kept[:K])

        def proj():
            if self.gather_fused:
                # the positions are the kept indices themselves
                tg.tg_project_rope_gather(h, self.kept[:K], self.Wqkv, self.kept[:K], self.qkv, self.ws_proj,
                                          self.Hq, self.Hkv, self.d_h, base=self.rope_base, v16=self.v16)
            else:
                tg.tg_project_rope(self.h_kept, self.Wqkv, self.pos[:K], self.qkv, self.ws_proj, self.Hq, self.Hkv,
                                   self.d_h, base=self.rope_base, v16=self.v16)

        def qkv():
            torch.matmul(self.h_kept, self.WqkvT, out=self.qkv)

        def rope():
            tg.tg_rope_apply(self.q, self.k, self.pos[:K], self.rope_base)

        def attn():
            if self.fused:
                tg.tg_gated_attention_f16v(self.q, self.k, self.v16, self.out, self.ws_attn,
                                           s_kept=self.s_kept[:K], gain=self.gain, tau=self.tau)
            else:
                tg.tg_gated_attention(self.q, self.k, self.v, self.out, self.ws_attn, s_kept=self.s_kept[:K],
                                      gain=self.gain, tau=self.tau)

        calls = {"gate": gate, "select": select, "gather": gather, "proj": proj, "qkv": qkv, "rope": rope,
                 "attn": attn}
        return {name: calls[name] for name in self.stages}

    def run(self, h: torch.Tensor, mark: Optional[Callable[[str], None]] = None):
        """Runs the steps on device-resident h [N, d]; returns (out [K, Hq, d_h], kept [K]).
        `mark(name)` is called before each step (self.stages) and with "end" after the last."""
        m = mark or (lambda _n: None)
        for name, call in self.stage_calls(h).items():
            m(name)
            call()
        m("end")
        return self.out, self.kept[:self.K]

    def run_host(self, h_host: torch.Tensor, h_dev: torch.Tensor, out_host: torch.Tensor,
                 kept_host: torch.Tensor):
        """End to end from host memory: copies pinned h_host into h_dev, runs the layer, and copies
        the attention output and kept indices back into pinned host tensors (all asynchronous)."""
        h_dev.copy_(h_host, non_blocking=True)
        out, kept = self.run(h_dev)
        out_host.copy_(out, non_blocking=True)
        kept_host.copy_(kept, non_blocking=True)
        return out_host, kept_host

    def positions(self) -> torch.Tensor:
        """[K] int32 original positions of the kept rows (the kept indices when the gather is fused)."""
        return self.kept[:self.K] if self.gather_fused else self.pos[:self.K]

    def launches_per_step(self) -> int:
        """libtokengate kernels per run(): gate (+ the RMSNorm-weight fold), select, then the projection with
        its gather and the attention; or a separate gather, the projection and the attention; or a gather,
        RoPE and the attention's two (V to fp16, attention) after the library GEMM."""
        n = 4 if self.gather_fused else (5 if self.fused else 6)
        return n + (1 if self.rms_weight is not None else 0)

    def device_status(self) -> int:
        """OR of the status words of the layer's workspaces (synchronizes the stream); 0 = no timeout
        and no value out of range."""
        st = tg.tg_device_status(self.ws) | tg.tg_device_status(self.ws_attn)
        return st | (tg.tg_device_status(self.ws_proj) if self.ws_proj is not None else 0)

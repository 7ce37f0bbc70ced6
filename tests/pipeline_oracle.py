"""The whole gate-layer prefill computed by the oracle alone (test infrastructure).

Each step is the oracle's own routine, in the order of the method's forward pass (aiproducthub.cn
article, paragraph 事件详情: score every token at the gate layer, keep the top-K document tokens and
every question token, run the layers above on the kept tokens only): gate score -> top-K select ->
gather -> projection -> RoPE -> token-gated attention.  The steps are only chained here; the heavy
ones are split over worker processes by rows (rows are independent in each of them).

The values handed from one step to the next are rounded where the library's interface stores them:
scores in fp32 (the select ranks fp32 scores), Q and K in bf16, and V in fp16 (the projection hands
the attention an fp16 copy of V; `v_format="bf16"` for a path whose attention reads bf16 V).  That is
the format of the interface, not arithmetic of the kernels, so the oracle rounds at the same places
and computes everything else in fp64.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np
import torch

import oracle
from tests import oracle_pool


def to_bf16(x: np.ndarray) -> np.ndarray:
    """Round to bf16 (nearest, ties to even: torch's conversion) and widen back to fp32."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).float().numpy()


def to_f16(x: np.ndarray) -> np.ndarray:
    """Round to fp16 (nearest, ties to even) and widen back to fp32."""
    return np.asarray(x, dtype=np.float64).astype(np.float16).astype(np.float32)


@dataclass
class OraclePrefill:
    scores: np.ndarray          # [N] fp64
    kept: np.ndarray            # [K] int32, the oracle's own selection
    threshold: float            # the k_doc-th document score in the selection order
    kept_used: np.ndarray       # the kept set the later steps ran on
    h_kept_bits: np.ndarray     # [K, d] uint16
    pos: np.ndarray             # [K] int32
    s_kept: np.ndarray          # [K] fp32
    q: np.ndarray               # [n_rows, Hq, d_h] fp64 (rotated), for the requested rows
    k: np.ndarray               # [K, Hkv, d_h] fp64 (rotated)
    v: np.ndarray               # [K, Hkv, d_h] fp64
    rows: np.ndarray            # query rows of q and out
    out: np.ndarray             # [n_rows, Hq, d_h] fp64 attention output
    absum_q: np.ndarray         # [n_rows, Hq * d_h] sum of |x| |W| per output (accumulation bound)
    absum_kv: np.ndarray        # [n_rows, 2 Hkv d_h]


def gate_layer(h_bits: np.ndarray, W1: np.ndarray, w2: np.ndarray, Wqkv: np.ndarray, doc_begin: int, doc_end: int,
               k_doc: int, Hq: int, Hkv: int, d_h: int, gain: np.ndarray, tau: float, rows: np.ndarray,
               eps: float = 1e-6, rope_base: float = 1e6, kept_override: Optional[np.ndarray] = None,
               scores: Optional[np.ndarray] = None, v_format: str = "f16") -> OraclePrefill:
    """h_bits: [N, d] uint16 (bf16 patterns of the hidden states at the gate layer); W1 [d_g, d], Wqkv
    [(Hq + 2 Hkv) d_h, d] fp32 values; rows: the kept rows whose attention output is wanted.
    kept_override: run the steps after the select on this kept set instead of the oracle's own (used
    only when the two differ in tokens the acceptance rule allows to differ).  scores: the oracle's
    gate scores when already computed."""
    h = h_bits.view(np.uint16).astype(np.uint32) << 16
    h = h.view(np.float32)
    if scores is None:
        scores = oracle_pool.gate_scores(h, W1, w2, eps=eps)
    s32 = scores.astype(np.float32)
    kept = oracle.topk_select(s32, doc_begin, doc_end, k_doc)
    thr = oracle.topk_threshold(s32, doc_begin, doc_end, k_doc)
    kept_used = kept if kept_override is None else np.asarray(kept_override, dtype=np.int32)
    h_kept_bits, pos, s_kept = oracle.gather_compact(h_bits, kept_used, scores=s32)
    x = (h_kept_bits.astype(np.uint32) << 16).view(np.float32)
    K = x.shape[0]
    cq = Hq * d_h
    ck = Hkv * d_h
    Wq, Wkv = Wqkv[:cq], Wqkv[cq:]
    rows = np.asarray(rows, dtype=np.int64)
    q_pre = oracle_pool.project(x[rows], Wq)
    kv_pre = oracle_pool.project(x, Wkv)
    absum_q = oracle_pool.project(np.abs(x[rows]), np.abs(Wq))
    absum_kv = oracle_pool.project(np.abs(x[rows]), np.abs(Wkv))
    # RoPE at the original positions (the oracle's rotation takes fp32 inputs: the fp64 projection is
    # rounded to fp32 there, 2^-24 relative, far below every tolerance that follows)
    q = oracle.rope(q_pre.astype(np.float32).reshape(len(rows), Hq, d_h), pos[rows], rope_base)
    k = oracle.rope(kv_pre[:, :ck].astype(np.float32).reshape(K, Hkv, d_h), pos, rope_base)
    v = kv_pre[:, ck:].reshape(K, Hkv, d_h)
    # attention over Q, K in bf16 and V in the interface's format; a full Q array holds the requested rows
    qf = np.zeros((K, Hq, d_h), dtype=np.float32)
    qf[rows] = to_bf16(q)
    vr = to_f16(v) if v_format == "f16" else to_bf16(v)
    out = oracle_pool.gated_attention(qf, to_bf16(k), vr, s=s_kept, g=gain, tau=tau, rows=rows)
    return OraclePrefill(scores=scores, kept=kept, threshold=thr, kept_used=kept_used, h_kept_bits=h_kept_bits,
                         pos=pos, s_kept=s_kept, q=q, k=k, v=v, rows=rows, out=out, absum_q=absum_q,
                         absum_kv=absum_kv)

"""Seeded synthetic inputs for the TokenGate prefill hot path.

This module only draws random numbers: it holds none of the method's
arithmetic, so both the CUDA path and the CPU oracle can be fed from it.
Everything is drawn on the CPU with ``torch.Generator().manual_seed(seed)`` in
fp32 and then rounded to bf16 where a workload is bf16.

The workloads stand in for the pages' evaluation suites (NIAH, RepoBench-P,
2WikiMultihopQA, MultiNews, BioDEX), which are not available: they keep the
lengths the pages report (16k to 128k tokens), the document/question split of
the prompt (only the document is prunable), and Qwen3-1.7B layer shapes
(hidden 2048, 16 query / 8 KV heads, head dim 128).
"""
from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Optional

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    N: int                 # tokens in the prompt
    doc_begin: int         # prunable document span [doc_begin, doc_end)
    doc_end: int
    d: int                 # hidden size
    d_g: int               # gate MLP width
    k_doc: int             # document tokens kept
    Hq: int
    Hkv: int
    d_h: int
    seed: int
    n_scaled: int          # rows of h scaled by `scale` (planted needles / heavy rows)
    scale: float
    tau: Optional[float] = None            # fixed temperature, else drawn
    tau_range: tuple = (0.8, 1.5)
    gain_range: tuple = (0.0, 2.0)
    zero_gain: bool = False
    bf16: bool = True
    rope_base: float = 1e6
    eps: float = 1e-6

    @property
    def n_doc(self) -> int:
        return self.doc_end - self.doc_begin

    @property
    def K(self) -> int:
        return min(self.k_doc, self.n_doc) + (self.N - self.n_doc)


# Tiny case (fp32 on the oracle side; the GPU sees the bf16-rounded values).
TINY = Workload("tiny-1k", N=1024, doc_begin=0, doc_end=960, d=256, d_g=64, k_doc=192,
                Hq=4, Hkv=2, d_h=64, seed=0, n_scaled=8, scale=4.0, tau=1.2,
                gain_range=(0.5, 1.5), bf16=False)
# Qwen3-1.7B-shaped gate layer at 16k.
L16K = Workload("qwen3-1.7b-16k", N=16384, doc_begin=0, doc_end=16000, d=2048, d_g=256,
                k_doc=1024, Hq=16, Hkv=8, d_h=128, seed=16, n_scaled=32, scale=4.0)
# Budget sweep at 32k (one fresh seed per budget) and the K = N reference run.
L32K_SWEEP = tuple(
    Workload(f"qwen3-1.7b-32k-k{k}", N=32768, doc_begin=0, doc_end=32256, d=2048, d_g=256,
             k_doc=k, Hq=16, Hkv=8, d_h=128, seed=3201 + i, n_scaled=0, scale=1.0)
    for i, k in enumerate((512, 2048, 8192, 16384)))
L32K_FULL = Workload("qwen3-1.7b-32k-full", N=32768, doc_begin=0, doc_end=32256, d=2048,
                     d_g=256, k_doc=32256, Hq=16, Hkv=8, d_h=128, seed=3205, n_scaled=0,
                     scale=1.0, tau=1.0, zero_gain=True)
# Long context at 128k: 3% of the rows scaled x3 (heavy-tailed rows).
L128K = Workload("qwen3-1.7b-128k", N=131072, doc_begin=0, doc_end=130560, d=2048, d_g=256,
                 k_doc=4096, Hq=16, Hkv=8, d_h=128, seed=128, n_scaled=(3 * 131072) // 100,
                 scale=3.0)

WORKLOADS = {w.name: w for w in (TINY, L16K, *L32K_SWEEP, L32K_FULL, L128K)}


def scaled(w: Workload, **kw) -> Workload:
    """A copy of a workload with some fields changed (smaller parity cases)."""
    return replace(w, **kw)


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def _q(x: torch.Tensor, bf16: bool) -> torch.Tensor:
    return x.to(torch.bfloat16) if bf16 else x


@dataclass
class GateInputs:
    h: torch.Tensor          # [N, d]
    W1: torch.Tensor         # [d_g, d]
    w2: torch.Tensor         # [d_g] fp32
    b1: Optional[torch.Tensor] = None
    b2: float = 0.0
    gamma: Optional[torch.Tensor] = None
    scaled_rows: torch.Tensor = field(default_factory=lambda: torch.empty(0, dtype=torch.long))


def gate_inputs(w: Workload, seed: Optional[int] = None, with_bias=False, with_gamma=False) -> GateInputs:
    """Hidden states at the gate layer and the gate MLP weights.

    h ~ N(0, 1) with `n_scaled` document rows (chosen by randperm over the
    document span) multiplied by `scale`; W1 ~ N(0, 1/d); w2 ~ N(0, 1/d_g)."""
    g = _gen(w.seed if seed is None else seed)
    h = torch.randn(w.N, w.d, generator=g)
    perm = torch.randperm(w.n_doc, generator=g)[: w.n_scaled] + w.doc_begin
    if w.n_scaled:
        h[perm] *= w.scale
    W1 = torch.randn(w.d_g, w.d, generator=g) / w.d ** 0.5
    w2 = torch.randn(w.d_g, generator=g) / w.d_g ** 0.5
    b1 = torch.randn(w.d_g, generator=g) * 0.1 if with_bias else None
    b2 = float(torch.randn(1, generator=g).item() * 0.1) if with_bias else 0.0
    gamma = (1.0 + 0.25 * torch.randn(w.d, generator=g)) if with_gamma else None
    if gamma is not None:
        gamma = _q(gamma, w.bf16)
    return GateInputs(h=_q(h, w.bf16), W1=_q(W1, w.bf16), w2=w2, b1=b1, b2=b2, gamma=gamma,
                      scaled_rows=perm)


@dataclass
class AttnParams:
    Wq: torch.Tensor         # [Hq*d_h, d]
    Wk: torch.Tensor         # [Hkv*d_h, d]
    Wv: torch.Tensor         # [Hkv*d_h, d]
    tau: float
    gain: torch.Tensor       # [Hq] fp32


def attn_params(w: Workload, seed: Optional[int] = None) -> AttnParams:
    """Random-init projections ~ N(0, 1/d), temperature and per-head gains."""
    g = _gen((w.seed if seed is None else seed) + 7919)
    Wq = torch.randn(w.Hq * w.d_h, w.d, generator=g) / w.d ** 0.5
    Wk = torch.randn(w.Hkv * w.d_h, w.d, generator=g) / w.d ** 0.5
    Wv = torch.randn(w.Hkv * w.d_h, w.d, generator=g) / w.d ** 0.5
    lo, hi = w.tau_range
    tau = w.tau if w.tau is not None else float(lo + (hi - lo) * torch.rand(1, generator=g).item())
    glo, ghi = w.gain_range
    gain = glo + (ghi - glo) * torch.rand(w.Hq, generator=g)
    if w.zero_gain:
        gain = torch.zeros(w.Hq)
    return AttnParams(Wq=_q(Wq, True), Wk=_q(Wk, True), Wv=_q(Wv, True), tau=tau, gain=gain)


@dataclass
class QKV:
    q: torch.Tensor          # [K, Hq, d_h] bf16
    k: torch.Tensor          # [K, Hkv, d_h] bf16
    v: torch.Tensor          # [K, Hkv, d_h] bf16
    s: torch.Tensor          # [K] fp32 kept-token scores
    gain: torch.Tensor       # [Hq] fp32
    tau: float
    pos: torch.Tensor        # [K] int32 ascending original positions


def qkv(K: int, Hq: int, Hkv: int, d_h: int, seed: int, score_std=0.6, tau_range=(0.8, 1.5),
        gain_range=(0.0, 2.0), n_pos: Optional[int] = None, heavy_frac=0.0, heavy_scale=3.0) -> QKV:
    """Direct attention inputs: q, k, v ~ N(0, 1) (what h' W^T gives for unit-rms rows and
    N(0, 1/d) weights), a fraction of rows scaled like the heavy rows of the 128k workload,
    scores ~ N(0, score_std^2), and K ascending positions drawn from [0, n_pos)."""
    g = _gen(seed)
    q = torch.randn(K, Hq, d_h, generator=g)
    k = torch.randn(K, Hkv, d_h, generator=g)
    v = torch.randn(K, Hkv, d_h, generator=g)
    if heavy_frac > 0:
        n = int(heavy_frac * K)
        rows = torch.randperm(K, generator=g)[:n]
        q[rows] *= heavy_scale
        k[rows] *= heavy_scale
        v[rows] *= heavy_scale
    s = torch.randn(K, generator=g) * score_std
    lo, hi = tau_range
    tau = float(lo + (hi - lo) * torch.rand(1, generator=g).item())
    glo, ghi = gain_range
    gain = glo + (ghi - glo) * torch.rand(Hq, generator=g)
    n_pos = n_pos or K
    pos = torch.sort(torch.randperm(n_pos, generator=g)[:K]).values.to(torch.int32)
    return QKV(q=q.to(torch.bfloat16), k=k.to(torch.bfloat16), v=v.to(torch.bfloat16), s=s,
               gain=gain, tau=tau, pos=pos)


def grad_out(K: int, Hq: int, d_h: int, seed: int, std: float = 1.0) -> torch.Tensor:
    """An upstream gradient for the attention output: [K, Hq, d_h] bf16 ~ N(0, std^2)."""
    g = _gen(seed)
    return (torch.randn(K, Hq, d_h, generator=g) * std).to(torch.bfloat16)


def score_vector(N: int, seed: int, kind: str = "normal") -> torch.Tensor:
    """fp32 score vectors for select-only stress cases.

    normal : N(0, 1)
    heavy  : 97% N(0, 1) and 3% of entries x3 (bucket skew in the high digits)
    ties   : N(0, 1) quantised to 64 levels, with +0/-0 mixed in
    const  : every score equal (pure index tie-break)
    special: normal plus +-inf, NaN, +0 and -0 sprinkled in
    """
    g = _gen(seed)
    s = torch.randn(N, generator=g)
    if kind == "normal":
        return s
    if kind == "heavy":
        idx = torch.randperm(N, generator=g)[: (3 * N) // 100]
        s[idx] *= 3.0
        return s
    if kind == "ties":
        s = torch.round(s * 8.0) / 8.0
        z = torch.rand(N, generator=g) < 0.5
        s[(s == 0) & z] = -0.0
        return s
    if kind == "const":
        return torch.full((N,), 0.25)
    if kind == "special":
        u = torch.rand(N, generator=g)
        s[u < 0.01] = float("nan")
        s[(u >= 0.01) & (u < 0.02)] = float("inf")
        s[(u >= 0.02) & (u < 0.03)] = float("-inf")
        s[(u >= 0.03) & (u < 0.04)] = 0.0
        s[(u >= 0.04) & (u < 0.05)] = -0.0
        return s
    raise ValueError(kind)

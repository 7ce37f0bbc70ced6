"""The prefill path as the benchmark runs it -- GatedPrefillLayer built by bench.make_layer for each
workload, at full size, one pass -- against the whole gate layer computed by the oracle alone from the
same hidden states (tests/pipeline_oracle.py).  The method's forward pass: score every token at the
gate layer, keep the top-K document tokens and every question token, run the next layer's attention
over the kept tokens only with the kept scores as a logit bias (aiproducthub.cn article, paragraph
事件详情; chathome.org article, sections TokenGate の学習可能なトークンプルーニングの仕組み and
トークンゲート付きアテンションとは).

Acceptance, step by step (the specification's rules, and bounds derived from the arithmetic):
  scores   every score within 5e-3 of the oracle's (the specification), and within a derived 2e-4
           (fp32 accumulation of d products and a fast exponential in SiLU);
  select   bit-exact against the oracle's select run on the GPU's own scores; against the oracle's
           own selection a token may be in one set and not the other only if its oracle score lies
           within 1e-4 of the oracle's threshold (the k_doc-th document score);
  gather   rows, positions and kept scores bit-exact;
  Q, K, V  on the sampled rows, every element within the bf16 roundings of the path of the exact
           value: the rotated q, k pairs within 2^-7 of the pair's magnitude (at most two roundings of
           a rotation that preserves the pair's norm), v within half a bf16 ulp, each plus 2^-20 of
           the sum of absolute products (fp32 accumulation);
  out      on the sampled rows: (a) against the oracle's attention over the path's own Q, K (bf16),
           V (the fp16 copy the projection writes and the attention reads) and kept scores -- the
           specification's 1e-2 as a raw max abs error wherever the output is below 2 in magnitude
           (its half ulp is at most 2^-8 there), and 1e-2 above the output's half ulp elsewhere;
           (b) against the oracle's own pipeline, whose Q and K are rounded to bf16 and V to fp16 at
           the same interface points: the same 1e-2 bar plus the first-order effect of the
           differences between the two sides' rounded Q, K, V and fp32 scores (each side rounds its
           own exact values, so single elements may differ by one ulp):
           |dO| <= max_c |dv_c| + 2 max_c |dl_c| max_c |v_c - O|, with dl_c the logit difference the
           two sides' inputs give.
"""
import numpy as np
import pytest
import torch

import bench
import oracle
from learned_token_pruning_tg_b200 import synth
from tests import pipeline_oracle

pytestmark = pytest.mark.gpu

WORKLOADS = ["tiny-1k", "qwen3-1.7b-16k", "qwen3-1.7b-32k-k512", "qwen3-1.7b-32k-k2048", "qwen3-1.7b-32k-k8192",
             "qwen3-1.7b-32k-k16384", "qwen3-1.7b-32k-full", "qwen3-1.7b-128k"]

ATTN_TOL = 1e-2


def half_ulp_bf16(x):
    a = np.abs(x)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, 2.0 ** (e - 8), 0.0)


def attn_excess(got, want):
    """Error above the bar's allowance: raw |got - want| where |want| < 2, else the excess over the
    output's own half ulp."""
    err = np.abs(got - want)
    return np.where(np.abs(want) < 2.0, err, err - half_ulp_bf16(want))


def sample_rows(K, kept, heavy_rows, n=48):
    rows = [np.linspace(0, K - 1, min(n, K)).astype(np.int64), np.arange(min(4, K)), np.arange(max(0, K - 8), K)]
    heavy_in_kept = np.flatnonzero(np.isin(kept, heavy_rows))
    rows.append(heavy_in_kept[:: max(1, len(heavy_in_kept) // 8)][:8])
    return np.unique(np.concatenate(rows))


CASES = [(name, False) for name in WORKLOADS] + [(name, True) for name in ("tiny-1k", "qwen3-1.7b-16k",
                                                                             "qwen3-1.7b-128k")]


@pytest.mark.parametrize("name,gather_into_projection", CASES,
                         ids=[f"{n}{'-gathered-projection' if g else ''}" for n, g in CASES])
def test_path_matches_oracle_pipeline(name, gather_into_projection):
    # gather_into_projection: the layer whose projection gathers the kept rows from h itself
    w = synth.WORKLOADS[name]
    gi = synth.gate_inputs(w)
    ap = synth.attn_params(w)
    dev = torch.device("cuda", 0)
    h = gi.h.to(torch.bfloat16)
    layer = bench.make_layer(w, gi, ap, dev, gather_into_projection=gather_into_projection)
    out, kept = layer.run(h.to(dev))
    torch.cuda.synchronize()
    assert layer.device_status() == 0
    K = w.K
    assert kept.shape[0] == K

    s_gpu = layer.scores.cpu().numpy()
    kept_gpu = kept.cpu().numpy()
    h_bits = h.view(torch.int16).numpy().view(np.uint16)
    W1 = gi.W1.to(torch.bfloat16).float().numpy()
    Wqkv = torch.cat([ap.Wq, ap.Wk, ap.Wv]).float().numpy()
    rows = sample_rows(K, kept_gpu, gi.scaled_rows.numpy())

    # select on the GPU's own scores: bit-exact
    assert np.array_equal(kept_gpu, oracle.topk_select(s_gpu, w.doc_begin, w.doc_end, w.k_doc))
    assert np.all(np.isin(np.arange(w.doc_end, w.N), kept_gpu)), "a question token was dropped"

    # the oracle's own pipeline (its own scores and selection; the steps after the select run on the
    # GPU's kept set only where the two sets differ in tokens the rule allows to differ)
    o = pipeline_oracle.gate_layer(h_bits, W1, gi.w2.numpy(), Wqkv, w.doc_begin, w.doc_end, w.k_doc, w.Hq, w.Hkv,
                                   w.d_h, ap.gain.numpy(), ap.tau, rows, eps=w.eps, rope_base=w.rope_base)
    err_s = np.max(np.abs(s_gpu - o.scores))
    assert err_s <= 5e-3 and err_s <= 2e-4, err_s
    diff = np.setxor1d(kept_gpu, o.kept)
    if len(diff):
        assert np.all(np.abs(o.scores[diff] - o.threshold) <= 1e-4), (diff, o.scores[diff], o.threshold)
        o = pipeline_oracle.gate_layer(h_bits, W1, gi.w2.numpy(), Wqkv, w.doc_begin, w.doc_end, w.k_doc, w.Hq,
                                       w.Hkv, w.d_h, ap.gain.numpy(), ap.tau, rows, eps=w.eps,
                                       rope_base=w.rope_base, kept_override=kept_gpu, scores=o.scores)

    # compaction: bit-exact against the oracle's gather of the same kept set with the GPU's scores (the
    # path gathers the rows inside the projection's operand loads, which the Q/K/V checks below cover;
    # the kept scores come from the select, the positions are the kept indices)
    want_h, want_pos, want_s = oracle.gather_compact(h_bits, kept_gpu, scores=s_gpu)
    if layer.h_kept is not None:
        assert np.array_equal(layer.h_kept.cpu().view(torch.int16).numpy().view(np.uint16), want_h)
    assert np.array_equal(layer.positions().cpu().numpy(), want_pos)
    assert np.array_equal(layer.s_kept[:K].cpu().numpy(), want_s)

    # Q, K, V on the sampled rows
    q_gpu = layer.q.float().cpu().numpy()
    k_gpu = layer.k.float().cpu().numpy()
    v_gpu = layer.v.float().cpu().numpy()
    Hq, Hkv, D = w.Hq, w.Hkv, w.d_h
    half = D // 2

    def check_rotated(got, want, absum):
        pair = np.sqrt(want[..., :half] ** 2 + want[..., half:] ** 2)
        pair = np.concatenate([pair, pair], axis=-1)
        bound = 2.0 ** -7 * pair + 2.0 ** -20 * 2 * absum + 1e-6
        assert np.all(np.abs(got - want) <= bound), np.max(np.abs(got - want) - bound)

    check_rotated(q_gpu[rows], o.q, o.absum_q.reshape(len(rows), Hq, D))
    absum_k = o.absum_kv[:, : Hkv * D].reshape(len(rows), Hkv, D)
    absum_v = o.absum_kv[:, Hkv * D:].reshape(len(rows), Hkv, D)
    check_rotated(k_gpu[rows], o.k[rows], absum_k)
    vb = half_ulp_bf16(o.v[rows]) + 2.0 ** -20 * absum_v + 1e-6
    assert np.all(np.abs(v_gpu[rows] - o.v[rows]) <= vb)
    if layer.v16 is not None:   # the fp16 copy of V: one rounding of the fp32 accumulator to fp16
        v16_rows = layer.v16.float().cpu().numpy().reshape(K, Hkv, D)[rows]
        assert np.all(np.abs(v16_rows - o.v[rows]) <= 2.0 ** -11 * np.abs(o.v[rows]) + 2.0 ** -20 * absum_v + 1e-6)

    got = out.float().cpu().numpy()[rows].astype(np.float64)
    assert np.all(np.isfinite(got))
    # (a) the kernel on the path's own intermediates: V as the attention reads it (fp16)
    from tests import oracle_pool
    v16_gpu = layer.v16.float().cpu().numpy().reshape(K, Hkv, D) if layer.v16 is not None else v_gpu
    want_a = oracle_pool.gated_attention(q_gpu, k_gpu, v16_gpu, s=want_s, g=ap.gain.numpy(), tau=ap.tau, rows=rows)
    ex_a = attn_excess(got, want_a)
    print(f"{name}: K={K} scores {err_s:.2e}, out vs oracle on the path's Q/K/V: raw max "
          f"{np.max(np.abs(got - want_a)):.2e}, excess {np.max(ex_a):.2e}")
    assert np.max(ex_a) <= ATTN_TOL

    # (b) against the oracle's own pipeline, with the first-order effect of the input differences
    q_or = np.zeros_like(q_gpu)
    q_or[rows] = pipeline_oracle.to_bf16(o.q)
    k_or = pipeline_oracle.to_bf16(o.k)
    v_or = pipeline_oracle.to_f16(o.v) if layer.v16 is not None else pipeline_oracle.to_bf16(o.v)
    v_gpu = v16_gpu
    s_or = o.s_kept.astype(np.float64)
    scale = ap.tau / np.sqrt(D)
    G = Hq // Hkv
    prop = np.zeros((len(rows), Hq, 1))
    for i, r in enumerate(rows):
        for hh in range(Hq):
            j = hh // G
            l_gpu = scale * (k_gpu[: r + 1, j].astype(np.float64) @ q_gpu[r, hh]) + ap.gain[hh].item() * want_s[: r + 1]
            l_or = scale * (k_or[: r + 1, j].astype(np.float64) @ q_or[r, hh]) + ap.gain[hh].item() * s_or[: r + 1]
            dl = np.max(np.abs(l_gpu - l_or))
            dv = np.max(np.abs(v_gpu[: r + 1, j] - v_or[: r + 1, j]))
            spread = np.max(np.abs(v_or[: r + 1, j] - o.out[i, hh]))
            prop[i, hh, 0] = dv + 2.0 * dl * spread
    ex_b = attn_excess(got, o.out) - prop
    print(f"{name}: out vs the oracle pipeline: raw max {np.max(np.abs(got - o.out)):.2e}, "
          f"largest propagation allowance {np.max(prop):.2e}, excess {np.max(ex_b):.2e}")
    assert np.max(ex_b) <= ATTN_TOL

"""The pruned prefill through a whole stack (learned_token_pruning_tg_b200.stack).

* Keeping every document token with zero gains and tau = 1 turns every gated
  layer into a plain one, so the pruned stack must equal the unpruned stack
  bit for bit (same kernels on the same bits; the bias step adds exact zeros).
* The kept set is the oracle's top-K of the GPU's own gate scores, bit-exact,
  and the question is always kept.
* A gated layer's attention, captured inside the stack (post-RoPE q, k, v, the
  gathered scores, the layer's gains and temperature), matches the oracle
  within the attention tolerance -- on every row of the small stack and on
  sampled rows of the 64k stack that the benchmark times.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from learned_token_pruning_tg_b200 import stack as stk
from tests import oracle_pool

pytestmark = pytest.mark.gpu

ATTN_TOL = 1e-2


def half_ulp_bf16(x):
    a = np.abs(x)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, 2.0 ** (e - 8), 0.0)


def check_captured_attention(cap, rows):
    q, k, v = (cap[n].float().cpu().numpy() for n in ("q", "k", "v"))
    want = oracle_pool.gated_attention(q, k, v, s=cap["s"].cpu().numpy(), g=cap["gain"].cpu().numpy(),
                                       tau=float(cap["tau"]), rows=rows)
    got = cap["out"].float().cpu().numpy()[rows].astype(np.float64)
    # raw error where |out| < 2 (its bf16 rounding is at most 2^-8 there), else above its half ulp
    err = np.abs(got - want)
    excess = np.where(np.abs(want) < 2.0, err, err - half_ulp_bf16(want))
    print(f"captured layer: raw max abs error {np.max(err):.3e}, max excess {np.max(excess):.3e}")
    assert np.max(excess) <= ATTN_TOL, np.max(excess)


def test_stack_all_kept_zero_gain_equals_dense():
    cfg = dataclasses.replace(stk.STACK_TINY, k_doc=stk.STACK_TINY.doc_end - stk.STACK_TINY.doc_begin)
    wts = stk.random_weights(cfg, "cuda")
    for lw in wts.layers:
        lw.gain.zero_()
        lw.tau = 1.0
    x = stk.random_embeddings(cfg, "cuda")
    s = stk.PrunedPrefillStack(cfg, wts)
    pruned = s.run(x, prune=True)
    dense = s.run(x, prune=False)
    torch.cuda.synchronize()
    assert s.device_status() == 0
    assert torch.equal(s.kept.cpu(), torch.arange(cfg.N, dtype=torch.int32))
    assert torch.equal(pruned.view(torch.int16), dense.view(torch.int16))


@pytest.mark.parametrize("cfg,rows", [(stk.STACK_TINY, None), (stk.STACK64K, "sample")])
def test_stack_select_and_gated_layer(cfg, rows):
    wts = stk.random_weights(cfg, "cuda")
    x = stk.random_embeddings(cfg, "cuda")
    s = stk.PrunedPrefillStack(cfg, wts)
    layer = cfg.gate_layer + 1 if cfg.n_layers <= 4 else cfg.n_layers - 1
    out = s.run(x, prune=True, capture=layer, keep_kv=True)
    torch.cuda.synchronize()
    # the KV cache: N keys per layer up to L, K kept keys (with their scores) above
    row = 2 * cfg.Hkv * cfg.d_h * 2
    L = cfg.gate_layer
    assert s.kv_bytes() == (L + 1) * cfg.N * row + (cfg.n_layers - L - 1) * cfg.K * (row + 4)
    assert s.device_status() == 0
    assert out.shape == (cfg.K, cfg.d) and torch.isfinite(out.float()).all()
    kept = s.kept.cpu().numpy()
    want = oracle.topk_select(s.scores.cpu().numpy(), cfg.doc_begin, cfg.doc_end, cfg.k_doc)
    assert np.array_equal(kept, want)
    assert np.all(np.isin(np.arange(cfg.doc_end, cfg.N), kept))
    K = cfg.K
    r = np.arange(K) if rows is None else np.unique(np.concatenate(
        [np.arange(0, K, 97), np.arange(K - 48, K), np.arange(0, 16)]))
    check_captured_attention(s.captured, r)

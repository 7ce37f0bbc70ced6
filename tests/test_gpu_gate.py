"""GPU parity of tg_gate_score (and gate -> select end to end) against the oracle.

Tolerances: scores max abs error <= 5e-3 (the specification's bar).  The GPU
computes the same sums in fp32 from the same bf16 inputs, so the observed error
is ~1e-6; a second, tighter bound (2e-4, derived from fp32 accumulation of d
products plus fast exp/divide in SiLU) catches precision regressions.  End to
end, a kept-set mismatch is allowed only for tokens whose oracle score lies
within 1e-4 of the oracle's K-th threshold.
"""
import numpy as np
import pytest
import torch

import oracle
from learned_token_pruning_tg_b200 import synth
from tests import oracle_pool
from learned_token_pruning_tg_b200 import tokengate as tg

pytestmark = pytest.mark.gpu

SPEC_TOL = 5e-3
TIGHT_TOL = 2e-4


def _gpu_scores(gi, eps=1e-6):
    h = gi.h.to(torch.bfloat16).cuda()
    W1 = gi.W1.to(torch.bfloat16).cuda()
    N, d = h.shape
    d_g = W1.shape[0]
    scores = torch.full((N,), float("nan"), device="cuda")
    ws = tg.new_workspace(N, d, d_g)
    tg.tg_gate_score(h, W1, gi.w2.cuda(), scores, ws,
                     b1=None if gi.b1 is None else gi.b1.cuda(), b2=gi.b2,
                     rms_weight=None if gi.gamma is None else gi.gamma.to(torch.bfloat16).cuda(), eps=eps)
    torch.cuda.synchronize()
    assert tg.tg_device_status(ws) == 0
    return scores.cpu().numpy()


def _oracle_scores(gi, rows=None, eps=1e-6):
    h = gi.h.to(torch.bfloat16).float().numpy()
    if rows is not None:
        h = h[rows]
    return oracle.gate_score(h, gi.W1.to(torch.bfloat16).float().numpy(), gi.w2.numpy(),
                             b1=None if gi.b1 is None else gi.b1.numpy(), b2=gi.b2,
                             gamma=None if gi.gamma is None else gi.gamma.to(torch.bfloat16).float().numpy(),
                             eps=eps, fold_gamma_bf16=True)


def _check(got, want):
    err = np.max(np.abs(got.astype(np.float64) - want))
    assert np.all(np.isfinite(got))
    assert err <= SPEC_TOL, err
    assert err <= TIGHT_TOL, err
    return err


@pytest.mark.parametrize("w", [synth.TINY, synth.L16K], ids=lambda w: w.name)
def test_gate_full_workloads(w):
    gi = synth.gate_inputs(w)
    _check(_gpu_scores(gi), _oracle_scores(gi))


@pytest.mark.parametrize("N,d,d_g,bias,gamma", [
    (1, 64, 64, False, False),        # single row, single K stage
    (127, 128, 128, True, False),     # one ragged tile
    (1000, 512, 256, True, True),     # ragged tail, bias and RMSNorm weight
    (4099, 2048, 256, False, True),   # many tiles, tail of 3 rows
    (20000, 1024, 64, True, False),   # more tiles than SMs, narrow gate
    (300, 8192, 128, False, False),   # long K loop
    # d_g = 256 runs on CTA pairs (256-row tiles shared by two CTAs): a pair with one row, a pair
    # whose second CTA has no rows, a tail of one row past a pair, a long K loop
    (1, 64, 256, False, False),
    (129, 128, 256, True, False),
    (257, 256, 256, False, False),
    (300, 8192, 256, True, True),
])
def test_gate_shapes(N, d, d_g, bias, gamma):
    w = synth.scaled(synth.L16K, N=N, doc_end=N, d=d, d_g=d_g, n_scaled=min(8, N), seed=N + d)
    gi = synth.gate_inputs(w, with_bias=bias, with_gamma=gamma)
    _check(_gpu_scores(gi), _oracle_scores(gi))


def test_gate_128k_sampled_rows():
    # Full 128k workload in the launch configuration the benchmark times; the oracle
    # checks a sample of rows (every scaled row's neighbourhood plus a stride).
    w = synth.L128K
    gi = synth.gate_inputs(w)
    got = _gpu_scores(gi)
    rows = np.unique(np.concatenate([np.arange(0, w.N, 97), gi.scaled_rows[:200].numpy(),
                                     np.arange(w.N - 130, w.N)]))
    _check(got[rows], _oracle_scores(gi, rows=rows))
    # RMSNorm cancels row scale: the x3 rows must not stand out in score distribution
    assert abs(np.std(got[gi.scaled_rows.numpy()]) - np.std(got)) < 0.1


@pytest.mark.parametrize("w", [synth.TINY, synth.L16K, synth.L128K], ids=lambda w: w.name)
def test_gate_then_select_end_to_end(w):
    gi = synth.gate_inputs(w)
    g = _gpu_scores(gi)
    # bit-exact select on the GPU's own scores
    s_gpu = torch.from_numpy(g).cuda()
    K = w.K
    kept = torch.empty(K, dtype=torch.int32, device="cuda")
    ws = tg.new_workspace(w.N)
    tg.tg_topk_select(s_gpu, w.doc_begin, w.doc_end, w.k_doc, kept, ws)
    torch.cuda.synchronize()
    kept = kept.cpu().numpy()
    assert np.array_equal(kept, oracle.topk_select(g, w.doc_begin, w.doc_end, w.k_doc))
    # against the oracle's own scores: mismatches only within 1e-4 of the threshold
    o = oracle_pool.gate_scores(gi.h.to(torch.bfloat16).float().numpy(), gi.W1.to(torch.bfloat16).float().numpy(),
                                gi.w2.numpy())
    o32 = o.astype(np.float32)
    want = oracle.topk_select(o32, w.doc_begin, w.doc_end, w.k_doc)
    thr = oracle.topk_threshold(o32, w.doc_begin, w.doc_end, w.k_doc)
    diff = np.setxor1d(kept, want)
    assert np.all(np.abs(o[diff] - thr) <= 1e-4), (len(diff), np.max(np.abs(o[diff] - thr)))
    # question tokens are always kept
    assert np.all(np.isin(np.arange(w.doc_end, w.N), kept))


def test_gate_repeatable_bit_exact():
    # Races between the TMA producer and the threads reading its stages show up as run-to-run
    # differences: the same launch repeated must give bit-identical scores.
    w = synth.L16K
    gi = synth.gate_inputs(w)
    first = _gpu_scores(gi)
    for _ in range(7):
        assert np.array_equal(_gpu_scores(gi), first)
    _check(first, _oracle_scores(gi))


@pytest.mark.parametrize("N,d,d_g,db,de,k", [
    (1024, 256, 64, 0, 960, 192),              # tiny workload's shape
    (16384, 2048, 256, 0, 16000, 1024),        # 16k (CTA-pair gate, one-cluster select)
    (131072, 2048, 256, 0, 130560, 4096),      # 128k
    (70001, 512, 128, 333, 69000, 12345),      # ragged span inside the prompt
    (300000, 64, 256, 1000, 299000, 50000),    # a span beyond one cluster: the cooperative select
    (5000, 128, 64, 0, 5000, 0),               # budget 0: nothing selected, the count still cleared
    (5000, 128, 64, 100, 4900, 10000),         # budget above the span: every token kept
])
def test_gate_and_select_pair(N, d, d_g, db, de, k):
    # tg_gate_score_for_select gives tg_gate_score's scores bit for bit and leaves the select's first
    # radix pass in the workspace; tg_topk_select_after_gate then gives the oracle's selection on those
    # scores and leaves the count at zero (three pairs in a row on one workspace).
    w = synth.scaled(synth.L16K, N=N, doc_begin=db, doc_end=de, d=d, d_g=d_g, k_doc=k, n_scaled=min(8, de - db),
                     seed=N + d_g)
    gi = synth.gate_inputs(w)
    h, W1, w2 = gi.h.to(torch.bfloat16).cuda(), gi.W1.to(torch.bfloat16).cuda(), gi.w2.cuda()
    ws = tg.new_workspace(N, d, d_g)
    plain = torch.empty(N, device="cuda")
    tg.tg_gate_score(h, W1, w2, plain, ws)
    K = tg.tg_kept_count(N, db, de, k)
    for it in range(3):
        scores = torch.full((N,), float("nan"), device="cuda")
        kept = torch.full((max(K, 1),), -1, dtype=torch.int32, device="cuda")
        s_kept = torch.full((max(K, 1),), float("nan"), device="cuda")
        tg.tg_gate_score_for_select(h, W1, w2, scores, ws, db, de)
        if it == 1:  # the variant that also writes the kept tokens' scores
            tg.tg_topk_select_after_gate_kept_scores(scores, db, de, k, kept[:K], s_kept[:K], ws)
        else:
            tg.tg_topk_select_after_gate(scores, db, de, k, kept[:K], ws)
        torch.cuda.synchronize()
        assert tg.tg_device_status(ws) == 0
        assert torch.equal(scores.view(torch.int32), plain.view(torch.int32))
        s_np = scores.cpu().numpy()
        kept_np = kept[:K].cpu().numpy()
        assert np.array_equal(kept_np, oracle.topk_select(s_np, db, de, k))
        if it == 1:
            assert np.array_equal(s_kept[:K].cpu().numpy().view(np.int32), s_np[kept_np].view(np.int32))
        # the first-pass count (2048 words after the status header and the barrier words) is zero again
        hist0 = ws[256 + 256: 256 + 256 + 2048 * 4].view(torch.int32)
        assert int(hist0.abs().sum().item()) == 0


@pytest.mark.parametrize("N,d,bias,gamma", [(129, 128, True, False), (4099, 2048, False, True), (300, 8192, True, True)])
def test_gate_one_cta_kernel_d_g_256(N, d, bias, gamma):
    # d_g = 256 on the one-CTA kernel (taken where a device offers no clusters of 2)
    tg.tg_debug_set_cta_pairs(False)
    try:
        w = synth.scaled(synth.L16K, N=N, doc_end=N, d=d, d_g=256, n_scaled=min(8, N), seed=N + d + 7)
        gi = synth.gate_inputs(w, with_bias=bias, with_gamma=gamma)
        _check(_gpu_scores(gi), _oracle_scores(gi))
    finally:
        tg.tg_debug_set_cta_pairs(True)

"""GPU parity of tg_topk_select, tg_gather_compact and tg_rope_apply against the oracle.

Select and gather are integer/index work: bit-exact.  RoPE rounds to bf16:
within one bf16 rounding of the oracle's fp64 result (plus fp32 arithmetic).
"""
import numpy as np
import pytest
import torch

import oracle
from learned_token_pruning_tg_b200 import synth
from learned_token_pruning_tg_b200 import tokengate as tg
from tests.guards import guarded

pytestmark = pytest.mark.gpu


def _select_gpu(s_cpu, db, de, k, ws=None):
    s = s_cpu.cuda()
    N = s.shape[0]
    K = tg.tg_kept_count(N, db, de, k)
    out = torch.full((max(K, 1),), -7, dtype=torch.int32, device="cuda")
    ws = ws if ws is not None else tg.new_workspace(N)
    tg.tg_topk_select(s, db, de, k, out, ws)
    torch.cuda.synchronize()
    assert tg.tg_device_status(ws) == 0
    return out[:K].cpu().numpy()


SELECT_CASES = [
    # N, doc_begin, doc_end, k_doc, kind, seed
    (1024, 0, 960, 192, "normal", 0),
    (16384, 0, 16000, 1024, "normal", 16),
    (32768, 0, 32256, 512, "heavy", 3201),
    (32768, 0, 32256, 16384, "ties", 3204),
    (131072, 0, 130560, 4096, "heavy", 128),
    (131072, 0, 130560, 4096, "ties", 129),
    (131072, 0, 130560, 4096, "special", 130),
    (131072, 512, 131072, 4096, "normal", 131),     # question first, document last
    (70001, 333, 69000, 12345, "special", 5),       # ragged everywhere
    (5000, 0, 5000, 2500, "const", 6),              # every score equal: index order decides
    (300000, 1000, 299000, 100000, "ties", 7),      # two keys per thread
    (2000000, 0, 1999000, 65536, "heavy", 8),       # many keys per thread
    (3, 0, 2, 1, "normal", 9),
    (262656, 0, 262144, 30000, "heavy", 10),      # the one-cluster shape's longest span (16 keys per thread)
    (262657, 0, 262145, 30000, "normal", 12),     # one key more: the cooperative shape
]


@pytest.mark.parametrize("N,db,de,k,kind,seed", SELECT_CASES)
def test_select_bit_exact(N, db, de, k, kind, seed):
    s = synth.score_vector(N, seed, kind)
    got = _select_gpu(s, db, de, k)
    want = oracle.topk_select(s.numpy(), db, de, k)
    assert got.shape == want.shape
    assert np.array_equal(got, want)


@pytest.mark.parametrize("k", [0, 1, 959, 960, 5000])
def test_select_budget_edges(k):
    s = synth.score_vector(1024, 11, "normal")
    assert np.array_equal(_select_gpu(s, 0, 960, k), oracle.topk_select(s.numpy(), 0, 960, k))


def test_select_empty_span_and_repeat_calls():
    s = synth.score_vector(4096, 12, "ties")
    assert np.array_equal(_select_gpu(s, 100, 100, 5), np.arange(4096))
    ws = tg.new_workspace(4096)
    for k in (3, 700, 2000, 3):          # the workspace is reused; histograms must self-clean
        assert np.array_equal(_select_gpu(s, 10, 4000, k, ws), oracle.topk_select(s.numpy(), 10, 4000, k))


@pytest.mark.parametrize("N,d,K,ld_pad", [(1024, 256, 256, 0), (16384, 2048, 1408, 0), (5000, 2048, 777, 64),
                                          (300, 136, 299, 8), (4096, 4096, 100, 0),
                                          (131072, 2048, 4608, 0),   # the 128k workload's kept set (bulk copies)
                                          (100, 2048, 33, 0),        # one row past a 32-row block
                                          (40, 16384, 9, 0),         # 32 KB rows: the 16-byte-vector copy
                                          (10, 64, 1, 0)])
def test_gather_bit_exact(N, d, K, ld_pad):
    g = torch.Generator().manual_seed(N + d)
    h_full = torch.randn(N, d + ld_pad, generator=g).to(torch.bfloat16)
    idx = torch.sort(torch.randperm(N, generator=g)[:K]).values.to(torch.int32)
    pos_in = (torch.arange(N, dtype=torch.int32) * 3 + 1)
    s = torch.randn(N, generator=g)
    hd = h_full.cuda()[:, :d]
    h_out, check_h = guarded((K, d), torch.bfloat16)      # guard bands around every output
    pos_out, check_p = guarded((K,), torch.int32)
    s_out, check_s = guarded((K,), torch.float32)
    tg.tg_gather_compact(hd, idx.cuda(), h_out, pos_out, pos_in=pos_in.cuda(), scores=s.cuda(), s_out=s_out)
    torch.cuda.synchronize()
    check_h(), check_p(), check_s()
    bits = h_full[:, :d].contiguous().view(torch.int16).numpy().view(np.uint16)
    want_h, want_pos, want_s = oracle.gather_compact(bits, idx.numpy(), pos_in=pos_in.numpy(), scores=s.numpy())
    assert np.array_equal(h_out.cpu().view(torch.int16).numpy().view(np.uint16), want_h)
    assert np.array_equal(pos_out.cpu().numpy(), want_pos)
    assert np.array_equal(s_out.cpu().numpy().view(np.uint32), want_s.view(np.uint32))
    # without pos_in the positions are the kept indices themselves
    tg.tg_gather_compact(hd, idx.cuda(), h_out, pos_out)
    torch.cuda.synchronize()
    assert np.array_equal(pos_out.cpu().numpy(), idx.numpy())


@pytest.mark.parametrize("d", [2048, 16384])
def test_gather_rejects_out_of_range_indices_without_reading(d):
    # A kept index outside [0, N) is not read: its row comes out zero, its position -1 and its score
    # NaN; every other row is copied exactly.  (The indices are only checked, never dereferenced, so
    # nothing here reads outside h.)
    N, K = 64, 12
    g = torch.Generator().manual_seed(d)
    h = torch.randn(N, d, generator=g).to(torch.bfloat16)
    s = torch.randn(N, generator=g)
    idx = torch.tensor([0, 3, N, 5, -1, 9, 2 ** 31 - 1, 20, 21, -(2 ** 31), 40, N - 1], dtype=torch.int32)
    h_out, check_h = guarded((K, d), torch.bfloat16)
    pos_out, check_p = guarded((K,), torch.int32)
    s_out, check_s = guarded((K,), torch.float32)
    h_out.fill_(7.0)
    tg.tg_gather_compact(h.cuda(), idx.cuda(), h_out, pos_out, scores=s.cuda(), s_out=s_out)
    torch.cuda.synchronize()
    check_h(), check_p(), check_s()
    bad = (idx < 0) | (idx >= N)
    got_h, got_p, got_s = h_out.cpu(), pos_out.cpu(), s_out.cpu()
    assert torch.equal(got_p[bad], torch.full((int(bad.sum()),), -1, dtype=torch.int32))
    assert torch.all(torch.isnan(got_s[bad])) and torch.all(got_h[bad] == 0)
    good = ~bad
    assert torch.equal(got_p[good], idx[good])
    assert torch.equal(got_h[good].view(torch.int16), h[idx[good].long()].view(torch.int16))
    assert torch.equal(got_s[good], s[idx[good].long()])


@pytest.mark.parametrize("K,Hq,Hkv,d_h,max_pos", [(256, 4, 2, 64, 1024), (1408, 16, 8, 128, 16384),
                                                  (4608, 16, 8, 128, 131072), (33, 2, 1, 128, 140000)])
def test_rope_against_oracle(K, Hq, Hkv, d_h, max_pos):
    g = torch.Generator().manual_seed(K)
    qkv = torch.randn(K, (Hq + 2 * Hkv) * d_h, generator=g).to(torch.bfloat16)
    pos = torch.sort(torch.randperm(max_pos, generator=g)[:K]).values.to(torch.int32)
    d = qkv.cuda()
    q = d[:, : Hq * d_h].view(K, Hq, d_h)
    k = d[:, Hq * d_h: (Hq + Hkv) * d_h].view(K, Hkv, d_h)
    v_before = d[:, (Hq + Hkv) * d_h:].clone()
    tg.tg_rope_apply(q, k, pos.cuda(), 1e6)
    torch.cuda.synchronize()
    q_ref = oracle.rope(qkv[:, : Hq * d_h].view(K, Hq, d_h).float().numpy(), pos.numpy(), 1e6)
    k_ref = oracle.rope(qkv[:, Hq * d_h:(Hq + Hkv) * d_h].view(K, Hkv, d_h).float().numpy(), pos.numpy(), 1e6)
    for got, ref in ((q, q_ref), (k, k_ref)):
        got = got.float().cpu().numpy().astype(np.float64)
        # one bf16 rounding (half an ulp: 2^-8 relative) plus fp32 arithmetic
        tol = np.abs(ref) * (2.0 ** -8 + 1e-6) + 1e-6
        assert np.all(np.abs(got - ref) <= tol), np.max(np.abs(got - ref) - tol)
    assert torch.equal(d[:, (Hq + Hkv) * d_h:], v_before)          # v untouched


@pytest.mark.parametrize("N,db,de,k", [(131072, 0, 130560, 4096), (300000, 1000, 299000, 100000)])
def test_select_repeatable(N, db, de, k):
    s = synth.score_vector(N, 21, "ties")
    ws = tg.new_workspace(N)
    first = _select_gpu(s, db, de, k, ws)
    for _ in range(5):
        assert np.array_equal(_select_gpu(s, db, de, k, ws), first)
    assert np.array_equal(first, oracle.topk_select(s.numpy(), db, de, k))

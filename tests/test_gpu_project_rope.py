"""GPU parity of tg_project_rope (the kept rows' Q/K/V projection with RoPE and V's fp16 copy in the
GEMM epilogue) against the oracle: the projection in fp64 (numpy) followed by the oracle's rotation.

Tolerance: the kernel rotates the fp32 accumulators and rounds once to bf16, so every element is
within half a bf16 ulp of the exact value plus fp32 accumulation over d products and fp32 cos / sin
(2^-20 of the sum of absolute terms bounds both here); the fp16 copy of V is the same accumulator
rounded to fp16 (half an fp16 ulp, 2^-11 relative, plus the same accumulation bound).
"""
import numpy as np
import pytest
import torch

import oracle
from learned_token_pruning_tg_b200 import tokengate as tg
from tests.guards import guarded

pytestmark = pytest.mark.gpu


def half_ulp_bf16(x):
    a = np.abs(x)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, 2.0 ** (e - 8), 0.0)


def run(K, d, Hq, Hkv, d_h, seed, rows=None):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(K, d, generator=g).to(torch.bfloat16)
    W = (torch.randn((Hq + 2 * Hkv) * d_h, d, generator=g) / d ** 0.5).to(torch.bfloat16)
    pos = torch.sort(torch.randperm(4 * K, generator=g)[:K]).values.to(torch.int32)
    cols = (Hq + 2 * Hkv) * d_h
    qkv, cq = guarded((K, cols), torch.bfloat16)
    v16, cv = guarded((K, Hkv * d_h), torch.float16)
    qkv.fill_(float("nan"))
    v16.fill_(float("nan"))
    ws = tg.new_workspace(K, d_h, op=tg.TG_OP_PROJECT)
    tg.tg_project_rope(x.cuda(), W.cuda(), pos.cuda(), qkv, ws, Hq, Hkv, d_h, base=1e6, v16=v16)
    torch.cuda.synchronize()
    cq(), cv()
    assert tg.tg_device_status(ws) == 0
    r = np.arange(K) if rows is None else np.asarray(rows)
    xf, Wf = x.float().numpy().astype(np.float64), W.float().numpy().astype(np.float64)
    proj = xf[r] @ Wf.T                                               # [rows, cols]
    absum = np.abs(xf[r]) @ np.abs(Wf).T
    q = proj[:, : Hq * d_h].reshape(len(r), Hq, d_h)
    k = proj[:, Hq * d_h: (Hq + Hkv) * d_h].reshape(len(r), Hkv, d_h)
    want = proj.copy()
    want[:, : Hq * d_h] = oracle.rope(q.astype(np.float32), pos.numpy()[r], 1e6).reshape(len(r), -1)
    want[:, Hq * d_h: (Hq + Hkv) * d_h] = oracle.rope(k.astype(np.float32), pos.numpy()[r], 1e6).reshape(len(r), -1)
    got = qkv.float().cpu().numpy()[r]
    return got, want, absum, v16.float().cpu().numpy()[r], Hq, Hkv, d_h


@pytest.mark.parametrize("K,d,Hq,Hkv,d_h", [(300, 256, 4, 2, 128), (129, 512, 4, 2, 64), (4608, 2048, 16, 8, 128)])
def test_project_rope_matches_oracle(K, d, Hq, Hkv, d_h):
    rows = None if K <= 1000 else np.unique(np.concatenate([np.arange(0, K, 37), np.arange(K - 40, K)]))
    got, want, absum, v16, Hq, Hkv, d_h = run(K, d, Hq, Hkv, d_h, seed=K + d, rows=rows)
    assert np.all(np.isfinite(got))
    # the oracle rotates fp32-rounded projections; that rounding and fp32 accumulation are both
    # covered by 2^-20 of the absolute sum (the rotation mixes two elements of equal scale)
    bound = half_ulp_bf16(want) + 2.0 ** -20 * 2 * absum + 1e-6
    assert np.all(np.abs(got - want) <= bound)
    vcols = slice((Hq + Hkv) * d_h, None)
    wv = want[:, vcols]
    assert np.all(np.abs(v16 - wv) <= 2.0 ** -11 * np.abs(wv) + 2.0 ** -20 * 2 * absum[:, vcols] + 1e-6)


@pytest.mark.parametrize("N,K,d,Hq,Hkv,d_h,bad", [
    (1000, 300, 256, 4, 2, 128, None),        # ragged K, repeated rows
    (5000, 129, 512, 4, 2, 64, None),         # d_h = 64, K not a multiple of 4
    (131072, 4608, 2048, 16, 8, 128, None),   # the 128k workload's kept set
    (1000, 300, 256, 4, 2, 128, 77),          # one index outside [0, N)
])
def test_project_rope_gather_matches_dense(N, K, d, Hq, Hkv, d_h, bad):
    # tg_project_rope_gather (rows gathered from h by TMA gather4 copies into the operand tiles) gives
    # tg_project_rope on the compacted rows bit for bit; that one is checked against the oracle above.
    # An index outside [0, N) is not followed: row 0 is read in its place and the status flags it.
    g = torch.Generator().manual_seed(N + K)
    h = torch.randn(N, d, generator=g).to(torch.bfloat16)
    W = (torch.randn((Hq + 2 * Hkv) * d_h, d, generator=g) / d ** 0.5).to(torch.bfloat16)
    rows = torch.randint(0, N, (K,), generator=g).to(torch.int32)
    if bad is not None:
        rows[bad] = N
    cols = (Hq + 2 * Hkv) * d_h
    x = h[torch.where(rows < N, rows, torch.zeros_like(rows)).long()].contiguous()
    outs = []
    for gather in (True, False):
        qkv, cq = guarded((K, cols), torch.bfloat16)
        v16, cv = guarded((K, Hkv * d_h), torch.float16)
        qkv.fill_(float("nan"))
        v16.fill_(float("nan"))
        ws = tg.new_workspace(K, d_h, op=tg.TG_OP_PROJECT)
        if gather:
            tg.tg_project_rope_gather(h.cuda(), rows.cuda(), W.cuda(), rows.cuda(), qkv, ws, Hq, Hkv, d_h, base=1e6,
                                      v16=v16)
        else:
            tg.tg_project_rope(x.cuda(), W.cuda(), rows.cuda(), qkv, ws, Hq, Hkv, d_h, base=1e6, v16=v16)
        torch.cuda.synchronize()
        cq(), cv()
        status = tg.tg_device_status(ws)
        if gather and bad is not None:
            assert status == tg.TG_STATUS_INDEX_RANGE
        else:
            assert status == 0
        outs.append((qkv.cpu(), v16.cpu()))
    assert torch.equal(outs[0][0].view(torch.int16), outs[1][0].view(torch.int16))
    assert torch.equal(outs[0][1].view(torch.int16), outs[1][1].view(torch.int16))


@pytest.fixture
def one_cta_kernels():
    # the one-CTA projection kernel (taken where a device offers no clusters of 2)
    tg.tg_debug_set_cta_pairs(False)
    yield
    tg.tg_debug_set_cta_pairs(True)


@pytest.mark.parametrize("K,d,Hq,Hkv,d_h", [(300, 256, 4, 2, 128), (4608, 2048, 16, 8, 128)])
def test_project_rope_one_cta_kernel(one_cta_kernels, K, d, Hq, Hkv, d_h):
    rows = None if K <= 1000 else np.unique(np.concatenate([np.arange(0, K, 37), np.arange(K - 40, K)]))
    got, want, absum, v16, Hq, Hkv, d_h = run(K, d, Hq, Hkv, d_h, seed=K + d + 1, rows=rows)
    assert np.all(np.isfinite(got))
    assert np.all(np.abs(got - want) <= half_ulp_bf16(want) + 2.0 ** -20 * 2 * absum + 1e-6)
    wv = want[:, (Hq + Hkv) * d_h:]
    assert np.all(np.abs(v16 - wv) <= 2.0 ** -11 * np.abs(wv) + 2.0 ** -20 * 2 * absum[:, (Hq + Hkv) * d_h:] + 1e-6)


@pytest.mark.parametrize("N,K,d,Hq,Hkv,d_h,bad", [(1000, 300, 256, 4, 2, 128, None), (5000, 129, 512, 4, 2, 64, 5)])
def test_project_rope_gather_one_cta_kernel(one_cta_kernels, N, K, d, Hq, Hkv, d_h, bad):
    test_project_rope_gather_matches_dense(N, K, d, Hq, Hkv, d_h, bad)

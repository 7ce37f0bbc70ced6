"""Pins of the oracle's token-gated attention, RoPE and gather.

Token-gated attention (TokenGate pages: kept-token score as a bias on the
attention logits above the gate, a learned per-head gain and a learned
temperature: aiproducthub.cn article, paragraph 事件详情; aisight.pl article,
section Jak to działa; chathome.org article, section トークンゲート付き
アテンションとは); the formula
l = tau q.k / sqrt(d_h) + g_h s_c is the specification's.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle


def _inputs(K, Hq, Hkv, d_h, seed, bf16=True):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(K, Hq, d_h, generator=g)
    k = torch.randn(K, Hkv, d_h, generator=g)
    v = torch.randn(K, Hkv, d_h, generator=g)
    if bf16:
        q, k, v = (t.bfloat16().float() for t in (q, k, v))
    s = torch.randn(K, generator=g) * 0.7
    gain = torch.rand(Hq, generator=g) * 2
    return q.numpy(), k.numpy(), v.numpy(), s.numpy(), gain.numpy()


def _sdpa(q, k, v, bias, scale):
    """torch's scaled_dot_product_attention in fp64 with an additive float mask."""
    Hq, Hkv = q.shape[1], k.shape[1]
    tq = torch.from_numpy(q).double().transpose(0, 1)                 # [Hq, K, d]
    tk = torch.from_numpy(k).double().transpose(0, 1).repeat_interleave(Hq // Hkv, 0)
    tv = torch.from_numpy(v).double().transpose(0, 1).repeat_interleave(Hq // Hkv, 0)
    out = F.scaled_dot_product_attention(tq, tk, tv, attn_mask=bias, scale=scale)
    return out.transpose(0, 1).numpy()                                # [K, Hq, d]


def test_plain_causal_when_k_eq_n_g0_tau1():
    q, k, v, s, _ = _inputs(70, 4, 2, 32, 0)
    ours = oracle.gated_attention(q, k, v, s=s, g=np.zeros(4, np.float32), tau=1.0)
    tq = torch.from_numpy(q).double().transpose(0, 1)
    tk = torch.from_numpy(k).double().transpose(0, 1).repeat_interleave(2, 0)
    tv = torch.from_numpy(v).double().transpose(0, 1).repeat_interleave(2, 0)
    ref = F.scaled_dot_product_attention(tq, tk, tv, is_causal=True).transpose(0, 1).numpy()
    assert np.max(np.abs(ours - ref)) < 1e-12


@pytest.mark.parametrize("Hq,Hkv,d_h", [(4, 2, 64), (6, 3, 16), (4, 4, 8)])
def test_gated_vs_library_sdpa_with_bias(Hq, Hkv, d_h):
    K = 53
    q, k, v, s, gain = _inputs(K, Hq, Hkv, d_h, Hq * 100 + d_h)
    tau = 1.37
    ours, lse = oracle.gated_attention(q, k, v, s=s, g=gain, tau=tau, want_lse=True)
    causal = torch.ones(K, K, dtype=torch.bool).tril()
    bias = torch.from_numpy(gain).double()[:, None, None] * torch.from_numpy(s).double()[None, None, :]
    bias = bias.expand(Hq, K, K).masked_fill(~causal, float("-inf"))
    ref = _sdpa(q, k, v, bias, tau / math.sqrt(d_h))
    assert np.max(np.abs(ours - ref)) < 1e-12
    # log-sum-exp of the logits, from the library
    tq = torch.from_numpy(q).double().transpose(0, 1)
    tk = torch.from_numpy(k).double().transpose(0, 1).repeat_interleave(Hq // Hkv, 0)
    logits = tq @ tk.transpose(1, 2) * (tau / math.sqrt(d_h)) + bias
    ref_lse = torch.logsumexp(logits, dim=-1).transpose(0, 1).numpy()   # [K, Hq]
    assert np.max(np.abs(lse - ref_lse)) < 1e-11


def test_augmented_dimension_identity():
    # tau q.k/sqrt(d) + g s  ==  q~ . k~  with q~ = [tau q/sqrt(d), g], k~ = [k, s]:
    # plain attention (g = 0) at scale 1 on d+1 dimensions gives the same output.
    K, Hq, Hkv, d = 41, 4, 2, 16
    q, k, v, s, gain = _inputs(K, Hq, Hkv, d, 11, bf16=False)
    tau = 0.9
    ours = oracle.gated_attention(q, k, v, s=s, g=gain, tau=tau)
    qa = np.concatenate([q * tau / math.sqrt(d), np.broadcast_to(gain[None, :, None], (K, Hq, 1))], -1)
    ka = np.concatenate([k, np.broadcast_to(s[:, None, None], (K, Hkv, 1))], -1)
    # d+1 = 17 dims: scale tau'/sqrt(17) = 1 needs tau' = sqrt(17); values padded with a zero column
    va = np.concatenate([v, np.zeros((K, Hkv, 1), np.float32)], -1)
    aug = oracle.gated_attention(qa.astype(np.float32), ka.astype(np.float32), va, tau=math.sqrt(d + 1))
    # qa was rounded to fp32 on the way in, so compare at fp32-input accuracy
    assert np.max(np.abs(ours - aug[..., :d])) < 1e-5


def test_constant_score_cancels():
    K, Hq, Hkv, d = 30, 2, 1, 8
    q, k, v, _, gain = _inputs(K, Hq, Hkv, d, 12)
    const = np.full(K, 0.8, np.float32)
    a = oracle.gated_attention(q, k, v, s=const, g=gain, tau=1.1)
    b = oracle.gated_attention(q, k, v, s=None, g=None, tau=1.1)
    assert np.max(np.abs(a - b)) < 1e-12


def test_first_row_is_first_value_and_dominant_key():
    K, Hq, Hkv, d = 25, 2, 1, 8
    q, k, v, s, _ = _inputs(K, Hq, Hkv, d, 13)
    out = oracle.gated_attention(q, k, v, s=s, g=np.ones(Hq, np.float32), tau=1.0)
    assert np.array_equal(out[0, 0], v[0, 0].astype(np.float64))
    # one key with a huge score and a large gain dominates every later row
    s2 = s.copy()
    s2[7] = 1.0e3
    out = oracle.gated_attention(q, k, v, s=s2, g=np.full(Hq, 5.0, np.float32), tau=1.0)
    for r in range(7, K):
        assert np.max(np.abs(out[r] - v[7, 0][None, :])) < 1e-12


def test_gqa_equals_duplicated_heads():
    K, Hq, Hkv, d = 33, 4, 2, 16
    q, k, v, s, gain = _inputs(K, Hq, Hkv, d, 14)
    a = oracle.gated_attention(q, k, v, s=s, g=gain, tau=1.2)
    kd = np.repeat(k, 2, axis=1)
    vd = np.repeat(v, 2, axis=1)
    b = oracle.gated_attention(q, kd, vd, s=s, g=gain, tau=1.2)
    assert np.array_equal(a, b)


def test_rows_subset_and_positions():
    K, Hq, Hkv, d = 40, 2, 2, 8
    q, k, v, s, gain = _inputs(K, Hq, Hkv, d, 15)
    full = oracle.gated_attention(q, k, v, s=s, g=gain, tau=1.0)
    rows = np.array([39, 0, 17])
    sub = oracle.gated_attention(q, k, v, s=s, g=gain, tau=1.0, rows=rows)
    assert np.array_equal(sub, full[rows])
    # ascending original positions give the same causality as compacted indices
    pos = np.sort(np.random.default_rng(0).choice(1000, K, replace=False)).astype(np.int32)
    withpos = oracle.gated_attention(q, k, v, s=s, g=gain, tau=1.0, pos=pos)
    assert np.array_equal(withpos, full)


def test_pruned_tokens_contribute_nothing():
    # Full-length attention where the pruned keys are masked out, restricted to the
    # kept query rows, equals attention over the compacted kept set.
    N, Hq, Hkv, d = 60, 2, 1, 8
    q, k, v, s, gain = _inputs(N, Hq, Hkv, d, 16)
    kept = oracle.topk_select(s, 0, 50, 20)
    compact = oracle.gated_attention(q[kept], k[kept], v[kept], s=s[kept], g=gain, tau=1.3,
                                     pos=kept.astype(np.int32))
    keep_mask = np.zeros(N, bool)
    keep_mask[kept] = True
    causal = torch.ones(N, N, dtype=torch.bool).tril() & torch.from_numpy(keep_mask)[None, :]
    bias = torch.from_numpy(gain).double()[:, None, None] * torch.from_numpy(s).double()[None, None, :]
    bias = bias.expand(Hq, N, N).masked_fill(~causal, float("-inf"))
    ref = _sdpa(q, k, v, bias, 1.3 / math.sqrt(d))[kept]
    assert np.max(np.abs(compact - ref)) < 1e-12
    # perturbing the pruned rows changes nothing in the compacted computation
    q2, k2, v2 = q.copy(), k.copy(), v.copy()
    pruned = np.setdiff1d(np.arange(N), kept)
    q2[pruned] += 5
    k2[pruned] -= 3
    v2[pruned] *= 7
    again = oracle.gated_attention(q2[kept], k2[kept], v2[kept], s=s[kept], g=gain, tau=1.3,
                                   pos=kept.astype(np.int32))
    assert np.array_equal(again, compact)


# ---------------------------------------------------------------- RoPE
def test_rope_identity_norm_and_relative():
    rng = np.random.default_rng(20)
    K, H, d = 16, 3, 64
    x = rng.standard_normal((K, H, d)).astype(np.float32)
    out0 = oracle.rope(x, np.zeros(K, np.int32))
    assert np.array_equal(out0, x.astype(np.float64))
    pos = rng.integers(0, 131072, K).astype(np.int32)
    out = oracle.rope(x, pos)
    half = d // 2
    n_in = x[..., :half].astype(np.float64) ** 2 + x[..., half:].astype(np.float64) ** 2
    n_out = out[..., :half] ** 2 + out[..., half:] ** 2
    assert np.max(np.abs(n_in - n_out)) < 1e-10
    # <R(m) a, R(n) b> depends only on m - n
    a = np.broadcast_to(x[0:1], (4, H, d)).copy()
    b = np.broadcast_to(x[1:2], (4, H, d)).copy()
    m = np.array([5, 105, 70005, 131000], np.int32)
    n = m - 3
    dots = np.sum(oracle.rope(a, m) * oracle.rope(b, n), axis=-1)
    assert np.max(np.abs(dots - dots[0:1])) < 1e-9


def test_rope_vs_complex_rotation():
    # Rotate-half pairs (t, t + d/2) as the complex number x_t + i x_{t+d/2},
    # multiplied by exp(i pos base^(-2t/d)) with numpy's complex arithmetic.
    rng = np.random.default_rng(21)
    K, H, d, base = 12, 2, 128, 1e6
    x = rng.standard_normal((K, H, d)).astype(np.float32)
    pos = rng.integers(0, 140000, K).astype(np.int32)
    z = x[..., : d // 2].astype(np.float64) + 1j * x[..., d // 2:].astype(np.float64)
    ang = pos[:, None].astype(np.float64) * base ** (-2.0 * np.arange(d // 2) / d)
    zr = z * np.exp(1j * ang)[:, None, :]
    ref = np.concatenate([zr.real, zr.imag], -1)
    assert np.max(np.abs(oracle.rope(x, pos, base) - ref)) < 1e-9


# ---------------------------------------------------------------- gather
def test_gather_identity_and_bits():
    rng = np.random.default_rng(22)
    N, d = 50, 24
    hb = rng.integers(0, 65536, (N, d)).astype(np.uint16)
    s = rng.standard_normal(N).astype(np.float32)
    out, pos, so = oracle.gather_compact(hb, np.arange(N, dtype=np.int32), scores=s)
    assert np.array_equal(out, hb) and np.array_equal(pos, np.arange(N)) and np.array_equal(so, s)
    idx = np.array([3, 4, 17, 49], np.int32)
    pin = (np.arange(N) * 10 + 1).astype(np.int32)
    out, pos, so = oracle.gather_compact(hb, idx, pos_in=pin, scores=s)
    assert np.array_equal(out, hb[idx]) and np.array_equal(pos, pin[idx]) and np.array_equal(so, s[idx])
    with pytest.raises(ValueError):
        oracle.gather_compact(hb, np.array([50], np.int32))

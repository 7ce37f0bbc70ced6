"""Pins of the oracle's gate score against facts that do not come from the oracle.

Gate (TokenGate pages: a small MLP scores every token's post-attention
residual at the gate layer: aiproducthub.cn article, paragraph 事件详情;
chathome.org article, section TokenGate の学習可能なトークンプルーニングの仕組み);
the MLP shape RMSNorm -> Linear -> SiLU -> Linear is the
specification's.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle


def test_hand_case_d2_dg1():
    # d = 2, d_g = 1, worked by hand:
    #   h = [3, 4], eps = 0.5  -> mean square = (9 + 16) / 2 = 12.5, r = 1/sqrt(13)
    #   W1 = [[1, 2]]          -> h . W1 = 3 + 8 = 11
    #   b1 = 0.5               -> u = 11/sqrt(13) + 0.5
    #   SiLU(u) = u / (1 + e^-u); w2 = 2, b2 = -1 -> s = 2 SiLU(u) - 1
    u = 11.0 / math.sqrt(13.0) + 0.5
    expect = 2.0 * u / (1.0 + math.exp(-u)) - 1.0
    s = oracle.gate_score(np.array([[3.0, 4.0]]), np.array([[1.0, 2.0]]), np.array([2.0]),
                          b1=np.array([0.5]), b2=-1.0, eps=0.5)
    assert s.shape == (1,)
    assert abs(s[0] - expect) < 1e-12


def test_zero_w1_closed_form():
    # W1 = 0 => u_j = b1_j for every token, s_i = sum_j SiLU(b1_j) w2_j + b2.
    rng = np.random.default_rng(1)
    N, d, d_g = 37, 48, 16
    h = rng.standard_normal((N, d)).astype(np.float32)
    b1 = rng.standard_normal(d_g).astype(np.float32)
    w2 = rng.standard_normal(d_g).astype(np.float32)
    s = oracle.gate_score(h, np.zeros((d_g, d), np.float32), w2, b1=b1, b2=0.25)
    expect = sum(float(b) / (1.0 + math.exp(-float(b))) * float(w) for b, w in zip(b1, w2)) + 0.25
    assert np.allclose(s, expect, rtol=0, atol=1e-12)


def test_row_scale_invariance():
    # RMSNorm divides out a row's scale: s(alpha h_i) = s(h_i) up to the eps term.
    rng = np.random.default_rng(2)
    N, d, d_g = 20, 64, 32
    h = rng.standard_normal((N, d)).astype(np.float32)
    W1 = (rng.standard_normal((d_g, d)) / 8).astype(np.float32)
    w2 = (rng.standard_normal(d_g) / 4).astype(np.float32)
    s1 = oracle.gate_score(h, W1, w2, eps=1e-6)
    s4 = oracle.gate_score(h * 4.0, W1, w2, eps=1e-6)
    assert np.max(np.abs(s1 - s4)) < 1e-5
    # with eps = 0 the invariance is exact up to rounding
    s1 = oracle.gate_score(h, W1, w2, eps=0.0)
    s4 = oracle.gate_score(h * 4.0, W1, w2, eps=0.0)
    assert np.max(np.abs(s1 - s4)) < 1e-12


@pytest.mark.parametrize("with_gamma", [False, True])
def test_against_torch_library_ops(with_gamma):
    # Library special case: torch's rms_norm, linear and silu in fp64.
    rng = np.random.default_rng(3)
    N, d, d_g = 50, 96, 24
    h = rng.standard_normal((N, d)).astype(np.float32)
    W1 = (rng.standard_normal((d_g, d)) / math.sqrt(d)).astype(np.float32)
    b1 = (0.1 * rng.standard_normal(d_g)).astype(np.float32)
    w2 = (rng.standard_normal(d_g) / math.sqrt(d_g)).astype(np.float32)
    gamma = (1 + 0.3 * rng.standard_normal(d)).astype(np.float32) if with_gamma else None
    s = oracle.gate_score(h, W1, w2, b1=b1, b2=-0.3, gamma=gamma, eps=1e-6, fold_gamma_bf16=False)
    th = torch.from_numpy(h).double()
    tg = None if gamma is None else torch.from_numpy(gamma).double()
    x = F.rms_norm(th, (d,), weight=tg, eps=1e-6)
    a = F.silu(F.linear(x, torch.from_numpy(W1).double(), torch.from_numpy(b1).double()))
    ref = F.linear(a, torch.from_numpy(w2).double()[None, :]).squeeze(1) - 0.3
    assert np.max(np.abs(s - ref.numpy())) < 1e-10


def test_gamma_fold_is_bf16_of_product():
    # fold_gamma_bf16: the weight used is bf16(gamma * W1) (torch's round-to-nearest-even).
    rng = np.random.default_rng(4)
    N, d, d_g = 9, 32, 8
    h = rng.standard_normal((N, d)).astype(np.float32)
    W1 = torch.randn(d_g, d, generator=torch.Generator().manual_seed(5)).bfloat16().float()
    gamma = (1 + 0.3 * torch.randn(d, generator=torch.Generator().manual_seed(6))).bfloat16().float()
    w2 = rng.standard_normal(d_g).astype(np.float32)
    folded = (gamma[None, :] * W1).bfloat16().float().numpy()
    s_fold = oracle.gate_score(h, W1.numpy(), w2, gamma=gamma.numpy(), fold_gamma_bf16=True)
    s_ref = oracle.gate_score(h, folded, w2, gamma=None)
    assert np.array_equal(s_fold, s_ref)


def test_round_bf16_matches_torch():
    x = torch.randn(5000, generator=torch.Generator().manual_seed(7)) * 100
    x = torch.cat([x, torch.tensor([1.00390625, 1.01171875, -0.0, float("inf"), 3.0e38])])
    ours = np.array([oracle.round_bf16(float(v)) for v in x], dtype=np.float32)
    ref = x.bfloat16().float().numpy()
    assert np.array_equal(ours.view(np.uint32), ref.view(np.uint32))


def test_single_unit_sign_flip_detected():
    # A transposed or mis-indexed W1 would change the result: swap two rows of W1 and
    # two entries of w2 together (a relabelling of the hidden units) leaves s unchanged,
    # while swapping only W1 rows changes it.
    rng = np.random.default_rng(8)
    N, d, d_g = 11, 16, 4
    h = rng.standard_normal((N, d)).astype(np.float32)
    W1 = rng.standard_normal((d_g, d)).astype(np.float32)
    w2 = np.array([1.0, -2.0, 0.5, 3.0], np.float32)
    s = oracle.gate_score(h, W1, w2)
    perm = [1, 0, 3, 2]
    assert np.allclose(oracle.gate_score(h, W1[perm], w2[perm]), s, rtol=0, atol=1e-12)
    assert not np.allclose(oracle.gate_score(h, W1[perm], w2), s, rtol=0, atol=1e-6)

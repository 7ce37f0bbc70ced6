"""Pins of the oracle's projection of the kept rows against facts that do not come from the oracle.

Above the gate only the kept tokens are processed, so the next layer's Q/K/V projections run on
the compacted rows (aiproducthub.cn article, paragraph 事件详情; chathome.org article, section
TokenGate の学習可能なトークンプルーニングの仕組み).  The projection is a bias-free linear map with
the weight stored one row per output feature (Qwen3's attention projections).
"""
import numpy as np
import torch
import torch.nn.functional as F

import oracle


def test_hand_case():
    # x = [[1, 2, 3], [-1, 0.5, 4]], W = [[1, 0, 0], [0, 1, -1]] (two output features of three
    # inputs), worked by hand:
    #   row 0: [1*1 + 2*0 + 3*0, 1*0 + 2*1 + 3*(-1)] = [1, -1]
    #   row 1: [-1, 0.5 - 4] = [-1, -3.5]
    x = np.array([[1.0, 2.0, 3.0], [-1.0, 0.5, 4.0]])
    W = np.array([[1.0, 0.0, 0.0], [0.0, 1.0, -1.0]])
    out = oracle.project(x, W)
    assert out.shape == (2, 2)
    assert np.array_equal(out, np.array([[1.0, -1.0], [-1.0, -3.5]]))


def test_rectangular_hand_case_orientation():
    # A weight with more outputs than inputs: W [3, 2] maps each 2-vector to 3 features
    # (W[j] . x), so a transposed reading would mix up which input each feature sees.
    x = np.array([[2.0, -3.0]])
    W = np.array([[1.0, 0.0], [0.0, 1.0], [1.0, 1.0]])
    assert np.array_equal(oracle.project(x, W), np.array([[2.0, -3.0, -1.0]]))


def test_matches_torch_linear_fp64():
    rng = np.random.default_rng(11)
    for K, d, n_out in ((1, 8, 8), (37, 64, 24), (130, 256, 384)):
        x = rng.standard_normal((K, d)).astype(np.float32)
        W = (rng.standard_normal((n_out, d)) / np.sqrt(d)).astype(np.float32)
        want = F.linear(torch.from_numpy(x).double(), torch.from_numpy(W).double()).numpy()
        got = oracle.project(x, W)
        assert np.max(np.abs(got - want)) <= 1e-12 * max(1.0, np.max(np.abs(want)))


def test_identity_and_permutation():
    rng = np.random.default_rng(12)
    x = rng.standard_normal((9, 16)).astype(np.float32)
    assert np.array_equal(oracle.project(x, np.eye(16, dtype=np.float32)), x.astype(np.float64))
    perm = rng.permutation(16)
    P = np.eye(16, dtype=np.float32)[perm]           # output feature j reads input perm[j]
    assert np.array_equal(oracle.project(x, P), x[:, perm].astype(np.float64))


def test_stacked_weights_give_column_blocks():
    # Stacking Wq, Wk, Wv row-wise projects to Q | K | V side by side; each row is independent,
    # so projecting a subset of rows gives the same rows.
    rng = np.random.default_rng(13)
    x = rng.standard_normal((20, 32)).astype(np.float32)
    Wq, Wk, Wv = (rng.standard_normal((n, 32)).astype(np.float32) for n in (16, 8, 8))
    full = oracle.project(x, np.concatenate([Wq, Wk, Wv]))
    assert np.array_equal(full[:, :16], oracle.project(x, Wq))
    assert np.array_equal(full[:, 16:24], oracle.project(x, Wk))
    assert np.array_equal(full[:, 24:], oracle.project(x, Wv))
    rows = np.array([0, 5, 19])
    assert np.array_equal(oracle.project(x[rows], np.concatenate([Wq, Wk, Wv])), full[rows])

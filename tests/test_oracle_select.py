"""Pins of the oracle's top-K selection.

Selection rule (TokenGate pages: top-K keeps the best-scored tokens and the
question is never pruned: aiproducthub.cn article, paragraph 事件详情;
aisight.pl article, section Jak to działa; chathome.org article, section
TokenGate の学習可能なトークンプルーニングの仕組み); tie rule (lower index first) and the
ascending output order are the specification's; NaN ranks below every number
and -0 equals +0 (a reading where both are silent).
"""
import itertools
import math

import numpy as np
import pytest

import oracle


def _beats(s, a, b):
    """True if token a ranks strictly before token b (brute-force statement of the order)."""
    sa, sb = float(s[a]), float(s[b])
    na, nb = math.isnan(sa), math.isnan(sb)
    if na != nb:
        return nb
    if not na and sa != sb:
        return sa > sb
    return a < b


def _brute_force(s, db, de, k):
    """Enumerate every k-subset of the document and keep those in which every kept
    token beats every dropped one; exactly one must exist."""
    doc = list(range(db, de))
    k = min(k, len(doc))
    ok = []
    for sub in itertools.combinations(doc, k):
        sub_set = set(sub)
        drop = [i for i in doc if i not in sub_set]
        if all(_beats(s, a, b) for a in sub for b in drop):
            ok.append(sub_set)
    assert len(ok) == 1
    other = [i for i in range(len(s)) if i < db or i >= de]
    return sorted(ok[0] | set(other))


@pytest.mark.parametrize("seed", range(12))
def test_brute_force_tiny(seed):
    rng = np.random.default_rng(seed)
    N = int(rng.integers(1, 12))
    db = int(rng.integers(0, N))
    de = int(rng.integers(db, N + 1))
    k = int(rng.integers(0, de - db + 2))
    # few distinct values so that ties are common; sprinkle +-0, NaN and +-inf
    vals = np.array([0.5, -0.5, 0.0, -0.0, 1.0, float("nan"), float("inf"), float("-inf")], np.float32)
    s = vals[rng.integers(0, len(vals), N)]
    got = oracle.topk_select(s, db, de, k)
    assert list(got) == _brute_force(s, db, de, k)


def test_hand_case_ties_zero_nan():
    # Document = indices 0..7, question = 8, 9; keep 4 document tokens.
    # scores:  0:1.0  1:NaN  2:2.0  3:-0.0  4:1.0  5:+0.0  6:-inf  7:1.0  8:-5  9:NaN
    # order: 2 (2.0), then the three 1.0s by index: 0, 4, 7 -> kept doc = {0, 2, 4, 7}.
    s = np.array([1.0, np.nan, 2.0, -0.0, 1.0, 0.0, -np.inf, 1.0, -5.0, np.nan], np.float32)
    assert list(oracle.topk_select(s, 0, 8, 4)) == [0, 2, 4, 7, 8, 9]
    # keep 5: next come the zeros, -0 == +0, so index 3 wins over 5.
    assert list(oracle.topk_select(s, 0, 8, 5)) == [0, 2, 3, 4, 7, 8, 9]
    # keep 7: zeros, then -inf (6) beats NaN (1).
    assert list(oracle.topk_select(s, 0, 8, 7)) == [0, 2, 3, 4, 5, 6, 7, 8, 9]
    # thresholds: the k-th document score in the order
    assert oracle.topk_threshold(s, 0, 8, 4) == 1.0
    assert oracle.topk_threshold(s, 0, 8, 7) == -np.inf


def test_budget_edge_cases():
    s = np.arange(10, dtype=np.float32)
    assert list(oracle.topk_select(s, 2, 8, 0)) == [0, 1, 8, 9]              # K_doc = 0
    assert list(oracle.topk_select(s, 2, 8, 6)) == list(range(10))            # K_doc = N_doc
    assert list(oracle.topk_select(s, 2, 8, 100)) == list(range(10))          # K_doc > N_doc
    assert list(oracle.topk_select(s, 4, 4, 3)) == list(range(10))            # empty span
    assert list(oracle.topk_select(s, 0, 10, 3)) == [7, 8, 9]                 # no question
    assert oracle.kept_count(10, 2, 8, 3) == 7
    assert oracle.kept_count(10, 2, 11, 3) == -1
    assert oracle.kept_count(10, 2, 8, -1) == -1
    with pytest.raises(ValueError):
        oracle.topk_select(s, 5, 3, 1)


@pytest.mark.parametrize("N,db,de,k", [(5000, 0, 4800, 700), (4096, 100, 4000, 1), (3000, 17, 2999, 2981)])
def test_invariants_random(N, db, de, k):
    rng = np.random.default_rng(N + k)
    s = (np.round(rng.standard_normal(N) * 16) / 16).astype(np.float32)   # many ties
    kept = oracle.topk_select(s, db, de, k)
    K = min(k, de - db) + N - (de - db)
    assert kept.shape == (K,)
    assert np.all(np.diff(kept) > 0)                                      # strictly ascending
    ks = set(kept.tolist())
    assert all(i in ks for i in range(N) if i < db or i >= de)            # question always kept
    doc_kept = [i for i in kept if db <= i < de]
    doc_drop = [i for i in range(db, de) if i not in ks]
    # library sort as the independent order: numpy lexsort by (-score, index)
    order = np.lexsort((np.arange(db, de), -s[db:de].astype(np.float64))) + db
    assert sorted(order[: len(doc_kept)].tolist()) == sorted(doc_kept)
    if doc_kept and doc_drop:
        worst_kept = order[len(doc_kept) - 1]
        best_drop = order[len(doc_kept)]
        assert _beats(s, worst_kept, best_drop)
        assert oracle.topk_threshold(s, db, de, k) == s[worst_kept]


def test_permuting_within_ties_picks_lower_indices():
    s = np.zeros(64, np.float32)
    s[[3, 9, 40]] = 1.0
    kept = oracle.topk_select(s, 0, 64, 10)
    assert kept.tolist() == [0, 1, 2, 3, 4, 5, 6, 7, 9, 40]

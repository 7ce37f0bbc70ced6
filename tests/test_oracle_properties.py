"""Property tests of the oracle's select (hypothesis): tiny random shapes and
scores drawn from a pool with ties, +0/-0, NaN and infinities, every budget
edge (0, inside, = n_doc, > n_doc), against a brute force written straight from
the order the specification fixes: score descending, index ascending on ties,
-0 equal to +0, NaN below every number, every token outside the span kept."""
import math

import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle

POOL = [0.0, -0.0, 1.0, -1.0, 2.5, 2.5, float("nan"), float("inf"), -float("inf"), 1e-30, -1e-30, 3.0]


def brute(scores, db, de, k):
    def key(i):
        v = float(scores[i])
        return (1, 0.0, i) if math.isnan(v) else (0, -(v + 0.0), i)  # + 0.0 folds -0 into +0
    doc = sorted(range(db, de), key=key)[: min(k, de - db)]
    return sorted(set(doc) | set(range(0, db)) | set(range(de, len(scores))))


@settings(max_examples=300, deadline=None)
@given(st.data())
def test_select_matches_the_specified_order(data):
    N = data.draw(st.integers(0, 40))
    db = data.draw(st.integers(0, N))
    de = data.draw(st.integers(db, N))
    k = data.draw(st.integers(0, N + 3))
    vals = data.draw(st.lists(st.sampled_from(POOL), min_size=N, max_size=N))
    scores = np.array(vals, dtype=np.float32)
    got = oracle.topk_select(scores, db, de, k) if N else np.empty(0, np.int32)
    assert list(got) == brute(scores, db, de, k)

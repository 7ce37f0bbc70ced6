"""GPU select against the oracle on hypothesis-drawn score vectors: ties, +0/-0,
NaN and infinities in every block of a multi-block grid, budget edges
(bit-exact), with a guard band around the output."""
import numpy as np
import pytest
import torch
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle
from learned_token_pruning_tg_b200 import tokengate as tg
from tests.guards import guarded

pytestmark = pytest.mark.gpu

POOL = np.array([0.0, -0.0, 1.0, -1.0, 2.5, float("nan"), float("inf"), -float("inf"), 1e-30, 3.0], np.float32)


@settings(max_examples=25, deadline=None)
@given(st.data())
def test_gpu_select_matches_oracle(data):
    N = data.draw(st.integers(1, 300000))
    db = data.draw(st.integers(0, N - 1))
    de = data.draw(st.integers(db + 1, N))
    k = data.draw(st.integers(0, de - db + 2))
    seed = data.draw(st.integers(0, 2 ** 31 - 1))
    rng = np.random.default_rng(seed)
    mix = data.draw(st.floats(0.0, 1.0))
    scores = np.where(rng.random(N) < mix, POOL[rng.integers(0, len(POOL), N)],
                      rng.standard_normal(N).astype(np.float32)).astype(np.float32)
    K = tg.tg_kept_count(N, db, de, k)
    out, check = guarded((max(K, 1),), torch.int32)
    ws = tg.new_workspace(N)
    tg.tg_topk_select(torch.from_numpy(scores).cuda(), db, de, k, out[:K], ws)
    torch.cuda.synchronize()
    check()
    assert tg.tg_device_status(ws) == 0
    assert np.array_equal(out[:K].cpu().numpy(), oracle.topk_select(scores, db, de, k))

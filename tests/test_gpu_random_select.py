"""GPU parity of tg_random_select (the random-K baseline selector) against the oracle.

Bit-exact: the keys are integers drawn from SplitMix64 on both sides and the
selection is the same total order, so the kept index lists must be equal.
"""
import numpy as np
import pytest
import torch

import oracle
from learned_token_pruning_tg_b200 import tokengate as tg

pytestmark = pytest.mark.gpu

M64 = (1 << 64) - 1


def run(N, db, de, k, seed, ws=None):
    K = tg.tg_kept_count(N, db, de, k)
    out = torch.full((max(K, 1),), -1, dtype=torch.int32, device="cuda")
    ws = ws if ws is not None else tg.new_workspace(N)
    tg.tg_random_select(N, db, de, k, seed, out[:K], ws)
    torch.cuda.synchronize()
    assert tg.tg_device_status(ws) == 0
    return out[:K].cpu().numpy()


@pytest.mark.parametrize("N,db,de,k,seed", [
    (1024, 0, 960, 192, 0),            # the tiny workload's span and budget
    (16384, 0, 16000, 1024, 16),
    (131072, 0, 130560, 4096, 128),    # the 128k workload
    (300000, 1000, 299000, 100000, M64),
    (5000, 17, 4990, 1, 7),
])
def test_random_select_bit_exact(N, db, de, k, seed):
    got = run(N, db, de, k, seed)
    assert np.array_equal(got, oracle.random_select(N, db, de, k, seed))


@pytest.mark.parametrize("k", [0, 1, 959, 960, 5000])
def test_random_select_budget_edges(k):
    assert np.array_equal(run(1024, 0, 960, k, 3), oracle.random_select(1024, 0, 960, k, 3))


def test_random_select_repeat_calls_one_workspace():
    ws = tg.new_workspace(131072)
    for seed in (1, 2, 3):
        got = run(131072, 0, 130560, 4096, seed, ws)
        assert np.array_equal(got, oracle.random_select(131072, 0, 130560, 4096, seed))

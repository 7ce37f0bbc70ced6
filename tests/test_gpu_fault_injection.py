"""Failure detection without a GPU fault.

The select's grid barrier (the cooperative launch shape, used for spans longer than one
thread-block cluster holds; shorter spans use hardware cluster barriers, which need no limit) is a
bounded spin.  With its time limit shrunk to a
nanosecond (tg_debug_set_select_wait_limit, a test hook) the blocks of a call
stop waiting for one another: the call must end by itself, report
TG_STATUS_SELECT_TIMEOUT in the workspace's status word (tg_device_status), and
leave the context usable -- after the workspace is zero-filled again the next
call is bit-exact.  Nothing here traps, faults or hangs the GPU.
"""
import numpy as np
import pytest
import torch

import oracle
from learned_token_pruning_tg_b200 import synth
from learned_token_pruning_tg_b200 import tokengate as tg

pytestmark = pytest.mark.gpu


def test_select_barrier_timeout_is_reported_and_the_context_recovers():
    N, db, de, k = 600000, 0, 599000, 4096   # beyond the one-cluster shape: the cooperative one
    s = synth.score_vector(N, seed=11, kind="normal").cuda()
    K = tg.tg_kept_count(N, db, de, k)
    out = torch.full((K,), -1, dtype=torch.int32, device="cuda")
    ws = tg.new_workspace(N)
    try:
        tg.tg_debug_set_select_wait_limit(1)
        tg.tg_topk_select(s, db, de, k, out, ws)
        torch.cuda.synchronize()
        status = tg.tg_device_status(ws)
    finally:
        tg.tg_debug_set_select_wait_limit(0)
    assert status & tg.TG_STATUS_SELECT_TIMEOUT
    # recovery: a fresh (zeroed) workspace state, the default limit, an exact result
    ws.zero_()
    tg.tg_topk_select(s, db, de, k, out, ws)
    torch.cuda.synchronize()
    assert tg.tg_device_status(ws) == 0
    assert np.array_equal(out.cpu().numpy(), oracle.topk_select(s.cpu().numpy(), db, de, k))

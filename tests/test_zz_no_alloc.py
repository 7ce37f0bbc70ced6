"""The allocation-free select entry point against the workspace one.

tg_topk_select_noalloc exists for callers that cannot allocate device memory
when they select tokens; its scratch is a static device array inside the
library that every call shares.  Its output must equal tg_topk_select's bit
for bit (selection is index work), on two calls in a row, since the second call
finds the array as the first one left it.  This file is collected last so that
a run that stops at the first failure has already run every other test.
"""
import numpy as np
import pytest
import torch

from learned_token_pruning_tg_b200 import synth
from learned_token_pruning_tg_b200 import tokengate as tg

pytestmark = pytest.mark.gpu


def _reference(s, db, de, k):
    N = s.shape[0]
    out = torch.full((tg.tg_kept_count(N, db, de, k),), -1, dtype=torch.int32, device="cuda")
    tg.tg_topk_select(s, db, de, k, out, tg.new_workspace(N))
    return out


def _noalloc(s, db, de, k):
    N = s.shape[0]
    out = torch.full((tg.tg_kept_count(N, db, de, k),), -1, dtype=torch.int32, device="cuda")
    tg.tg_topk_select_noalloc(s, db, de, k, out)
    return out


@pytest.mark.parametrize("N,db,de,k,kind", [
    (131072, 0, 130560, 4096, "heavy"),     # the 128k workload's span and budget
    (16384, 0, 16000, 1024, "ties"),        # 16k workload, many tied scores
    (70001, 333, 69000, 12345, "special"),  # ragged span, NaN / inf / signed zeros
])
def test_noalloc_matches_workspace_select_on_two_calls(N, db, de, k, kind):
    s = synth.score_vector(N, 31, kind).cuda()
    want = _reference(s, db, de, k)
    first = _noalloc(s, db, de, k)
    second = _noalloc(s, db, de, k)
    torch.cuda.synchronize()
    assert torch.equal(first, want)
    assert torch.equal(second, want)


def test_noalloc_second_call_with_other_inputs():
    # state left by one call must not leak into the next one with different inputs
    a = synth.score_vector(131072, 32, "normal").cuda()
    b = synth.score_vector(40000, 33, "heavy").cuda()
    ra, rb = _reference(a, 0, 130560, 4096), _reference(b, 100, 39000, 5000)
    oa, ob = _noalloc(a, 0, 130560, 4096), _noalloc(b, 100, 39000, 5000)
    torch.cuda.synchronize()
    assert torch.equal(oa, ra) and torch.equal(ob, rb)


def test_noalloc_rejects_spans_beyond_its_limit():
    # one past #SMs * 1024 * 16 document tokens (the largest grid the select kernel uses)
    n_doc = torch.cuda.get_device_properties(0).multi_processor_count * 1024 * 16 + 1
    big = torch.zeros(n_doc + 5, dtype=torch.float32, device="cuda")
    out = torch.empty(tg.tg_kept_count(n_doc + 5, 0, n_doc, 16), dtype=torch.int32, device="cuda")
    with pytest.raises(tg.TokenGateError) as e:
        tg.tg_topk_select_noalloc(big, 0, n_doc, 16, out)
    assert e.value.status == tg.TG_ERR_UNSUPPORTED


def test_noalloc_timeout_is_reported_by_its_status_query():
    # The static array's status word carries a select timeout to the caller.  The grid barrier's limit is
    # shrunk to a nanosecond (the fault-injection hook: nothing traps or hangs), the call's blocks stop
    # waiting and set TG_STATUS_SELECT_TIMEOUT, the status query reports it, and the next call -- which
    # clears the array first -- is exact again and reports nothing.
    s = synth.score_vector(131072, 34, "normal").cuda()
    want = _reference(s, 0, 130560, 4096)
    try:
        tg.tg_debug_set_select_wait_limit(1)
        _noalloc(s, 0, 130560, 4096)
        bits = tg.tg_topk_select_noalloc_status()
    finally:
        tg.tg_debug_set_select_wait_limit(0)
    assert bits & tg.TG_STATUS_SELECT_TIMEOUT
    again = _noalloc(s, 0, 130560, 4096)
    assert tg.tg_topk_select_noalloc_status() == 0
    assert torch.equal(again, want)

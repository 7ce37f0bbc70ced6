"""Host logic of the path module that needs no device: the NVTX step marks."""
import torch

from learned_token_pruning_tg_b200 import path


def test_nvtx_marks_one_balanced_range_per_step(monkeypatch):
    log = []
    monkeypatch.setattr(torch.cuda.nvtx, "range_push", lambda name: log.append(("push", name)))
    monkeypatch.setattr(torch.cuda.nvtx, "range_pop", lambda: log.append(("pop",)))
    mark = path.nvtx_marks()
    for name in path.STAGES + ("end",):
        mark(name)
    want = []
    for name in path.STAGES:
        want += [("push", "tg:" + name), ("pop",)]
    assert log == want

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


def _layer(**kw):
    # a layer built on the CPU: buffers and stage lists only (no kernel runs)
    N, d, d_g, Hq, Hkv, d_h = 1024, 256, 64, 4, 2, 64
    g = torch.Generator().manual_seed(0)
    W1 = torch.randn(d_g, d, generator=g)
    w2 = torch.randn(d_g, generator=g)
    Wqkv = torch.randn((Hq + 2 * Hkv) * d_h, d, generator=g)
    return path.GatedPrefillLayer(N, 0, 960, 192, W1, w2, Wqkv, Hq, Hkv, d_h, torch.zeros(Hq), 1.0, device="cpu",
                                  **kw)


def test_layer_stages_and_launch_counts():
    # the default path: gate, select, gather, fused projection, attention (5 kernels)
    lay = _layer()
    assert lay.stages == path.STAGES == ("gate", "select", "gather", "proj", "attn")
    assert lay.K == 256 and lay.h_kept is not None and lay.launches_per_step() == 5
    assert list(lay.stage_calls(torch.zeros(1024, 256, dtype=torch.bfloat16))) == list(lay.stages)
    assert lay.positions().data_ptr() == lay.pos.data_ptr()
    # the gather inside the projection: no compacted rows, positions are the kept indices
    g = _layer(gather_into_projection=True)
    assert g.stages == ("gate", "select", "proj", "attn") and g.h_kept is None and g.launches_per_step() == 4
    assert g.positions().data_ptr() == g.kept.data_ptr()
    # the library GEMM + RoPE pass + attention converting V itself
    u = _layer(fused_projection=False)
    assert u.stages == ("gate", "select", "gather", "qkv", "rope", "attn") and u.launches_per_step() == 6
    assert u.v16 is None and u.ws_proj is None

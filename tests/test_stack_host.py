"""Host-side pieces of the pruned stack (no GPU): shapes and kept counts of the
configurations, seeded weights, and the torch RMSNorm glue against its formula."""
import math

import torch

from learned_token_pruning_tg_b200 import stack as stk


def test_configs_kept_count():
    c = stk.STACK64K
    assert c.K == 8192 + (c.N - (c.doc_end - c.doc_begin)) == 8704
    assert 0 <= c.gate_layer < c.n_layers - 1
    assert stk.STACK_TINY.K == 192 + 64


def test_random_weights_shapes_and_seed():
    c = stk.STACK_TINY
    a = stk.random_weights(c, "cpu")
    b = stk.random_weights(c, "cpu")
    assert len(a.layers) == c.n_layers
    lw = a.layers[0]
    assert lw.Wqkv.shape == ((c.Hq + 2 * c.Hkv) * c.d_h, c.d) and lw.Wqkv.dtype == torch.bfloat16
    assert lw.Wo.shape == (c.d, c.Hq * c.d_h) and lw.Wgu.shape == (2 * c.d_ff, c.d) and lw.Wd.shape == (c.d, c.d_ff)
    assert a.W1.shape == (c.d_g, c.d) and a.w2.shape == (c.d_g,)
    assert all(0.8 <= l.tau <= 1.5 for l in a.layers)
    assert torch.equal(a.layers[-1].Wd, b.layers[-1].Wd)            # seeded


def test_rms_norm_formula():
    x = torch.tensor([[3.0, -4.0, 0.0, 0.0]]).to(torch.bfloat16)
    w = torch.tensor([1.0, 2.0, 1.0, 1.0]).to(torch.bfloat16)
    y = stk.rms_norm(x, w, 0.0).float()
    r = 1.0 / math.sqrt((9 + 16) / 4)                               # mean of squares 6.25
    assert torch.allclose(y, torch.tensor([[3 * r, -8 * r, 0.0, 0.0]]), rtol=2 ** -8)

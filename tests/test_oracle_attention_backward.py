"""Pins of the oracle's gated-attention backward (oracle.gated_attention_backward).

None of these re-types the backward.  They check it against
* central differences of the oracle's own forward (a separate routine), with
  inputs on a 2^-8 grid and steps of 2^-10 so that every perturbed input is
  exact in fp32 and the only error is the O(step^2) truncation;
* torch autograd in fp64 through a forward written here with torch ops
  (masked logits, softmax, weighted sum) -- a mechanical derivative of the
  definition, independent of the hand-derived chain rule;
* identities of the mathematics that hold at any size: a constant added to
  every score cancels (sum_c ds_c = 0); scaling q, or every key, by a factor
  is scaling tau (sum q.dq = tau dtau = sum k.dk); the softmax weights of a row
  sum to one (sum_c dv_c = sum of dout over the group's rows); row 0 sees only
  key 0, so its dq is zero; grouped-query heads equal duplicated KV heads.
"""
import numpy as np
import pytest
import torch

import oracle

STEP = 2.0 ** -10


def grid_inputs(rng, K, Hq, Hkv, d_h):
    def g(*shape, scale=1.0):
        return (np.round(rng.standard_normal(shape) * scale * 256) / 256).astype(np.float32)
    return dict(q=g(K, Hq, d_h), k=g(K, Hkv, d_h), v=g(K, Hkv, d_h), dout=g(K, Hq, d_h), s=g(K, scale=2.0),
                g=(np.round(rng.random(Hq) * 2 * 256) / 256).astype(np.float32))


def loss(x, tau, pos=None):
    out = oracle.gated_attention(x["q"], x["k"], x["v"], s=x["s"], g=x["g"], tau=tau, pos=pos)
    return float(np.sum(x["dout"].astype(np.float64) * out))


@pytest.mark.parametrize("pos", [None, np.array([0, 3, 4, 9, 10], dtype=np.int32)])
def test_backward_matches_central_differences(pos):
    rng = np.random.default_rng(5)
    K, Hq, Hkv, d_h, tau = 5, 4, 2, 4, 1.25
    x = grid_inputs(rng, K, Hq, Hkv, d_h)
    got = oracle.gated_attention_backward(x["q"], x["k"], x["v"], x["dout"], s=x["s"], g=x["g"], tau=tau, pos=pos)
    for name, key in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("s", "ds"), ("g", "dg")):
        base = x[name]
        fd = np.zeros(base.shape)
        for idx in np.ndindex(base.shape):
            plus = {**x, name: base.copy()}
            minus = {**x, name: base.copy()}
            plus[name][idx] += STEP
            minus[name][idx] -= STEP
            assert plus[name][idx] - STEP == base[idx]     # the step is exact in fp32
            fd[idx] = (loss(plus, tau, pos) - loss(minus, tau, pos)) / (2 * STEP)
        np.testing.assert_allclose(got[key], fd, rtol=0, atol=2e-6, err_msg=key)
    h = 1e-5
    fd_tau = (loss(x, tau + h, pos) - loss(x, tau - h, pos)) / (2 * h)
    assert abs(got["dtau"] - fd_tau) <= 1e-7


def torch_forward(q, k, v, s, g, tau, pos):
    K, Hq, d_h = q.shape
    G = Hq // k.shape[1]
    kk = k.repeat_interleave(G, dim=1)            # [K, Hq, d_h]
    vv = v.repeat_interleave(G, dim=1)
    logits = torch.einsum("rhd,chd->hrc", q, kk) * tau / d_h ** 0.5 + g[:, None, None] * s[None, None, :]
    visible = pos[None, :] <= pos[:, None]        # [r, c]
    logits = logits.masked_fill(~visible[None], float("-inf"))
    p = torch.softmax(logits, dim=-1)
    return torch.einsum("hrc,chd->rhd", p, vv)


@pytest.mark.parametrize("K,Hq,Hkv,d_h,use_pos", [(33, 4, 2, 16, False), (40, 8, 2, 8, True), (17, 3, 1, 32, False)])
def test_backward_matches_torch_autograd(K, Hq, Hkv, d_h, use_pos):
    rng = np.random.default_rng(K + Hq)
    x = grid_inputs(rng, K, Hq, Hkv, d_h)
    tau = 0.9
    pos = np.sort(rng.choice(4 * K, K, replace=False)).astype(np.int32) if use_pos else None
    got = oracle.gated_attention_backward(x["q"], x["k"], x["v"], x["dout"], s=x["s"], g=x["g"], tau=tau, pos=pos)
    t = {n: torch.tensor(x[n], dtype=torch.float64, requires_grad=n != "dout") for n in x}
    tt = torch.tensor(tau, dtype=torch.float64, requires_grad=True)
    tp = torch.arange(K) if pos is None else torch.tensor(pos.astype(np.int64))
    out = torch_forward(t["q"], t["k"], t["v"], t["s"], t["g"], tt, tp)
    (out * t["dout"]).sum().backward()
    for name, key in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("s", "ds"), ("g", "dg")):
        np.testing.assert_allclose(got[key], t[name].grad.numpy(), rtol=1e-9, atol=1e-11, err_msg=key)
    assert abs(got["dtau"] - tt.grad.item()) <= 1e-9 * max(1.0, abs(tt.grad.item()))


def test_backward_identities():
    rng = np.random.default_rng(11)
    K, Hq, Hkv, d_h, tau = 70, 8, 2, 32, 1.4
    x = {n: a.astype(np.float32) for n, a in grid_inputs(rng, K, Hq, Hkv, d_h).items()}
    b = oracle.gated_attention_backward(x["q"], x["k"], x["v"], x["dout"], s=x["s"], g=x["g"], tau=tau)
    # a constant added to every kept score shifts every visible logit of a row alike
    assert abs(b["ds"].sum()) <= 1e-10 * np.abs(b["ds"]).sum()
    # q -> a q and k -> a k both act like tau -> a tau
    qdq = float(np.sum(x["q"].astype(np.float64) * b["dq"]))
    kdk = float(np.sum(x["k"].astype(np.float64) * b["dk"]))
    assert abs(qdq - tau * b["dtau"]) <= 1e-10 * max(1.0, abs(qdq))
    assert abs(kdk - tau * b["dtau"]) <= 1e-10 * max(1.0, abs(kdk))
    # every row's softmax weights sum to one
    G = Hq // Hkv
    want_dv = x["dout"].astype(np.float64).reshape(K, Hkv, G, d_h).sum(axis=(0, 2))
    np.testing.assert_allclose(b["dv"].sum(axis=0), want_dv, rtol=1e-10, atol=1e-10)
    # row 0 sees key 0 alone: its softmax weight is the constant 1
    assert np.all(b["dq"][0] == 0.0)
    # without a bias term the score gradient vanishes; the gain gradient does not
    z = oracle.gated_attention_backward(x["q"], x["k"], x["v"], x["dout"], s=x["s"], g=np.zeros(Hq, np.float32),
                                        tau=tau)
    assert np.all(z["ds"] == 0.0) and np.any(z["dg"] != 0.0)


def test_backward_grouped_heads_equal_duplicated_kv_heads():
    rng = np.random.default_rng(12)
    K, Hq, Hkv, d_h, tau = 25, 6, 2, 8, 1.1
    x = grid_inputs(rng, K, Hq, Hkv, d_h)
    G = Hq // Hkv
    b = oracle.gated_attention_backward(x["q"], x["k"], x["v"], x["dout"], s=x["s"], g=x["g"], tau=tau)
    kd, vd = np.repeat(x["k"], G, axis=1), np.repeat(x["v"], G, axis=1)
    d = oracle.gated_attention_backward(x["q"], kd, vd, x["dout"], s=x["s"], g=x["g"], tau=tau)
    np.testing.assert_allclose(d["dk"].reshape(K, Hkv, G, d_h).sum(axis=2), b["dk"], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(d["dv"].reshape(K, Hkv, G, d_h).sum(axis=2), b["dv"], rtol=1e-12, atol=1e-13)
    for key in ("dq", "ds", "dg"):
        np.testing.assert_allclose(d[key], b[key], rtol=1e-12, atol=1e-13)


def test_backward_split_by_kv_head_equals_whole():
    from tests import oracle_pool
    rng = np.random.default_rng(13)
    K, Hq, Hkv, d_h, tau = 30, 6, 3, 8, 0.8
    x = grid_inputs(rng, K, Hq, Hkv, d_h)
    whole = oracle.gated_attention_backward(x["q"], x["k"], x["v"], x["dout"], s=x["s"], g=x["g"], tau=tau)
    split = oracle_pool.gated_attention_backward(x["q"], x["k"], x["v"], x["dout"], s=x["s"], g=x["g"], tau=tau)
    for key in ("dq", "dk", "dv", "ds", "dg"):
        np.testing.assert_allclose(split[key], whole[key], rtol=1e-12, atol=1e-14)
    assert abs(split["dtau"] - whole["dtau"]) <= 1e-12 * max(1.0, abs(whole["dtau"]))

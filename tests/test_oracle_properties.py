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


def _torch_gated_attention(q, k, v, s, g, tau, pos):
    """The gated attention written with torch ops in fp64 (masked logits, softmax, weighted sum)."""
    import torch
    K, Hq, d_h = q.shape
    G = Hq // k.shape[1]
    kk, vv = k.repeat_interleave(G, dim=1), v.repeat_interleave(G, dim=1)
    logits = torch.einsum("rhd,chd->hrc", q, kk) * tau / d_h ** 0.5 + g[:, None, None] * s[None, None, :]
    logits = logits.masked_fill(~(pos[None, :] <= pos[:, None])[None], float("-inf"))
    return torch.einsum("hrc,chd->rhd", torch.softmax(logits, dim=-1), vv)


@settings(max_examples=60, deadline=None)
@given(st.data())
def test_attention_forward_and_backward_match_torch(data):
    """Random tiny shapes, gains, temperatures and position patterns: the oracle's forward against a
    torch fp64 forward, and its backward against torch autograd of that forward."""
    import torch
    Hkv = data.draw(st.integers(1, 3))
    G = data.draw(st.sampled_from([1, 2, 4]))
    Hq, d_h, K = Hkv * G, data.draw(st.sampled_from([2, 4, 8])), data.draw(st.integers(1, 12))
    tau = data.draw(st.floats(0.25, 3.0))
    seed = data.draw(st.integers(0, 2 ** 31 - 1))
    gaps = data.draw(st.booleans())
    rng = np.random.default_rng(seed)
    x = {n: rng.standard_normal(shape).astype(np.float32) for n, shape in
         (("q", (K, Hq, d_h)), ("k", (K, Hkv, d_h)), ("v", (K, Hkv, d_h)), ("dout", (K, Hq, d_h)), ("s", (K,)))}
    x["g"] = (2.0 * rng.random(Hq)).astype(np.float32)
    pos = np.sort(rng.choice(5 * K, K, replace=False)).astype(np.int32) if gaps else None
    want_out = oracle.gated_attention(x["q"], x["k"], x["v"], s=x["s"], g=x["g"], tau=tau, pos=pos)
    grads = oracle.gated_attention_backward(x["q"], x["k"], x["v"], x["dout"], s=x["s"], g=x["g"], tau=tau, pos=pos)
    t = {n: torch.tensor(a, dtype=torch.float64, requires_grad=n != "dout") for n, a in x.items()}
    tt = torch.tensor(tau, dtype=torch.float64, requires_grad=True)
    tp = torch.arange(K) if pos is None else torch.tensor(pos.astype(np.int64))
    out = _torch_gated_attention(t["q"], t["k"], t["v"], t["s"], t["g"], tt, tp)
    np.testing.assert_allclose(want_out, out.detach().numpy(), rtol=1e-10, atol=1e-12)
    (out * t["dout"]).sum().backward()
    for name, key in (("q", "dq"), ("k", "dk"), ("v", "dv"), ("s", "ds"), ("g", "dg")):
        np.testing.assert_allclose(grads[key], t[name].grad.numpy(), rtol=1e-9, atol=1e-11, err_msg=key)
    assert abs(grads["dtau"] - tt.grad.item()) <= 1e-9 * max(1.0, abs(tt.grad.item()))


@settings(max_examples=80, deadline=None)
@given(st.data())
def test_gate_matches_torch_library_ops(data):
    """Random tiny gate shapes, eps, biases and RMSNorm weights against torch's rms_norm, linear and
    silu in fp64 (the RMSNorm weight applied exactly: fold_gamma_bf16=False)."""
    import torch
    import torch.nn.functional as F
    N, d, d_g = data.draw(st.integers(1, 9)), data.draw(st.integers(1, 24)), data.draw(st.integers(1, 8))
    eps = data.draw(st.sampled_from([0.0, 1e-6, 1e-2]))
    b2 = data.draw(st.floats(-2.0, 2.0))
    use_b1, use_gamma = data.draw(st.booleans()), data.draw(st.booleans())
    rng = np.random.default_rng(data.draw(st.integers(0, 2 ** 31 - 1)))
    h = rng.standard_normal((N, d)).astype(np.float32)
    if eps == 0.0:
        h[np.all(h == 0, axis=1)] = 1.0     # no all-zero row when nothing keeps the norm finite
    W1 = rng.standard_normal((d_g, d)).astype(np.float32)
    w2 = rng.standard_normal(d_g).astype(np.float32)
    b1 = rng.standard_normal(d_g).astype(np.float32) if use_b1 else None
    gamma = (1 + 0.5 * rng.standard_normal(d)).astype(np.float32) if use_gamma else None
    s = oracle.gate_score(h, W1, w2, b1=b1, b2=b2, gamma=gamma, eps=eps, fold_gamma_bf16=False)
    x = F.rms_norm(torch.from_numpy(h).double(), (d,), weight=None if gamma is None else
                   torch.from_numpy(gamma).double(), eps=eps)
    a = F.silu(F.linear(x, torch.from_numpy(W1).double(), None if b1 is None else torch.from_numpy(b1).double()))
    ref = (a @ torch.from_numpy(w2).double()) + b2
    np.testing.assert_allclose(s, ref.numpy(), rtol=1e-9, atol=1e-10)


@settings(max_examples=80, deadline=None)
@given(st.data())
def test_rope_matches_complex_rotation(data):
    """Random shapes, positions and bases against numpy's complex multiplication: the rotate-half
    pair (t, t + d_h/2) is the complex number x_t + i x_{t+d_h/2} turned by pos * base^(-2t/d_h)."""
    K, H = data.draw(st.integers(1, 6)), data.draw(st.integers(1, 4))
    d_h = 2 * data.draw(st.integers(1, 16))
    base = data.draw(st.sampled_from([10.0, 1e4, 1e6]))
    rng = np.random.default_rng(data.draw(st.integers(0, 2 ** 31 - 1)))
    x = rng.standard_normal((K, H, d_h)).astype(np.float32)
    pos = rng.integers(0, 200000, K).astype(np.int32)
    got = oracle.rope(x, pos, base)
    half = d_h // 2
    z = x[..., :half].astype(np.float64) + 1j * x[..., half:].astype(np.float64)
    ang = pos.astype(np.float64)[:, None, None] * base ** (-2.0 * np.arange(half) / d_h)[None, None, :]
    w = z * np.exp(1j * ang)
    np.testing.assert_allclose(got, np.concatenate([w.real, w.imag], axis=-1), rtol=1e-9, atol=1e-9)


@settings(max_examples=80, deadline=None)
@given(st.data())
def test_gather_matches_fancy_indexing(data):
    """Random kept sets (ascending, as the select produces them) against numpy fancy indexing of the
    rows, the positions and the scores."""
    N, d = data.draw(st.integers(1, 40)), data.draw(st.integers(1, 12))
    rng = np.random.default_rng(data.draw(st.integers(0, 2 ** 31 - 1)))
    idx = np.sort(rng.choice(N, data.draw(st.integers(0, N)), replace=False)).astype(np.int32)
    bits = rng.integers(0, 2 ** 16, (N, d)).astype(np.uint16)
    pos_in = np.sort(rng.choice(10 * N, N, replace=False)).astype(np.int32)
    scores = rng.standard_normal(N).astype(np.float32)
    h_out, pos_out, s_out = oracle.gather_compact(bits, idx, pos_in=pos_in, scores=scores)
    assert np.array_equal(h_out, bits[idx])
    assert np.array_equal(pos_out, pos_in[idx])
    assert np.array_equal(s_out, scores[idx])

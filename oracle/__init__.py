"""Python wrapper of the plain-C fp64 oracle (TEST INFRASTRUCTURE ONLY).

Only the tests, the smoke check and the CPU-baseline leg of the benchmark may
import this package.  The product path (libtokengate and its binding) never
does, and the two share no code.  Arrays are numpy; fp32 inputs carry the exact
values the GPU sees (bf16 widened to fp32), outputs are fp64.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        # TG_ORACLE_LIB lets the mutation test load a deliberately broken copy.
        path = os.environ.get("TG_ORACLE_LIB") or _build.build()
        L = ctypes.CDLL(path)
        i64, i32, dbl = ctypes.c_int64, ctypes.c_int, ctypes.c_double
        vp = ctypes.c_void_p
        L.tgo_kept_count.argtypes = [i64, i64, i64, i64]
        L.tgo_kept_count.restype = i64
        L.tgo_gate_score.argtypes = [vp, i64, i32, i64, vp, i32, dbl, vp, vp, vp, dbl, i32, vp]
        L.tgo_gate_score.restype = i32
        L.tgo_topk_select.argtypes = [vp, i64, i64, i64, i64, vp]
        L.tgo_topk_select.restype = i64
        L.tgo_topk_threshold.argtypes = [vp, i64, i64, i64, i64]
        L.tgo_topk_threshold.restype = dbl
        L.tgo_gather_compact.argtypes = [vp, i64, i32, i64, vp, i64, vp, vp, vp, vp, vp]
        L.tgo_gather_compact.restype = i32
        L.tgo_project.argtypes = [vp, i64, i32, i64, vp, i32, vp]
        L.tgo_project.restype = i32
        L.tgo_rope.argtypes = [vp, i64, i32, i32, vp, dbl, vp]
        L.tgo_rope.restype = i32
        L.tgo_gated_attention.argtypes = [vp, vp, vp, i64, i32, i32, i32, vp, vp, vp, dbl, vp, i64, vp, vp]
        L.tgo_gated_attention.restype = i32
        L.tgo_gated_attention_backward.argtypes = [vp, vp, vp, i64, i32, i32, i32, vp, vp, vp, dbl, vp,
                                                   vp, vp, vp, vp, vp, vp]
        L.tgo_gated_attention_backward.restype = i32
        L.tgo_random_select.argtypes = [i64, i64, i64, i64, ctypes.c_uint64, vp]
        L.tgo_random_select.restype = i64
        L.tgo_splitmix64_stream.argtypes = [ctypes.c_uint64, i64, vp]
        L.tgo_splitmix64_stream.restype = i32
        L.tgo_round_bf16.argtypes = [ctypes.c_float]
        L.tgo_round_bf16.restype = ctypes.c_float
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f32(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float32)


def kept_count(N, doc_begin, doc_end, k_doc):
    return int(lib().tgo_kept_count(N, doc_begin, doc_end, k_doc))


def round_bf16(x: float) -> float:
    return float(lib().tgo_round_bf16(float(x)))


def gate_score(h, W1, w2, b1=None, b2=0.0, gamma=None, eps=1e-6, fold_gamma_bf16=True):
    """s[N] (fp64) for h[N, d] (fp32 values), W1[d_g, d], w2[d_g]."""
    h = _f32(h)
    W1 = _f32(W1)
    w2 = _f32(w2)
    b1 = _f32(b1)
    gamma = _f32(gamma)
    N, d = h.shape
    d_g = W1.shape[0]
    assert W1.shape == (d_g, d) and w2.shape == (d_g,)
    s = np.empty(N, dtype=np.float64)
    rc = lib().tgo_gate_score(_p(h), N, d, d, _p(gamma), int(bool(fold_gamma_bf16)), float(eps),
                              _p(W1), _p(b1), _p(w2), float(b2), d_g, _p(s))
    if rc != 0:
        raise ValueError("tgo_gate_score: bad arguments")
    return s


def topk_select(scores, doc_begin, doc_end, k_doc):
    """Kept indices (int32, ascending) for fp32 scores."""
    s = _f32(scores)
    N = s.shape[0]
    K = kept_count(N, doc_begin, doc_end, k_doc)
    if K < 0:
        raise ValueError("bad span or budget")
    out = np.empty(max(K, 1), dtype=np.int32)
    n = lib().tgo_topk_select(_p(s), N, doc_begin, doc_end, k_doc, _p(out))
    if n != K:
        raise ValueError("tgo_topk_select failed")
    return out[:K]


def splitmix64_stream(state, n):
    """n successive SplitMix64 outputs from `state` (uint64)."""
    out = np.empty(max(n, 1), dtype=np.uint64)
    if lib().tgo_splitmix64_stream(ctypes.c_uint64(state), n, _p(out)) != 0:
        raise ValueError("tgo_splitmix64_stream failed")
    return out[:n]


def random_select(N, doc_begin, doc_end, k_doc, seed):
    """Random-K kept indices (int32, ascending): the k_doc document tokens with the largest
    SplitMix64 keys drawn from `seed`, plus every token outside the span."""
    K = kept_count(N, doc_begin, doc_end, k_doc)
    if K < 0:
        raise ValueError("bad span or budget")
    out = np.empty(max(K, 1), dtype=np.int32)
    n = lib().tgo_random_select(N, doc_begin, doc_end, k_doc, ctypes.c_uint64(seed), _p(out))
    if n != K:
        raise ValueError("tgo_random_select failed")
    return out[:K]


def topk_threshold(scores, doc_begin, doc_end, k_doc):
    s = _f32(scores)
    return float(lib().tgo_topk_threshold(_p(s), s.shape[0], doc_begin, doc_end, k_doc))


def gather_compact(h_bits, idx, pos_in=None, scores=None):
    """h_bits: uint16 [N, d] (bf16 bit patterns).  Returns (h_out, pos_out, s_out)."""
    h_bits = np.ascontiguousarray(h_bits, dtype=np.uint16)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    N, d = h_bits.shape
    K = idx.shape[0]
    h_out = np.empty((K, d), dtype=np.uint16)
    pos_out = np.empty(K, dtype=np.int32)
    s = _f32(scores)
    s_out = np.empty(K, dtype=np.float32) if s is not None else None
    pin = None if pos_in is None else np.ascontiguousarray(pos_in, dtype=np.int32)
    rc = lib().tgo_gather_compact(_p(h_bits), N, d, d, _p(idx), K, _p(pin), _p(s),
                                  _p(h_out), _p(pos_out), _p(s_out))
    if rc != 0:
        raise ValueError("tgo_gather_compact: bad index")
    return h_out, pos_out, s_out


def project(x, W):
    """x [K, d] fp32 values, W [n_out, d] (one row per output feature); returns fp64 [K, n_out]
    = x W^T."""
    x = _f32(x)
    W = _f32(W)
    K, d = x.shape
    n_out = W.shape[0]
    assert W.shape == (n_out, d)
    out = np.empty((max(K, 1), n_out), dtype=np.float64)
    if lib().tgo_project(_p(x), K, d, d, _p(W), n_out, _p(out)) != 0:
        raise ValueError("tgo_project: bad arguments")
    return out[:K]


def rope(x, pos, base=1e6):
    """x: [K, H, d_h] fp32 values; returns fp64 rotated copy."""
    x = _f32(x)
    K, H, d_h = x.shape
    pos = np.ascontiguousarray(pos, dtype=np.int32)
    out = np.empty((K, H, d_h), dtype=np.float64)
    if lib().tgo_rope(_p(x), K, H, d_h, _p(pos), float(base), _p(out)) != 0:
        raise ValueError("tgo_rope: bad arguments")
    return out


def gated_attention(q, k, v, s=None, g=None, tau=1.0, pos=None, rows=None, want_lse=False):
    """q [K,Hq,d_h], k/v [K,Hkv,d_h] fp32 values; returns out fp64 [n_rows,Hq,d_h]
    (and lse [n_rows,Hq] if asked)."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    K, Hq, d_h = q.shape
    Hkv = k.shape[1]
    s = _f32(s)
    g = _f32(g)
    pos = None if pos is None else np.ascontiguousarray(pos, dtype=np.int32)
    rows_a = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    n_rows = K if rows_a is None else rows_a.shape[0]
    out = np.empty((max(n_rows, 1), Hq, d_h), dtype=np.float64)
    lse = np.empty((max(n_rows, 1), Hq), dtype=np.float64) if want_lse else None
    rc = lib().tgo_gated_attention(_p(q), _p(k), _p(v), K, Hq, Hkv, d_h, _p(pos), _p(s), _p(g),
                                   float(tau), _p(rows_a), n_rows, _p(out), _p(lse))
    if rc != 0:
        raise ValueError("tgo_gated_attention: bad arguments")
    out = out[:n_rows]
    if want_lse:
        return out, lse[:n_rows]
    return out


def gated_attention_backward(q, k, v, dout, s=None, g=None, tau=1.0, pos=None):
    """Gradients of sum(dout * out) of gated_attention with respect to every input.
    q [K,Hq,d_h], k/v [K,Hkv,d_h], dout [K,Hq,d_h] fp32 values; returns a dict of fp64 arrays
    dq [K,Hq,d_h], dk, dv [K,Hkv,d_h], ds [K], dg [Hq] and the float dtau."""
    q, k, v, dout = _f32(q), _f32(k), _f32(v), _f32(dout)
    K, Hq, d_h = q.shape
    Hkv = k.shape[1]
    s, g = _f32(s), _f32(g)
    pos = None if pos is None else np.ascontiguousarray(pos, dtype=np.int32)
    dq = np.empty((max(K, 1), Hq, d_h), dtype=np.float64)
    dk = np.empty((max(K, 1), Hkv, d_h), dtype=np.float64)
    dv = np.empty((max(K, 1), Hkv, d_h), dtype=np.float64)
    ds = np.empty(max(K, 1), dtype=np.float64)
    dg = np.empty(Hq, dtype=np.float64)
    dtau = np.empty(1, dtype=np.float64)
    rc = lib().tgo_gated_attention_backward(_p(q), _p(k), _p(v), K, Hq, Hkv, d_h, _p(pos), _p(s), _p(g),
                                            float(tau), _p(dout), _p(dq), _p(dk), _p(dv), _p(ds), _p(dg),
                                            _p(dtau))
    if rc != 0:
        raise ValueError("tgo_gated_attention_backward: bad arguments")
    return {"dq": dq[:K], "dk": dk[:K], "dv": dv[:K], "ds": ds[:K], "dg": dg, "dtau": float(dtau[0])}


__all__ = ["lib", "kept_count", "round_bf16", "gate_score", "topk_select", "topk_threshold",
           "gather_compact", "project", "rope", "gated_attention", "gated_attention_backward"]

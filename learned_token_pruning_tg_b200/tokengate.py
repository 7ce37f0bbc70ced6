"""Thin Python binding of libtokengate (argument marshalling only).

Every function has the name of the C entry point it calls (include/tokengate.h)
and takes torch CUDA tensors; it checks dtypes, shapes and strides, passes raw
device pointers and torch's current CUDA stream, and raises TokenGateError on a
non-OK status.  All computation happens in the library's kernels.  There is no
CPU fallback: if libtokengate.so is missing the first call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libtokengate.so")

TG_OK, TG_ERR_INVALID_ARG, TG_ERR_UNSUPPORTED, TG_ERR_CUDA, TG_ERR_TIMEOUT, TG_ERR_RANGE = range(6)
TG_OP_GATE, TG_OP_SELECT, TG_OP_ATTENTION, TG_OP_ALL, TG_OP_DECODE, TG_OP_ATTENTION_BACKWARD, TG_OP_PROJECT = range(7)
TG_STATUS_SELECT_TIMEOUT, TG_STATUS_GATE_TIMEOUT, TG_STATUS_ATTENTION_TIMEOUT, TG_STATUS_DECODE_TIMEOUT = 1, 2, 4, 8
TG_STATUS_BACKWARD_TIMEOUT, TG_STATUS_PROJECT_TIMEOUT, TG_STATUS_V_RANGE = 16, 32, 64
TG_STATUS_INDEX_RANGE = 128

_lib = None


class TokenGateError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn}: {status_string(status)} (status {status})")


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m learned_token_pruning_tg_b200.build` (no fallback path exists)")
        L = ctypes.CDLL(LIB_PATH)
        vp, i64, i32, f32, f64, sz = (ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_float,
                                      ctypes.c_double, ctypes.c_size_t)
        L.tg_status_string.argtypes = [ctypes.c_int]
        L.tg_status_string.restype = ctypes.c_char_p
        L.tg_version.restype = i32
        L.tg_kept_count.argtypes = [i64, i64, i64, i64]
        L.tg_kept_count.restype = i64
        L.tg_workspace_bytes.argtypes = [ctypes.c_int, i64, i32, i32]
        L.tg_workspace_bytes.restype = sz
        L.tg_gate_score.argtypes = [vp, i64, i32, i64, vp, f32, vp, vp, vp, f32, i32, vp, vp, sz, vp]
        L.tg_topk_select.argtypes = [vp, i64, i64, i64, i64, vp, vp, sz, vp]
        L.tg_gate_score_for_select.argtypes = [vp, i64, i32, i64, vp, f32, vp, vp, vp, f32, i32, vp, i64, i64, vp, sz,
                                               vp]
        L.tg_topk_select_after_gate.argtypes = [vp, i64, i64, i64, i64, vp, vp, sz, vp]
        L.tg_topk_select_after_gate_kept_scores.argtypes = [vp, i64, i64, i64, i64, vp, vp, vp, sz, vp]
        L.tg_topk_select_noalloc.argtypes = [vp, i64, i64, i64, i64, vp, vp]
        L.tg_topk_select_noalloc_status.argtypes = [ctypes.POINTER(ctypes.c_uint32), vp]
        L.tg_random_select.argtypes = [i64, i64, i64, i64, ctypes.c_uint64, vp, vp, sz, vp]
        L.tg_gather_compact.argtypes = [vp, i64, i32, i64, vp, i64, vp, vp, vp, vp, vp, vp]
        L.tg_rope_apply.argtypes = [vp, i64, vp, i64, vp, i64, i32, i32, i32, f64, vp]
        L.tg_gated_attention.argtypes = [vp, i64, vp, i64, vp, i64, i64, i32, i32, i32, vp, vp, f32, vp, vp,
                                         vp, sz, vp]
        L.tg_gated_attention_f16v.argtypes = [vp, i64, vp, i64, vp, i64, i32, i32, i32, vp, vp, f32, vp, vp, vp, sz,
                                              vp]
        L.tg_gated_decode.argtypes = [vp, vp, i64, vp, i64, i64, i32, i32, i32, vp, vp, f32, vp, vp, vp, sz, vp]
        L.tg_project_rope.argtypes = [vp, i64, i32, i64, vp, i32, i32, i32, vp, f64, vp, i64, vp, vp, sz, vp]
        L.tg_project_rope_gather.argtypes = [vp, i64, i32, i64, vp, i64, vp, i32, i32, i32, vp, f64, vp, i64, vp, vp,
                                             sz, vp]
        L.tg_gated_attention_backward.argtypes = [vp, i64, vp, i64, vp, i64, i64, i32, i32, i32, vp, vp, f32, vp,
                                                  vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.tg_debug_set_select_wait_limit.argtypes = [ctypes.c_uint64]
        L.tg_debug_set_cta_pairs.argtypes = [ctypes.c_int]
        L.tg_device_status.argtypes = [vp, ctypes.POINTER(ctypes.c_uint32), vp]
        for fn in ("tg_gate_score", "tg_gate_score_for_select", "tg_topk_select", "tg_topk_select_after_gate", "tg_topk_select_noalloc", "tg_random_select", "tg_gather_compact",
                   "tg_rope_apply",
                   "tg_gated_attention", "tg_gated_attention_f16v", "tg_project_rope",
                   "tg_gated_attention_backward", "tg_gated_decode", "tg_debug_set_select_wait_limit", "tg_device_status",
                   "tg_project_rope_gather", "tg_topk_select_after_gate_kept_scores", "tg_topk_select_noalloc_status",
                   "tg_debug_set_cta_pairs"):
            getattr(L, fn).restype = ctypes.c_int
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().tg_status_string(status).decode()


def _check(fn: str, status: int):
    if status != TG_OK:
        raise TokenGateError(fn, status)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _req(t, name, dtype, dim=None):
    if t is None:
        return
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if dim is not None and t.dim() != dim:
        raise ValueError(f"{name} must have {dim} dims, got {t.dim()}")


def _row_stride(t, name):
    """Token stride (elements) of a [rows, ...] tensor whose trailing dims are dense."""
    inner = 1
    for d in range(t.dim() - 1, 0, -1):
        if t.size(d) != 1 and t.stride(d) != inner:
            raise ValueError(f"{name}: trailing dims must be contiguous")
        inner *= t.size(d)
    return t.stride(0) if t.size(0) > 1 else max(inner, 1)


def tg_version() -> int:
    return int(lib().tg_version())


def tg_kept_count(N: int, doc_begin: int, doc_end: int, k_doc: int) -> int:
    return int(lib().tg_kept_count(N, doc_begin, doc_end, k_doc))


def tg_workspace_bytes(op: int, N: int, d: int = 0, d_g: int = 0) -> int:
    return int(lib().tg_workspace_bytes(op, N, d, d_g))


def new_workspace(N: int, d: int = 0, d_g: int = 0, op: int = TG_OP_ALL, device=None) -> torch.Tensor:
    """A zero-filled device workspace usable by every call (torch allocates it)."""
    n = tg_workspace_bytes(op, N, d, d_g)
    return torch.zeros(max(n, 256), dtype=torch.uint8, device=device or "cuda")


def tg_gate_score(h, W1, w2, scores, workspace, b1=None, b2: float = 0.0, rms_weight=None,
                  eps: float = 1e-6, stream=None):
    _req(h, "h", torch.bfloat16, 2)
    _req(W1, "W1", torch.bfloat16, 2)
    _req(w2, "w2", torch.float32, 1)
    _req(scores, "scores", torch.float32, 1)
    _req(b1, "b1", torch.float32, 1)
    _req(rms_weight, "rms_weight", torch.bfloat16, 1)
    N, d = h.shape
    d_g = W1.shape[0]
    if h.stride(1) != 1 or not W1.is_contiguous() or not w2.is_contiguous() or not scores.is_contiguous():
        raise ValueError("h rows, W1, w2 and scores must be dense")
    if W1.shape[1] != d or w2.shape[0] != d_g or scores.shape[0] != N:
        raise ValueError("shape mismatch")
    ld_h = h.stride(0) if N > 1 else d
    _check("tg_gate_score", lib().tg_gate_score(
        _ptr(h), N, d, ld_h, _ptr(rms_weight), eps, _ptr(W1), _ptr(b1), _ptr(w2), b2, d_g,
        _ptr(scores), _ptr(workspace), workspace.numel(), _stream(stream)))
    return scores


def _gate_args(h, W1, w2, scores, b1, rms_weight):
    _req(h, "h", torch.bfloat16, 2)
    _req(W1, "W1", torch.bfloat16, 2)
    _req(w2, "w2", torch.float32, 1)
    _req(scores, "scores", torch.float32, 1)
    _req(b1, "b1", torch.float32, 1)
    _req(rms_weight, "rms_weight", torch.bfloat16, 1)
    N, d = h.shape
    d_g = W1.shape[0]
    if h.stride(1) != 1 or not W1.is_contiguous() or not w2.is_contiguous() or not scores.is_contiguous():
        raise ValueError("h rows, W1, w2 and scores must be dense")
    if W1.shape[1] != d or w2.shape[0] != d_g or scores.shape[0] != N:
        raise ValueError("shape mismatch")
    return N, d, (h.stride(0) if N > 1 else d), d_g


def tg_gate_score_for_select(h, W1, w2, scores, workspace, doc_begin: int, doc_end: int, b1=None, b2: float = 0.0,
                             rms_weight=None, eps: float = 1e-6, stream=None):
    """tg_gate_score that also leaves the select's first radix pass over [doc_begin, doc_end) in the
    workspace, for a tg_topk_select_after_gate on the same workspace right after it."""
    N, d, ld_h, d_g = _gate_args(h, W1, w2, scores, b1, rms_weight)
    _check("tg_gate_score_for_select", lib().tg_gate_score_for_select(
        _ptr(h), N, d, ld_h, _ptr(rms_weight), eps, _ptr(W1), _ptr(b1), _ptr(w2), b2, d_g,
        _ptr(scores), doc_begin, doc_end, _ptr(workspace), workspace.numel(), _stream(stream)))
    return scores


def tg_topk_select_after_gate(scores, doc_begin: int, doc_end: int, k_doc: int, kept_idx, workspace, stream=None):
    """tg_topk_select starting from the first radix pass tg_gate_score_for_select left in the workspace."""
    _req(scores, "scores", torch.float32, 1)
    _req(kept_idx, "kept_idx", torch.int32, 1)
    N = scores.shape[0]
    K = tg_kept_count(N, doc_begin, doc_end, k_doc)
    if K < 0:
        raise TokenGateError("tg_topk_select_after_gate", TG_ERR_INVALID_ARG)
    if kept_idx.numel() < K or not scores.is_contiguous() or not kept_idx.is_contiguous():
        raise ValueError("kept_idx too small or not contiguous")
    _check("tg_topk_select_after_gate", lib().tg_topk_select_after_gate(
        _ptr(scores), N, doc_begin, doc_end, k_doc, _ptr(kept_idx), _ptr(workspace), workspace.numel(),
        _stream(stream)))
    return kept_idx


def tg_topk_select_after_gate_kept_scores(scores, doc_begin: int, doc_end: int, k_doc: int, kept_idx, s_kept,
                                          workspace, stream=None):
    """tg_topk_select_after_gate that also writes s_kept[i] = scores[kept_idx[i]]."""
    _req(scores, "scores", torch.float32, 1)
    _req(kept_idx, "kept_idx", torch.int32, 1)
    _req(s_kept, "s_kept", torch.float32, 1)
    N = scores.shape[0]
    K = tg_kept_count(N, doc_begin, doc_end, k_doc)
    if K < 0:
        raise TokenGateError("tg_topk_select_after_gate_kept_scores", TG_ERR_INVALID_ARG)
    if (kept_idx.numel() < K or s_kept.numel() < K or not scores.is_contiguous() or not kept_idx.is_contiguous()
            or not s_kept.is_contiguous()):
        raise ValueError("kept_idx or s_kept too small or not contiguous")
    _check("tg_topk_select_after_gate_kept_scores", lib().tg_topk_select_after_gate_kept_scores(
        _ptr(scores), N, doc_begin, doc_end, k_doc, _ptr(kept_idx), _ptr(s_kept), _ptr(workspace),
        workspace.numel(), _stream(stream)))
    return kept_idx, s_kept


def tg_topk_select(scores, doc_begin: int, doc_end: int, k_doc: int, kept_idx, workspace, stream=None):
    _req(scores, "scores", torch.float32, 1)
    _req(kept_idx, "kept_idx", torch.int32, 1)
    N = scores.shape[0]
    K = tg_kept_count(N, doc_begin, doc_end, k_doc)
    if K < 0:
        raise TokenGateError("tg_topk_select", TG_ERR_INVALID_ARG)
    if kept_idx.numel() < K or not scores.is_contiguous() or not kept_idx.is_contiguous():
        raise ValueError("kept_idx too small or not contiguous")
    _check("tg_topk_select", lib().tg_topk_select(
        _ptr(scores), N, doc_begin, doc_end, k_doc, _ptr(kept_idx), _ptr(workspace), workspace.numel(),
        _stream(stream)))
    return kept_idx


def tg_topk_select_noalloc(scores, doc_begin: int, doc_end: int, k_doc: int, kept_idx, stream=None):
    """tg_topk_select without a workspace: for callers that cannot allocate device memory
    when they select.  Its scratch is a static array inside the library shared by every call,
    so calls must not overlap on the GPU."""
    _req(scores, "scores", torch.float32, 1)
    _req(kept_idx, "kept_idx", torch.int32, 1)
    N = scores.shape[0]
    K = tg_kept_count(N, doc_begin, doc_end, k_doc)
    if K < 0:
        raise TokenGateError("tg_topk_select_noalloc", TG_ERR_INVALID_ARG)
    if kept_idx.numel() < K or not scores.is_contiguous() or not kept_idx.is_contiguous():
        raise ValueError("kept_idx too small or not contiguous")
    _check("tg_topk_select_noalloc", lib().tg_topk_select_noalloc(
        _ptr(scores), N, doc_begin, doc_end, k_doc, _ptr(kept_idx), _stream(stream)))
    return kept_idx


def tg_topk_select_noalloc_status(stream=None) -> int:
    """Raw TG_STATUS_* bits the last tg_topk_select_noalloc call on the current device left (synchronizes
    the stream); raises only if the read fails."""
    w = ctypes.c_uint32(0)
    st = lib().tg_topk_select_noalloc_status(ctypes.byref(w), _stream(stream))
    if st not in (TG_OK, TG_ERR_TIMEOUT):
        raise TokenGateError("tg_topk_select_noalloc_status", st)
    return int(w.value)


def tg_random_select(N: int, doc_begin: int, doc_end: int, k_doc: int, seed: int, kept_idx, workspace, stream=None):
    """The random-K selector: k_doc document tokens drawn from SplitMix64(seed), plus every token outside
    the span, ascending (same output layout as tg_topk_select)."""
    _req(kept_idx, "kept_idx", torch.int32, 1)
    K = tg_kept_count(N, doc_begin, doc_end, k_doc)
    if K < 0:
        raise TokenGateError("tg_random_select", TG_ERR_INVALID_ARG)
    if kept_idx.numel() < K or not kept_idx.is_contiguous():
        raise ValueError("kept_idx too small or not contiguous")
    _check("tg_random_select", lib().tg_random_select(
        N, doc_begin, doc_end, k_doc, ctypes.c_uint64(seed & ((1 << 64) - 1)), _ptr(kept_idx), _ptr(workspace),
        workspace.numel(), _stream(stream)))
    return kept_idx


def tg_gather_compact(h, kept_idx, h_out, pos_out, pos_in=None, scores=None, s_out=None, stream=None):
    _req(h, "h", torch.bfloat16, 2)
    _req(h_out, "h_out", torch.bfloat16, 2)
    _req(kept_idx, "kept_idx", torch.int32, 1)
    _req(pos_out, "pos_out", torch.int32, 1)
    _req(pos_in, "pos_in", torch.int32, 1)
    _req(scores, "scores", torch.float32, 1)
    _req(s_out, "s_out", torch.float32, 1)
    N, d = h.shape
    K = kept_idx.shape[0]
    if h.stride(1) != 1 or not h_out.is_contiguous() or h_out.shape != (K, d):
        raise ValueError("h rows must be dense and h_out [K, d] contiguous")
    ld_h = h.stride(0) if N > 1 else d
    _check("tg_gather_compact", lib().tg_gather_compact(
        _ptr(h), N, d, ld_h, _ptr(kept_idx), K, _ptr(pos_in), _ptr(scores), _ptr(h_out), _ptr(pos_out),
        _ptr(s_out), _stream(stream)))
    return h_out, pos_out, s_out


def tg_rope_apply(q, k, pos, base: float = 1e6, stream=None):
    """In place on q [K, Hq, d_h] and k [K, Hkv, d_h] (token stride may be padded)."""
    _req(q, "q", torch.bfloat16, 3)
    _req(k, "k", torch.bfloat16, 3)
    _req(pos, "pos", torch.int32, 1)
    K, Hq, d_h = q.shape
    Hkv = k.shape[1]
    _check("tg_rope_apply", lib().tg_rope_apply(
        _ptr(q), _row_stride(q, "q"), _ptr(k), _row_stride(k, "k"), _ptr(pos), K, Hq, Hkv, d_h, base,
        _stream(stream)))
    return q, k


def tg_gated_attention(q, k, v, out, workspace, s_kept=None, gain=None, tau: float = 1.0, lse=None,
                       stream=None):
    _req(q, "q", torch.bfloat16, 3)
    _req(k, "k", torch.bfloat16, 3)
    _req(v, "v", torch.bfloat16, 3)
    _req(out, "out", torch.bfloat16, 3)
    _req(s_kept, "s_kept", torch.float32, 1)
    _req(gain, "gain", torch.float32, 1)
    _req(lse, "lse", torch.float32, 2)
    K, Hq, d_h = q.shape
    Hkv = k.shape[1]
    if not out.is_contiguous() or out.shape != (K, Hq, d_h):
        raise ValueError("out must be a contiguous [K, Hq, d_h] tensor")
    _check("tg_gated_attention", lib().tg_gated_attention(
        _ptr(q), _row_stride(q, "q"), _ptr(k), _row_stride(k, "k"), _ptr(v), _row_stride(v, "v"), K, Hq, Hkv,
        d_h, _ptr(s_kept), _ptr(gain), tau, _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(),
        _stream(stream)))
    return out


def tg_gated_attention_f16v(q, k, v16, out, workspace, s_kept=None, gain=None, tau: float = 1.0, lse=None,
                            stream=None):
    """tg_gated_attention over an fp16 copy of V (v16 [K, Hkv, d_h] or [K, Hkv d_h] fp16, dense), as
    tg_project_rope writes it."""
    _req(q, "q", torch.bfloat16, 3)
    _req(k, "k", torch.bfloat16, 3)
    _req(v16, "v16", torch.float16)
    _req(out, "out", torch.bfloat16, 3)
    _req(s_kept, "s_kept", torch.float32, 1)
    _req(gain, "gain", torch.float32, 1)
    _req(lse, "lse", torch.float32, 2)
    K, Hq, d_h = q.shape
    Hkv = k.shape[1]
    if not out.is_contiguous() or out.shape != (K, Hq, d_h):
        raise ValueError("out must be a contiguous [K, Hq, d_h] tensor")
    if not v16.is_contiguous() or v16.numel() != K * Hkv * d_h or v16.shape[0] != K:
        raise ValueError("v16 must be a contiguous [K, Hkv, d_h] fp16 tensor")
    _check("tg_gated_attention_f16v", lib().tg_gated_attention_f16v(
        _ptr(q), _row_stride(q, "q"), _ptr(k), _row_stride(k, "k"), _ptr(v16), K, Hq, Hkv, d_h, _ptr(s_kept),
        _ptr(gain), tau, _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(), _stream(stream)))
    return out


def tg_gated_attention_backward(q, k, v, out, dout, lse, dq, dk, dv, workspace, s_kept=None, gain=None,
                                tau: float = 1.0, ds=None, dg=None, dtau=None, stream=None):
    """Gradients of tg_gated_attention: out, dout [K, Hq, d_h] and lse [Hq, K] from the forward call;
    writes dq [K, Hq, d_h], dk and dv [K, Hkv, d_h] (bf16) and, when given, ds [K], dg [Hq], dtau [1]
    (fp32)."""
    for t, n, r in ((q, "q", 3), (k, "k", 3), (v, "v", 3), (out, "out", 3), (dout, "dout", 3), (dq, "dq", 3),
                    (dk, "dk", 3), (dv, "dv", 3)):
        _req(t, n, torch.bfloat16, r)
    for t, n, r in ((lse, "lse", 2), (s_kept, "s_kept", 1), (gain, "gain", 1), (ds, "ds", 1), (dg, "dg", 1),
                    (dtau, "dtau", 1)):
        _req(t, n, torch.float32, r)
    if lse is None:
        raise ValueError("lse (the forward's log-sum-exp) is required")
    K, Hq, d_h = q.shape
    Hkv = k.shape[1]
    for t, n, shape in ((out, "out", (K, Hq, d_h)), (dout, "dout", (K, Hq, d_h)), (dq, "dq", (K, Hq, d_h)),
                        (dk, "dk", (K, Hkv, d_h)), (dv, "dv", (K, Hkv, d_h)), (lse, "lse", (Hq, K))):
        if not t.is_contiguous() or tuple(t.shape) != shape:
            raise ValueError(f"{n} must be a contiguous {list(shape)} tensor")
    _check("tg_gated_attention_backward", lib().tg_gated_attention_backward(
        _ptr(q), _row_stride(q, "q"), _ptr(k), _row_stride(k, "k"), _ptr(v), _row_stride(v, "v"), K, Hq, Hkv,
        d_h, _ptr(s_kept), _ptr(gain), tau, _ptr(out), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv),
        _ptr(ds), _ptr(dg), _ptr(dtau), _ptr(workspace), workspace.numel(), _stream(stream)))
    return dq, dk, dv


def tg_project_rope(x, W, pos, qkv, workspace, Hq: int, Hkv: int, d_h: int, base: float = 1e6, v16=None,
                    stream=None):
    """qkv [K, (Hq + 2 Hkv) d_h] = x [K, d] W^T with RoPE at pos on the query and key heads; the value
    heads also into v16 [K, Hkv d_h] fp16 when given."""
    _req(x, "x", torch.bfloat16, 2)
    _req(W, "W", torch.bfloat16, 2)
    _req(pos, "pos", torch.int32, 1)
    _req(qkv, "qkv", torch.bfloat16, 2)
    _req(v16, "v16", torch.float16, 2)
    K, d = x.shape
    cols = (Hq + 2 * Hkv) * d_h
    if tuple(W.shape) != (cols, d) or not W.is_contiguous():
        raise ValueError("W must be a contiguous [(Hq + 2 Hkv) d_h, d] tensor")
    if qkv.shape[0] != K or qkv.shape[1] != cols or qkv.stride(1) != 1 or pos.shape[0] < K:
        raise ValueError("shape mismatch")
    if v16 is not None and (tuple(v16.shape) != (K, Hkv * d_h) or not v16.is_contiguous()):
        raise ValueError("v16 must be a contiguous [K, Hkv d_h] tensor")
    _check("tg_project_rope", lib().tg_project_rope(
        _ptr(x), K, d, x.stride(0), _ptr(W), Hq, Hkv, d_h, _ptr(pos), float(base), _ptr(qkv), qkv.stride(0),
        _ptr(v16), _ptr(workspace), workspace.numel(), _stream(stream)))
    return qkv


def tg_project_rope_gather(h, rows, W, pos, qkv, workspace, Hq: int, Hkv: int, d_h: int, base: float = 1e6,
                           v16=None, stream=None):
    """tg_project_rope over the rows h[rows[r]] (rows [K] int32), gathered into the GEMM's operand tiles."""
    _req(h, "h", torch.bfloat16, 2)
    _req(rows, "rows", torch.int32, 1)
    _req(W, "W", torch.bfloat16, 2)
    _req(pos, "pos", torch.int32, 1)
    _req(qkv, "qkv", torch.bfloat16, 2)
    _req(v16, "v16", torch.float16, 2)
    N, d = h.shape
    K = qkv.shape[0]
    cols = (Hq + 2 * Hkv) * d_h
    if tuple(W.shape) != (cols, d) or not W.is_contiguous():
        raise ValueError("W must be a contiguous [(Hq + 2 Hkv) d_h, d] tensor")
    if (qkv.shape[1] != cols or qkv.stride(1) != 1 or pos.shape[0] < K or rows.shape[0] < K
            or not rows.is_contiguous()):
        raise ValueError("shape mismatch")
    if v16 is not None and (tuple(v16.shape) != (K, Hkv * d_h) or not v16.is_contiguous()):
        raise ValueError("v16 must be a contiguous [K, Hkv d_h] tensor")
    _check("tg_project_rope_gather", lib().tg_project_rope_gather(
        _ptr(h), N, d, h.stride(0), _ptr(rows), K, _ptr(W), Hq, Hkv, d_h, _ptr(pos), float(base), _ptr(qkv),
        qkv.stride(0), _ptr(v16), _ptr(workspace), workspace.numel(), _stream(stream)))
    return qkv


def tg_gated_decode(q, k_cache, v_cache, out, workspace, s_cache=None, gain=None, tau: float = 1.0, lse=None,
                    stream=None):
    """One decoding step: q [Hq, d_h] over the T rows of k_cache, v_cache [T, Hkv, d_h] (token stride
    may be padded); out [Hq, d_h]."""
    _req(q, "q", torch.bfloat16, 2)
    _req(k_cache, "k_cache", torch.bfloat16, 3)
    _req(v_cache, "v_cache", torch.bfloat16, 3)
    _req(out, "out", torch.bfloat16, 2)
    _req(s_cache, "s_cache", torch.float32, 1)
    _req(gain, "gain", torch.float32, 1)
    _req(lse, "lse", torch.float32, 1)
    Hq, d_h = q.shape
    T, Hkv = k_cache.shape[0], k_cache.shape[1]
    if not q.is_contiguous() or not out.is_contiguous() or out.shape != q.shape:
        raise ValueError("q and out must be contiguous [Hq, d_h] tensors")
    if v_cache.shape != k_cache.shape or (s_cache is not None and s_cache.shape[0] < T):
        raise ValueError("shape mismatch")
    _check("tg_gated_decode", lib().tg_gated_decode(
        _ptr(q), _ptr(k_cache), _row_stride(k_cache, "k_cache"), _ptr(v_cache), _row_stride(v_cache, "v_cache"), T,
        Hq, Hkv, d_h, _ptr(s_cache), _ptr(gain), tau, _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(),
        _stream(stream)))
    return out


def tg_debug_set_select_wait_limit(ns: int) -> None:
    """Test hook: the select's grid-barrier time limit on the current device (0 = the default)."""
    _check("tg_debug_set_select_wait_limit", lib().tg_debug_set_select_wait_limit(ctypes.c_uint64(ns)))


def tg_debug_set_cta_pairs(enabled: bool) -> None:
    """Test hook: False makes the gate (d_g = 256) and the projection run their one-CTA kernels."""
    _check("tg_debug_set_cta_pairs", lib().tg_debug_set_cta_pairs(1 if enabled else 0))


def tg_device_status(workspace, stream=None) -> int:
    """Raw TG_STATUS_* bits of the workspace (synchronizes the stream); raises only if the read fails."""
    w = ctypes.c_uint32(0)
    st = lib().tg_device_status(_ptr(workspace), ctypes.byref(w), _stream(stream))
    if st not in (TG_OK, TG_ERR_TIMEOUT, TG_ERR_RANGE):
        raise TokenGateError("tg_device_status", st)
    return int(w.value)

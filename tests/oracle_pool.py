"""Run the single-threaded oracle on row chunks in parallel worker processes.

The pool uses the spawn start method, so it is safe to create after CUDA has
been initialised in the parent.  Each worker runs the unmodified oracle on its
chunk; results are concatenated in row order.
"""
import atexit
import concurrent.futures as cf
import multiprocessing as mp
import os

import numpy as np

_pool = None


def pool():
    global _pool
    if _pool is None:
        n = max(1, min(16, (os.cpu_count() or 2) - 1))
        _pool = cf.ProcessPoolExecutor(max_workers=n, mp_context=mp.get_context("spawn"))
        atexit.register(_pool.shutdown, wait=True)
    return _pool


def _gate_chunk(h, W1, w2, b1, b2, gamma, eps):
    import oracle
    return oracle.gate_score(h, W1, w2, b1=b1, b2=b2, gamma=gamma, eps=eps, fold_gamma_bf16=True)


def gate_scores(h, W1, w2, b1=None, b2=0.0, gamma=None, eps=1e-6, chunk=4096):
    """Oracle gate scores of every row of h (fp32 numpy) using all host cores."""
    futs = [pool().submit(_gate_chunk, h[lo:lo + chunk], W1, w2, b1, b2, gamma, eps)
            for lo in range(0, h.shape[0], chunk)]
    return np.concatenate([f.result() for f in futs])


def _attn_chunk(q, k, v, s, g, tau, pos, rows):
    import oracle
    return oracle.gated_attention(q, k, v, s=s, g=g, tau=tau, pos=pos, rows=rows)


def gated_attention(q, k, v, s=None, g=None, tau=1.0, pos=None, rows=None, n_chunks=None):
    """Oracle attention for the given rows (default all), split across workers."""
    rows = np.arange(q.shape[0]) if rows is None else np.asarray(rows)
    n = n_chunks or max(1, min(64, len(rows)))
    parts = np.array_split(rows, n)
    futs = [pool().submit(_attn_chunk, q, k, v, s, g, tau, pos, p) for p in parts if len(p)]
    return np.concatenate([f.result() for f in futs])


def _bwd_group(q, k, v, dout, s, g, tau):
    import oracle
    return oracle.gated_attention_backward(q, k, v, dout, s=s, g=g, tau=tau)


def gated_attention_backward(q, k, v, dout, s=None, g=None, tau=1.0):
    """Oracle backward split by KV head: each worker runs one KV head and its query heads (an
    independent problem), and the parts are put back together (ds and dtau summed)."""
    K, Hq, d_h = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    futs = [pool().submit(_bwd_group, np.ascontiguousarray(q[:, j * G:(j + 1) * G]),
                          np.ascontiguousarray(k[:, j:j + 1]), np.ascontiguousarray(v[:, j:j + 1]),
                          np.ascontiguousarray(dout[:, j * G:(j + 1) * G]), s,
                          None if g is None else np.ascontiguousarray(g[j * G:(j + 1) * G]), tau)
            for j in range(Hkv)]
    parts = [f.result() for f in futs]
    return {"dq": np.concatenate([p["dq"] for p in parts], axis=1),
            "dk": np.concatenate([p["dk"] for p in parts], axis=1),
            "dv": np.concatenate([p["dv"] for p in parts], axis=1),
            "ds": np.sum([p["ds"] for p in parts], axis=0),
            "dg": np.concatenate([p["dg"] for p in parts]),
            "dtau": float(np.sum([p["dtau"] for p in parts]))}


def _project_chunk(x, W):
    import oracle
    return oracle.project(x, W)


def project(x, W, chunk=None):
    """Oracle projection x W^T (fp64) of every row of x, row chunks split across workers."""
    n_workers = pool()._max_workers
    chunk = chunk or max(64, -(-x.shape[0] // (2 * n_workers)))
    futs = [pool().submit(_project_chunk, x[lo:lo + chunk], W) for lo in range(0, x.shape[0], chunk)]
    return np.concatenate([f.result() for f in futs]) if futs else np.empty((0, W.shape[0]))

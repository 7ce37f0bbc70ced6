"""The C-ABI library builds, loads, and exports every entry point include/*.h declares.

Host-only checks (no device work): kept count, workspace sizes, status strings.
"""
import ctypes
import glob
import os
import re

import pytest

from learned_token_pruning_tg_b200 import build as tg_build
from learned_token_pruning_tg_b200 import tokengate as tg

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names |= set(re.findall(r"\b(tg_[a-z0-9_]+)\s*\(", src))
    return sorted(names)


@pytest.fixture(scope="module")
def lib():
    tg_build.build()
    return tg.lib()


def test_every_declared_symbol_is_exported(lib):
    names = _declared()
    assert "tg_gate_score" in names and "tg_gated_attention" in names
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"


def test_only_tg_symbols_exported():
    out = os.popen(f"nm -D --defined-only {tg.LIB_PATH}").read().split("\n")
    syms = [l.split()[-1] for l in out if l.strip()]
    bad = [s for s in syms if not s.startswith("tg_")]
    assert not bad, bad


def test_host_only_calls(lib):
    assert tg.tg_kept_count(131072, 0, 130560, 4096) == 4608
    assert tg.tg_kept_count(16384, 0, 16000, 1024) == 1408
    assert tg.tg_kept_count(10, 2, 8, 100) == 10
    assert tg.tg_kept_count(10, 2, 11, 1) == -1
    assert tg.tg_kept_count(10, 3, 2, 1) == -1
    assert tg.tg_kept_count(10, 2, 8, -1) == -1
    assert tg.tg_workspace_bytes(tg.TG_OP_SELECT, 131072) > 256
    assert tg.tg_workspace_bytes(tg.TG_OP_GATE, 131072, 2048, 256) >= 2048 * 256 * 2
    assert tg.tg_workspace_bytes(tg.TG_OP_ALL, 131072, 2048, 256) >= tg.tg_workspace_bytes(tg.TG_OP_SELECT, 1)
    assert tg.tg_workspace_bytes(tg.TG_OP_GATE, -1, 2048, 256) == 0
    # attention: N = K kept tokens, d = Hkv * d_h (an fp16 copy of V lives in the workspace)
    attn = tg.tg_workspace_bytes(tg.TG_OP_ATTENTION, 4608, 1024)
    assert attn >= 4608 * 1024 * 2 and attn % 16 == 0
    assert tg.tg_workspace_bytes(tg.TG_OP_ATTENTION, 4608, 0) == 0
    assert tg.tg_workspace_bytes(tg.TG_OP_ALL, 4608, 1024, 256) >= attn
    assert tg.tg_workspace_bytes(tg.TG_OP_ALL, 4608, 1024, 256) >= tg.tg_workspace_bytes(tg.TG_OP_GATE, 4608, 1024, 256)
    assert tg.status_string(tg.TG_OK) == "ok"
    assert "timed out" in tg.status_string(tg.TG_ERR_TIMEOUT)
    assert "fp16" in tg.status_string(tg.TG_ERR_RANGE)
    assert tg.tg_version() >= 100


def test_argument_errors_before_launch(lib):
    # Host validation rejects bad arguments without touching the device.
    vp = ctypes.c_void_p
    assert lib.tg_topk_select(None, 10, 2, 11, 1, None, None, 0, None) == tg.TG_ERR_INVALID_ARG
    assert lib.tg_topk_select(vp(16), 10, 2, 8, 3, None, None, 0, None) == tg.TG_ERR_INVALID_ARG
    assert lib.tg_gather_compact(vp(16), 10, 12, 12, None, 3, None, None, vp(16), vp(16), None,
                                 None) == tg.TG_ERR_INVALID_ARG
    assert lib.tg_gather_compact(vp(16), 10, 12, 12, vp(16), 3, None, None, vp(16), vp(16), None,
                                 None) == tg.TG_ERR_UNSUPPORTED          # d % 8 != 0
    assert lib.tg_rope_apply(vp(16), 96 * 2, vp(16), 96, vp(16), 4, 2, 1, 96, 1e6,
                             None) == tg.TG_ERR_UNSUPPORTED              # d_h = 96
    assert lib.tg_gate_score(vp(16), 10, 100, 100, None, 1e-6, vp(16), None, vp(16), 0.0, 64, vp(16),
                             vp(256), 1 << 20, None) == tg.TG_ERR_UNSUPPORTED   # d % 64 != 0
    assert lib.tg_gate_score(vp(16), 10, 128, 128, None, 1e-6, vp(16), None, vp(16), 0.0, 96, vp(16),
                             vp(256), 1 << 20, None) == tg.TG_ERR_UNSUPPORTED   # d_g = 96
    assert lib.tg_gated_attention(vp(16), 128, vp(16), 128, vp(16), 128, 5, 3, 2, 64, None, None, 1.0,
                                  vp(16), None, vp(256), 256, None) == tg.TG_ERR_INVALID_ARG  # Hq % Hkv
    assert lib.tg_gated_attention(vp(16), 96, vp(16), 96, vp(16), 96, 5, 1, 1, 96, None, None, 1.0,
                                  vp(16), None, vp(256), 256, None) == tg.TG_ERR_UNSUPPORTED  # d_h = 96
    assert lib.tg_gated_attention(vp(17), 128, vp(16), 128, vp(16), 128, 5, 2, 2, 64, None, None, 1.0,
                                  vp(16), None, vp(256), 256, None) == tg.TG_ERR_INVALID_ARG  # misaligned
    for tau in (0.0, -1.0, float("nan")):   # the temperature must be positive
        assert lib.tg_gated_attention(vp(16), 128, vp(16), 128, vp(16), 128, 5, 2, 2, 64, None, None, tau,
                                      vp(16), None, vp(256), 1 << 20, None) == tg.TG_ERR_INVALID_ARG
    assert lib.tg_gated_attention(vp(16), 128, vp(16), 128, vp(16), 128, 5, 2, 2, 64, None, None, 1.0,
                                  vp(16), None, vp(256), 256, None) == tg.TG_ERR_INVALID_ARG  # workspace too small
    # the fp16-V variant: same checks, and a workspace of the status header only is enough
    f16v = lib.tg_gated_attention_f16v
    assert f16v(vp(16), 128, vp(16), 128, vp(16), 5, 3, 2, 64, None, None, 1.0, vp(16), None, vp(256), 1 << 20,
                None) == tg.TG_ERR_INVALID_ARG    # Hq % Hkv
    assert f16v(vp(16), 96, vp(16), 96, vp(16), 5, 1, 1, 96, None, None, 1.0, vp(16), None, vp(256), 1 << 20,
                None) == tg.TG_ERR_UNSUPPORTED    # d_h = 96
    assert f16v(vp(16), 128, vp(16), 128, vp(24), 5, 2, 2, 64, None, None, 1.0, vp(16), None, vp(256), 1 << 20,
                None) == tg.TG_ERR_INVALID_ARG    # v16 misaligned
    assert f16v(vp(16), 128, vp(16), 128, None, 5, 2, 2, 64, None, None, 1.0, vp(16), None, vp(256), 1 << 20,
                None) == tg.TG_ERR_INVALID_ARG    # no v16
    assert f16v(vp(16), 128, vp(16), 128, vp(16), 5, 2, 2, 64, None, None, -1.0, vp(16), None, vp(256), 1 << 20,
                None) == tg.TG_ERR_INVALID_ARG    # tau <= 0
    assert f16v(vp(16), 128, vp(16), 128, vp(16), 5, 2, 2, 64, None, None, 1.0, vp(16), None, vp(256), 16,
                None) == tg.TG_ERR_INVALID_ARG    # workspace too small
    assert f16v(vp(16), 128, vp(16), 128, vp(16), 0, 2, 2, 64, None, None, 1.0, vp(16), None, vp(256), 16,
                None) == tg.TG_OK                 # K = 0: nothing to do
    assert tg.tg_workspace_bytes(tg.TG_OP_ATTENTION, 0, 1024) < tg.tg_workspace_bytes(tg.TG_OP_ATTENTION, 4608, 1024)


def test_decode_and_random_select_argument_errors(lib):
    vp = ctypes.c_void_p
    INV, UNS = tg.TG_ERR_INVALID_ARG, tg.TG_ERR_UNSUPPORTED
    big = tg.tg_workspace_bytes(tg.TG_OP_DECODE, 0, 64, 0)
    assert big > 0

    def dec(q=16, ldk=1024, ldv=1024, T=100, Hq=16, Hkv=8, d_h=128, tau=1.0, ws_bytes=big, out=16):
        return lib.tg_gated_decode(vp(q), vp(4096), ldk, vp(8192), ldv, T, Hq, Hkv, d_h, None, None, tau,
                                   vp(out) if out else None, None, vp(256), ws_bytes, None)

    assert dec(T=0) == INV
    assert dec(Hq=12, Hkv=8) == INV                 # Hq % Hkv
    assert dec(tau=float("nan")) == INV
    assert dec(out=0) == INV                        # no output
    assert dec(d_h=96) == UNS
    assert dec(Hq=16, Hkv=1, ldk=128, ldv=128) == UNS   # 16 query heads per KV head
    assert dec(Hq=128, Hkv=128, ldk=128 * 128, ldv=128 * 128, ws_bytes=1 << 30) == UNS   # Hkv > 64
    assert dec(q=24) == INV                         # q not 16-byte aligned
    assert dec(ldk=1028) == INV                     # stride not a multiple of 8 elements
    assert dec(ldv=512) == INV                      # stride shorter than a row
    assert dec(ws_bytes=tg.tg_workspace_bytes(tg.TG_OP_DECODE, 0, 16, 0) - 16) == INV
    rs = lib.tg_random_select
    assert rs(10, 2, 11, 1, 7, vp(16), vp(256), 1 << 20, None) == INV      # span past N
    assert rs(10, 2, 8, -1, 7, vp(16), vp(256), 1 << 20, None) == INV      # negative budget
    assert rs(10, 2, 8, 3, 7, None, vp(256), 1 << 20, None) == INV         # no output
    assert rs(1000, 0, 900, 10, 7, vp(16), vp(256), 16, None) == INV       # workspace too small
    assert rs(1000, 0, 900, 10, 7, vp(16), None, 1 << 20, None) == INV     # no workspace
    assert rs(0, 0, 0, 5, 7, None, None, 0, None) == tg.TG_OK              # nothing to keep


def test_backward_workspace_and_argument_errors(lib):
    vp = ctypes.c_void_p
    INV, UNS = tg.TG_ERR_INVALID_ARG, tg.TG_ERR_UNSUPPORTED
    # workspace: lse2 and D per head and padded row, ds per KV head and padded row, dg and dtau partials
    ws = tg.tg_workspace_bytes(tg.TG_OP_ATTENTION_BACKWARD, 4608, 16, 8)
    assert ws >= 256 + 4 * (2 * 16 * 4608 + 8 * 4608 + 2 * 16 * 36) and ws % 256 == 0
    assert tg.tg_workspace_bytes(tg.TG_OP_ATTENTION_BACKWARD, 4608, 16, 3) == 0   # Hq % Hkv
    assert tg.tg_workspace_bytes(tg.TG_OP_ATTENTION_BACKWARD, -1, 16, 8) == 0
    big = tg.tg_workspace_bytes(tg.TG_OP_ATTENTION_BACKWARD, 300, 16, 8)

    def bwd(q=16, K=300, Hq=16, Hkv=8, d_h=128, tau=1.0, lse=16, dq=16, ws_bytes=big, ldq=None):
        ldq = Hq * d_h if ldq is None else ldq
        return lib.tg_gated_attention_backward(vp(q), ldq, vp(4096), Hkv * d_h, vp(8192), Hkv * d_h, K, Hq, Hkv,
                                               d_h, None, None, tau, vp(16), vp(32), vp(lse) if lse else None,
                                               vp(dq) if dq else None, vp(48), vp(64), None, None, None, vp(256),
                                               ws_bytes, None)

    assert bwd(tau=0.0) == INV and bwd(tau=float("nan")) == INV
    assert bwd(Hq=12, Hkv=8) == INV
    assert bwd(d_h=96) == UNS
    assert bwd(Hq=16, Hkv=1) == UNS                 # 16 query heads per KV head
    assert bwd(lse=0) == INV                        # the forward's log-sum-exp is required
    assert bwd(dq=0) == INV
    assert bwd(q=24) == INV                         # misaligned
    assert bwd(ldq=16 * 128 + 4) == INV             # stride not a multiple of 8
    assert bwd(ws_bytes=big - 256) == INV


def test_project_rope_workspace_and_argument_errors(lib):
    vp = ctypes.c_void_p
    INV, UNS = tg.TG_ERR_INVALID_ARG, tg.TG_ERR_UNSUPPORTED
    ws = tg.tg_workspace_bytes(tg.TG_OP_PROJECT, 4608, 128)
    assert ws >= 256 and ws % 256 == 0                        # the status word
    assert tg.tg_workspace_bytes(tg.TG_OP_PROJECT, 4608, 96) == 0

    def proj(x=16, K=300, d=2048, ldx=2048, Hq=16, Hkv=8, d_h=128, base=1e6, ldo=4096, v16=None, ws_bytes=ws):
        return lib.tg_project_rope(vp(x), K, d, ldx, vp(4096), Hq, Hkv, d_h, vp(64), base, vp(8192), ldo,
                                   vp(v16) if v16 else None, vp(256), ws_bytes, None)

    assert proj(base=0.0) == INV
    assert proj(d=2000, ldx=2000) == UNS            # d not a multiple of 64
    assert proj(Hq=15, Hkv=8) == UNS                # (Hq + 2 Hkv) d_h not a multiple of 256
    assert proj(d_h=96) == UNS
    assert proj(x=24) == INV                        # misaligned
    assert proj(ldo=4092) == INV                    # output stride not a multiple of 8
    assert proj(ldo=2048) == INV                    # output stride shorter than a row
    assert proj(v16=40) == INV                      # misaligned fp16 copy
    assert proj(ws_bytes=128) == INV                 # shorter than the status word
    assert proj(K=0) == tg.TG_OK


def test_gathered_projection_and_kept_scores_argument_errors(lib):
    # host-side rejections, before any device work
    vp = ctypes.c_void_p
    INV = tg.TG_ERR_INVALID_ARG
    ws = tg.tg_workspace_bytes(tg.TG_OP_PROJECT, 300, 128)

    def projg(N=1000, rows=64, K=300, h=16):
        return lib.tg_project_rope_gather(vp(h), N, 256, 256, vp(rows) if rows else None, K, vp(4096), 4, 2, 128,
                                          vp(64), 1e6, vp(8192), 1024, None, vp(256), ws, None)

    assert projg(N=-1) == INV
    assert projg(rows=0) == INV                      # no index array
    assert projg(N=0) == INV                         # rows to gather from an empty h
    assert projg(K=0) == tg.TG_OK                    # nothing to do
    assert projg(h=24) == INV                        # misaligned h
    sel = lib.tg_topk_select_after_gate_kept_scores
    assert sel(vp(16), 1000, 0, 960, 256, vp(64), None, vp(256), 1 << 20, None) == INV  # no s_kept
    assert sel(None, 1000, 0, 960, 256, vp(64), vp(128), vp(256), 1 << 20, None) == INV  # no scores

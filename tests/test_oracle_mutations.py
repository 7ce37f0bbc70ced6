"""The oracle's pins must catch plausible mistakes.

Each case copies the oracle's C source, plants one mistake (a dropped term, a
wrong sign, index or operand), compiles the copy on the CPU and runs the
oracle pin tests against it in a subprocess: at least one pin must fail.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "tg_oracle.c")

MUTATIONS = {
    "gate_drop_eps": ("sqrt(ss / (double)d + eps)", "sqrt(ss / (double)d)"),
    "gate_sum_not_mean": ("sqrt(ss / (double)d + eps)", "sqrt(ss + eps)"),
    "gate_transposed_w1": ("acc += (double)hi[c] * W[(size_t)j * d + c];",
                           "acc += (double)hi[c] * W[(size_t)c * d_g + j];"),
    "gate_sigmoid_not_silu": ("double a = u / (1.0 + exp(-u));", "double a = 1.0 / (1.0 + exp(-u));"),
    "gate_drop_b1": ("double u = r * acc + (b1 ? (double)b1[j] : 0.0);", "double u = r * acc;"),
    "select_ties_high_index": ("return (a > b) - (a < b);", "return (a < b) - (a > b);"),
    "select_nan_on_top": ("return na ? 1 : -1;", "return na ? -1 : 1;"),
    "select_drop_question": ("if (i < doc_begin || i >= doc_end)\n            keep[i] = 1;", "(void)0;"),
    "attn_bias_sign": ("scale * dot + gain *", "scale * dot - gain *"),
    "attn_kv_head": ("int kvh = h / group;", "int kvh = h % Hkv;"),
    "attn_strict_causal": ("(pos[c] <= pos[r]) : (c <= r)", "(pos[c] < pos[r]) : (c < r)"),
    "attn_scale_no_sqrt": ("tau / sqrt((double)d_h)", "tau / (double)d_h"),
    "rope_sign": ("o[t] = x1 * c - x2 * s;", "o[t] = x1 * c + x2 * s;"),
    "rope_pairing": ("double x1 = xr[t], x2 = xr[t + half];", "double x1 = xr[2 * t], x2 = xr[2 * t + 1];"),
    "bwd_drop_softmax_mean": ("double dl = prob[c] * (dprob[c] - mean);", "double dl = prob[c] * dprob[c];"),
    "bwd_dk_wrong_operand": ("dkc[t] += dl * scale * (double)qr[t];", "dkc[t] += dl * scale * (double)kc[t];"),
    "bwd_dv_uses_dl": ("dvc[t] += prob[c] * (double)dor[t];", "dvc[t] += dl * (double)dor[t];"),
    "bwd_dtau_no_sqrt": ("dtau_sum += dl * dot[c] * inv_sqrt_d;", "dtau_sum += dl * dot[c];"),
    "bwd_ds_no_gain": ("ds[c] += dl * gain;", "ds[c] += dl;"),
    "bwd_kv_head": ("int kv_head = h / group;", "int kv_head = h % Hkv;"),
    "bwd_unnormalised_p": ("prob[c] /= denom;", "(void)denom;"),
    "rope_frequency_exponent": ("double inv_freq = pow(base, -2.0 * (double)t / (double)d_h);",
                                "double inv_freq = pow(base, -(double)t / (double)d_h);"),
    "project_transposed_w": ("acc += (double)xr[c] * (double)wj[c];",
                             "acc += (double)xr[c] * (double)W[(size_t)c * (size_t)n_out + j];"),
    "project_drop_last_term": ("for (int c = 0; c < d; ++c)\n                acc += (double)xr[c]",
                               "for (int c = 0; c < d - 1; ++c)\n                acc += (double)xr[c]"),
    "gather_pos_index": ("pos_out[r] = pos_in ? pos_in[i] : (int32_t)i;",
                         "pos_out[r] = pos_in ? pos_in[r] : (int32_t)i;"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_mutation(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor not found for {name}"
    mutated = tmp_path / "tg_oracle.c"
    mutated.write_text(src.replace(old, new))
    (tmp_path / "tg_oracle.h").write_text(open(os.path.join(ROOT, "oracle", "tg_oracle.h")).read())
    lib = tmp_path / "libmut.so"
    subprocess.run(["gcc", "-std=c11", "-O1", "-fPIC", "-shared", "-w", "-o", str(lib), str(mutated), "-lm"],
                   check=True)
    env = dict(os.environ, TG_ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        "tests/test_oracle_gate.py", "tests/test_oracle_select.py",
                        "tests/test_oracle_attention.py", "tests/test_oracle_attention_backward.py",
                        "tests/test_oracle_properties.py", "tests/test_oracle_project.py"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"no pin caught mutation {name}:\n{r.stdout[-2000:]}"

"""Host-side pieces of bench.py that need no GPU: the oracle baselines' sampling and extrapolation."""
import bench


def test_backward_oracle_sample_is_bounded_and_extrapolated():
    t, sample = bench.oracle_backward_sample(600, 4, 2, 64, budget_s=0.3)
    # the whole problem is small enough to be the sample: no extrapolation beyond the KV heads
    assert "first 600 of 600" in sample and t > 0
    t_big, sample_big = bench.oracle_backward_sample(20000, 4, 2, 64, budget_s=0.3)
    assert "of 20000 tokens" in sample_big
    ks = int(sample_big.split("over the first ")[1].split(" ")[0])
    assert 64 <= ks < 20000
    # extrapolated by the causal pair count: far above the sample's own time
    assert t_big > t


def test_decode_oracle_sample_extrapolates_by_keys():
    t1, s1 = bench.oracle_decode_sample([3000], 4, 2, 64, budget_s=0.05)
    t2, s2 = bench.oracle_decode_sample([3000, 3000, 1000], 4, 2, 64, budget_s=0.05)
    assert t1 > 0 and t2 > 0 and "of the 3 layer(s)" in s2
    ts = int(s1.split("over a ")[1].split("-key")[0])
    assert 256 <= ts <= 3000


def test_oracle_step_sample_runs_on_the_workload_data():
    from learned_token_pruning_tg_b200 import synth
    w = synth.scaled(synth.L16K, name="small", N=2048, doc_end=1920, k_doc=256, n_scaled=8)
    gi, ap = synth.gate_inputs(w), synth.attn_params(w)
    t, sample, parts = bench.oracle_sample(w, gi, ap, budget_s=0.3)
    assert t > 0 and set(parts) == {"gate_s", "select_s", "gather_s", "proj_s", "rope_s", "attn_s"}
    assert all(v >= 0 for v in parts.values()) and abs(sum(parts.values()) - t) < 1e-9
    assert f"/{w.N} rows" in sample and f"/{w.K} kept rows" in sample


def test_host_info_and_flush_rule():
    from learned_token_pruning_tg_b200 import synth
    info = bench.host_info()
    assert info["nproc"] >= 1
    # 16k (h = 67 MB) and 32k (134 MB) are below twice the L2, 128k (537 MB) is not
    assert bench.needs_flush(synth.L16K) and bench.needs_flush(synth.L32K_FULL)
    assert not bench.needs_flush(synth.L128K)
    assert set(bench.BENCH_WORKLOADS) >= {"qwen3-1.7b-16k", "qwen3-1.7b-32k-full", "qwen3-1.7b-128k",
                                          "qwen3-1.7b-32k-k512", "qwen3-1.7b-32k-k16384"}
    assert "tiny-1k" not in bench.BENCH_WORKLOADS

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

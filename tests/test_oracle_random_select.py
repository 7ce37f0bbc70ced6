"""Oracle pins for the random-K selector (the pages' budget-matched random baseline).

* The generator: SplitMix64 started from state 0 yields the published first
  outputs 0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F.
* The selection: brute force over the keys (largest first, lower index on
  ties) on small cases, the invariants (count, ascending, every token outside
  the span kept), budget edges, and determinism in the seed.
* Uniformity: over many seeds every document token is kept about k/n_doc of
  the time (a 6-sigma binomial bound per token) -- a wrong key (e.g. the low
  32 bits, or the doc-relative counter) would still pass the brute force but
  not the published vectors; a biased one fails here.
"""
import numpy as np
import pytest

import oracle

M64 = (1 << 64) - 1


def test_splitmix64_published_vectors():
    out = oracle.splitmix64_stream(0, 3)
    assert [int(x) for x in out] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def brute(N, db, de, k, seed):
    keys = oracle.splitmix64_stream(seed, N) >> np.uint64(32)
    doc = sorted(range(db, de), key=lambda i: (-int(keys[i]), i))[: min(k, de - db)]
    return np.array(sorted(set(doc) | set(range(0, db)) | set(range(de, N))), dtype=np.int32)


@pytest.mark.parametrize("N,db,de,k,seed", [(10, 2, 8, 3, 0), (100, 0, 90, 17, 1), (257, 5, 250, 0, 2),
                                            (257, 5, 250, 245, 3), (257, 5, 250, 500, 4), (1000, 0, 1000, 999, M64)])
def test_random_select_brute_force(N, db, de, k, seed):
    got = oracle.random_select(N, db, de, k, seed)
    assert np.array_equal(got, brute(N, db, de, k, seed))
    assert len(got) == oracle.kept_count(N, db, de, k)
    assert np.all(np.diff(got) > 0)
    assert np.all(np.isin(np.concatenate([np.arange(db), np.arange(de, N)]), got))


def test_random_select_seed_determinism():
    a = oracle.random_select(5000, 0, 4800, 300, 42)
    assert np.array_equal(a, oracle.random_select(5000, 0, 4800, 300, 42))
    assert not np.array_equal(a, oracle.random_select(5000, 0, 4800, 300, 43))


def test_random_select_uniform_over_seeds():
    N, db, de, k, trials = 400, 0, 384, 48, 400
    counts = np.zeros(N)
    for t in range(trials):
        counts[oracle.random_select(N, db, de, k, 1000 + t)] += 1
    p = k / (de - db)
    mu, sd = trials * p, np.sqrt(trials * p * (1 - p))
    assert np.all(np.abs(counts[db:de] - mu) <= 6 * sd)
    assert np.all(counts[de:] == trials)

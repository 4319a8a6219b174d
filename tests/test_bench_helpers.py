"""The benchmark's pair counter (the metric's numerator) against the oracle's
brute-force count over rows, and its per-row variant."""
import numpy as np
import pytest

import bench
import oracle


@pytest.mark.parametrize("seed", range(6))
def test_pair_formula_matches_brute_force(seed):
    rng = np.random.default_rng(seed)
    N = int(rng.integers(1, 700))
    v = np.nonzero(rng.random(N) < rng.uniform(0, 0.5))[0].astype(np.int32)
    s = np.nonzero(rng.random(N) < rng.uniform(0, 0.5))[0].astype(np.int32)
    assert bench.pairs_per_set(N, v, s) == oracle.count_pairs(N, v, s)
    rows = np.arange(N)
    assert int(bench.row_pairs(rows, v, s).sum()) == oracle.count_pairs(N, v, s)


def test_dense_and_empty():
    N = 300
    assert bench.pairs_per_set(N, np.arange(N), []) == N * (N + 1) // 2
    assert bench.pairs_per_set(N, [], []) == 0
    assert bench.pairs_per_set(N, [], [0]) == N

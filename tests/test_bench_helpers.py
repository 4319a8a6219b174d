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


def test_block_pairs_brute_force():
    # causal pairs inside kept blocks, against an explicit count
    rng = np.random.default_rng(3)
    for N in (1, 128, 300, 1000):
        T = (N + 127) // 128
        keep = np.tril(rng.random((2, T, T)) < 0.4)
        keep[:, np.arange(T), np.arange(T)] = rng.random((2, T)) < 0.8
        W = (T + 31) // 32
        mask = np.zeros((2, T, W), np.uint32)
        for h in range(2):
            for I in range(T):
                for J in range(T):
                    if keep[h, I, J]:
                        mask[h, I, J >> 5] |= np.uint32(1 << (J & 31))
        want = 0
        for h in range(2):
            for i in range(N):
                for j in range(i + 1):
                    want += int(keep[h, i // 128, j // 128])
        assert bench.block_pairs(mask, N) == want


def test_block_kernel_rooflines():
    import types
    props = types.SimpleNamespace(multi_processor_count=148)
    k = bench.block_kernel_rooflines(131072, 32, 128, 4.0, 8.0, 1e15, 6.0,
                                     {"sm_mhz": 1965.0}, props)
    T = 1024
    fma = 16 * 128 * 32 * T * (T - 1) / 2
    peak = 148 * 64 * 2 * 1965e6 / 1e12
    assert abs(k["discovery"]["achieved_tflops"] - round(2 * fma / 4e-3 / 1e12, 2)) < 1e-9
    assert abs(k["discovery"]["peak_tflops"] - round(peak, 2)) < 1e-9
    assert k["attention"]["frac"] == 0.75
    # no clock samples: the nominal maximum clock
    k2 = bench.block_kernel_rooflines(131072, 32, 128, 4.0, 8.0, 1e15, 6.0, {"sm_mhz": None}, props)
    assert k2["discovery"]["peak_tflops"] == k["discovery"]["peak_tflops"]


def test_cpu_baseline_reports_sparse_and_dense_rows():
    import oracle
    from vs_workloads import WORKLOADS
    w = WORKLOADS["tiny_1k"]
    Qb, Kb, Vb = w.qkv()
    lv, ls = w.all_scores()
    sets = []
    for scores, k, tau in ((lv, w.k_v, w.tau_v), (ls, w.k_s, w.tau_s)):
        idx = np.empty((w.H_sel, k), np.int32)
        cnt = np.empty(w.H_sel, np.int32)
        for h in range(w.H_sel):
            idx[h], cnt[h], _ = oracle.select(scores[h], w.select_mode_id, k, tau)
        sets += [idx, cnt]
    cb = bench.cpu_baseline(w, Qb, Kb, Vb, *sets, seconds=0.05)
    assert cb["kind"] == "oracle" and cb["value"] > 0
    assert cb["sparse_row_ms"] > 0 and cb["dense_row_ms"] > 0


def test_indexer_roofline_terms():
    import types
    w = types.SimpleNamespace(indexer=True, hidden=256)
    peaks = {"bf16_tflops": 1500.0, "hbm_gbs": 6000.0}
    N, Hkv, d = 262144, 8, 128
    k = bench.kernel_rooflines(w, peaks, N, 32, Hkv, d, 8, 1e15, 1e9, 10.0, 1.0, 2.0, 0, 0)
    flops = 2.0 * N * Hkv * (2 * d * 256 + 2 * 256)
    nbytes = N * Hkv * (4 * d + 8) + 4 * 256 * (2 * d + 2)
    t = max(flops / 1.5e15, nbytes / 6e12)
    assert k["indexer"]["bound"] == ("tensor" if flops / 1.5e15 >= nbytes / 6e12 else "hbm")
    assert abs(k["indexer"]["frac"] - round(t / 2e-3, 4)) < 1e-12
    assert abs(k["indexer"]["achieved_gbs"] - round(nbytes / 2e-3 / 1e9, 1)) < 1e-9


def test_e2e_unit_order():
    # two heavy and two light KV groups of 2 heads; copies cost about as much as a
    # light group's compute.  The chosen order covers every head once, splits the
    # first and last group into heads, and is no longer (in the model) than
    # heaviest-first, which leaves the light groups' copies out for the end.
    Hkv, G = 4, 2
    head_cost = [8.0, 8.0, 0.2, 0.2, 8.0, 8.0, 0.2, 0.2]
    units = bench.e2e_units(Hkv, G, head_cost, 1.0, 2.0, 1.0)
    heads = sorted(h for _, h0, h1 in units for h in range(h0, h1))
    assert heads == list(range(Hkv * G))
    assert units[0][2] - units[0][1] == 1 and units[-1][2] - units[-1][1] == 1
    first, last = units[0][0], units[-1][0]
    assert head_cost[first * G] == 8.0 and head_cost[last * G] == 8.0

    def model(us):
        t_in = t_c = t_out = 0.0
        seen = set()
        for g, h0, h1 in us:
            t_in += (h1 - h0) + (0.0 if g in seen else 2.0)
            seen.add(g)
            t_c = max(t_c, t_in) + sum(head_cost[h0:h1]) + 0.05
            t_out = max(t_out, t_c) + (h1 - h0)
        return t_out

    hf_units = [(0, 0, 1), (0, 1, 2), (2, 4, 6), (1, 2, 4), (3, 6, 7), (3, 7, 8)]
    assert model(units) <= model(hf_units)
    assert model(units) < model(hf_units) - 0.5

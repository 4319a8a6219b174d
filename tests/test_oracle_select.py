"""Pins for the oracle's selection (CPU only).

Selection follows the VSPrefill pages' budgets: a fixed top-k, or the
cumulative-threshold rule over the predicted scores (Technical Summary,
section 2 Adaptive Inference Pipeline, Dynamic Budgeting).  Each test pins
the oracle to something other than itself: a hand-worked example, a closed
form, a library sort, or an exact (fsum) brute force.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def test_worked_example_fixture():
    g = json.load(open(os.path.join(GOLD, "select_worked_example.json")))
    s = np.log(np.array(g["A"], np.float64)).astype(np.float32)
    for c in g["cases"]:
        if c["mode"] == "threshold":
            idx, cnt, _ = oracle.select(s, oracle.THRESHOLD, c["cap"], c["tau"])
        elif c["mode"] == "maxfrac":
            idx, cnt, _ = oracle.select(s, oracle.MAXFRAC, c["cap"], c["alpha"])
        else:
            idx, cnt, _ = oracle.select(s, oracle.TOPK, c["k"])
        assert cnt == c["count"], c
        assert list(idx[:cnt]) == c["idx"], c
        assert all(x == -1 for x in idx[cnt:])


def test_all_equal_threshold_closed_form():
    # all p_r = 1, Z = N: smallest k with k >= tau*N is ceil(tau*N); ties -> smallest indices
    for N, tau in ((1024, 0.9), (1000, 0.5), (7, 0.3), (4096, 0.95)):
        idx, cnt, _ = oracle.select(np.full(N, 1.25, np.float32), oracle.THRESHOLD, N, tau)
        k = math.ceil(tau * N - 1e-12)
        assert cnt == k
        assert np.array_equal(idx[:k], np.arange(k))
    idx, cnt, _ = oracle.select(np.zeros(1024, np.float32), oracle.THRESHOLD, 1024, 0.9)
    assert cnt == 922


def test_topk_full_and_one_hot():
    rng = np.random.default_rng(0)
    s = rng.standard_normal(500).astype(np.float32)
    idx, cnt, _ = oracle.select(s, oracle.TOPK, 500)
    assert cnt == 500 and np.array_equal(idx, np.arange(500))
    s = np.zeros(300, np.float32)
    s[123] = 100.0
    idx, cnt, _ = oracle.select(s, oracle.THRESHOLD, 300, 0.99)
    assert cnt == 1 and idx[0] == 123


def test_tie_block_takes_smaller_indices():
    s = np.array([5, 3, 1, 3, 3, 0, 3], np.float32)
    idx, cnt, _ = oracle.select(s, oracle.TOPK, 3)
    assert list(idx) == [0, 1, 3]
    # threshold whose crossing lands inside the tie block
    idx, cnt, _ = oracle.select(np.array([0, 0, 0, 0], np.float32), oracle.THRESHOLD, 4, 0.6)
    assert cnt == 3 and list(idx[:3]) == [0, 1, 2]


@pytest.mark.parametrize("seed", range(8))
def test_topk_matches_library_sort(seed):
    rng = np.random.default_rng(seed)
    N = int(rng.integers(1, 3000))
    s = rng.standard_normal(N).astype(np.float32)
    s[rng.integers(0, N, N // 5)] = s[0]  # inject ties
    k = int(rng.integers(1, N + 1))
    order = np.lexsort((np.arange(N), -s.astype(np.float64)))
    want = np.sort(order[:k])
    idx, cnt, _ = oracle.select(s, oracle.TOPK, k)
    assert cnt == k and np.array_equal(idx, want)


@pytest.mark.parametrize("seed", range(8))
def test_threshold_matches_exact_sum_brute_force(seed):
    rng = np.random.default_rng(100 + seed)
    N = int(rng.integers(2, 4000))
    s = (rng.standard_normal(N) * rng.uniform(0.1, 4)).astype(np.float32)
    tau = float(rng.uniform(0.05, 0.999))
    order = sorted(range(N), key=lambda r: (-float(s[r]), r))
    smax = float(s[order[0]])
    p = [math.exp(float(s[r]) - smax) for r in order]
    Z = math.fsum(p)
    k = None
    for r in range(N):
        if math.fsum(p[: r + 1]) >= tau * Z:
            k = r + 1
            break
    idx, cnt, margin = oracle.select(s, oracle.THRESHOLD, N, tau)
    if margin > 1e-9:
        assert cnt == k
        assert np.array_equal(idx[:cnt], np.sort(order[:k]))


def test_threshold_cap_binds():
    rng = np.random.default_rng(5)
    s = (0.01 * rng.standard_normal(2048)).astype(np.float32)  # near uniform: needs ~95% of N
    idx, cnt, _ = oracle.select(s, oracle.THRESHOLD, 64, 0.95)
    assert cnt == 64
    order = np.lexsort((np.arange(2048), -s.astype(np.float64)))
    assert np.array_equal(idx, np.sort(order[:64]))


def test_special_values():
    s = np.array([0.0, -np.inf, np.nan, -1.0], np.float32)
    # tau = 1 keeps exactly the entries with p > 0: 0.0 and -1.0
    idx, cnt, _ = oracle.select(s, oracle.THRESHOLD, 4, 1.0)
    assert cnt == 2 and list(idx[:2]) == [0, 3]
    # order: 0.0 (0), -1.0 (3), -inf (1), NaN (2)
    idx, cnt, _ = oracle.select(s, oracle.TOPK, 3)
    assert list(idx) == [0, 1, 3]
    idx, cnt, _ = oracle.select(s, oracle.TOPK, 4)
    assert list(idx) == [0, 1, 2, 3]
    # all NaN: Z = 0 -> k = 1, the smallest index
    idx, cnt, _ = oracle.select(np.full(5, np.nan, np.float32), oracle.THRESHOLD, 5, 0.5)
    assert cnt == 1 and idx[0] == 0
    # +0.0 and -0.0 tie and fall back to index order
    idx, cnt, _ = oracle.select(np.array([-0.0, 0.0, -1.0], np.float32), oracle.TOPK, 1)
    assert idx[0] == 0


def test_invalid_arguments():
    s = np.zeros(10, np.float32)
    for k in (0, 11):
        with pytest.raises(ValueError):
            oracle.select(s, oracle.TOPK, k)
    for tau in (0.0, 1.5, -1.0, float("nan")):
        with pytest.raises(ValueError):
            oracle.select(s, oracle.THRESHOLD, 5, tau)
        with pytest.raises(ValueError):
            oracle.select(s, oracle.MAXFRAC, 5, tau)
    with pytest.raises(ValueError):
        oracle.select(s, 3, 5, 0.5)


def test_margin_detects_boundary():
    # tau*Z lands exactly on a prefix sum -> margin ~ 0
    s = np.zeros(10, np.float32)
    _, cnt, margin = oracle.select(s, oracle.THRESHOLD, 10, 0.5)
    assert cnt == 5 and margin < 1e-12


def test_margin_ignores_decisions_hidden_by_the_cap():
    s = np.zeros(10, np.float32)
    _, cnt, margin = oracle.select(s, oracle.THRESHOLD, 3, 0.5)  # uncapped k = 5 on a boundary
    assert cnt == 3 and margin == np.inf
    _, cnt, margin = oracle.select(s, oracle.THRESHOLD, 5, 0.5)  # cap == k: boundary matters
    assert cnt == 5 and margin < 1e-12


# ------------------------------------------------------------- max-based rule


@pytest.mark.parametrize("seed", range(8))
def test_maxfrac_matches_probability_brute_force(seed):
    # the rule as the page states it, on softmax probabilities: keep r iff
    # prob_r >= alpha * max(prob); probabilities from an fsum normaliser
    rng = np.random.default_rng(300 + seed)
    N = int(rng.integers(2, 5000))
    s = (rng.standard_normal(N) * rng.uniform(0.2, 3)).astype(np.float32)
    alpha = float(np.exp(-rng.uniform(0.01, 6)))
    z = math.fsum(math.exp(float(x) - float(s.max())) for x in s)
    prob = [math.exp(float(x) - float(s.max())) / z for x in s]
    pmax = max(prob)
    rel = [p / (alpha * pmax) for p in prob]
    if min(abs(r - 1.0) for r in rel) < 1e-9:
        pytest.skip("an entry sits on the boundary")
    want = [r for r in range(N) if prob[r] >= alpha * pmax]
    idx, cnt, margin = oracle.select(s, oracle.MAXFRAC, N, alpha)
    assert margin == np.inf
    assert cnt == len(want)
    assert list(idx[:cnt]) == want and all(x == -1 for x in idx[cnt:])


def test_maxfrac_closed_form_linear_decay():
    # logits -r/4 (exact in fp32): exp(-r/4) >= alpha  <=>  r <= -4 ln(alpha)
    N = 400
    s = (-np.arange(N) / 4.0).astype(np.float32)
    for lna in (-0.1, -2.6, -10.3, -50.05):
        idx, cnt, _ = oracle.select(s, oracle.MAXFRAC, N, math.exp(lna))
        k = math.floor(-4.0 * lna) + 1
        assert cnt == k and np.array_equal(idx[:k], np.arange(k))
    # alpha = 1 keeps the maximum and its ties only
    idx, cnt, _ = oracle.select(np.array([1, 3, 3, 2], np.float32), oracle.MAXFRAC, 4, 1.0)
    assert cnt == 2 and list(idx[:2]) == [1, 2]


def test_maxfrac_is_a_prefix_of_the_order_and_shift_invariant():
    rng = np.random.default_rng(9)
    s = rng.integers(-40, 40, 3000).astype(np.float32)  # integers: shifts stay exact
    for alpha in (0.9, 0.05, 1e-6):
        idx, cnt, _ = oracle.select(s, oracle.MAXFRAC, 3000, alpha)
        tidx, tcnt, _ = oracle.select(s, oracle.TOPK, cnt)
        assert np.array_equal(idx[:cnt], tidx)
        sidx, scnt, _ = oracle.select(s + np.float32(1000), oracle.MAXFRAC, 3000, alpha)
        assert scnt == cnt and np.array_equal(sidx, idx)


def test_maxfrac_cap_and_special_values():
    rng = np.random.default_rng(11)
    s = (0.01 * rng.standard_normal(2048)).astype(np.float32)  # all within 0.1 of the max
    idx, cnt, _ = oracle.select(s, oracle.MAXFRAC, 100, 0.5)
    order = np.lexsort((np.arange(2048), -s.astype(np.float64)))
    assert cnt == 100 and np.array_equal(idx, np.sort(order[:100]))
    # NaN and -inf are never kept next to a finite maximum
    s = np.array([np.nan, -np.inf, 0.0, -1.0, np.nan], np.float32)
    idx, cnt, _ = oracle.select(s, oracle.MAXFRAC, 5, 1e-30)
    assert cnt == 2 and list(idx[:2]) == [2, 3]
    # all NaN: one entry, the smallest index
    idx, cnt, _ = oracle.select(np.full(4, np.nan, np.float32), oracle.MAXFRAC, 4, 0.5)
    assert cnt == 1 and idx[0] == 0
    # an infinite maximum keeps only its ties; an all -inf row keeps every -inf
    s = np.array([np.inf, 5.0, np.inf, np.nan], np.float32)
    idx, cnt, _ = oracle.select(s, oracle.MAXFRAC, 4, 1e-30)
    assert cnt == 2 and list(idx[:2]) == [0, 2]
    s = np.array([-np.inf, np.nan, -np.inf], np.float32)
    idx, cnt, _ = oracle.select(s, oracle.MAXFRAC, 3, 0.5)
    assert cnt == 2 and list(idx[:2]) == [0, 2]


def test_maxfrac_boundary_is_kept():
    # the page discards scores *below* alpha * max, so a score exactly on the
    # threshold stays: pick differences d with log(exp(d)) == d in fp64
    hits = 0
    for q in range(1, 200):
        d = -q / 8.0
        alpha = math.exp(d)
        if math.log(alpha) != d:
            continue
        hits += 1
        s = np.array([0.0, d, d - 0.125], np.float32)
        idx, cnt, _ = oracle.select(s, oracle.MAXFRAC, 3, alpha)
        assert cnt == 2 and list(idx[:2]) == [0, 1]
    assert hits > 20

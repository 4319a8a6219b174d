"""Pins for the oracle's ground-truth aggregation (CPU only).

The distillation target of the VSPrefill pages (Technical Summary, section 2,
"Distillation Training"): full attention weights summed along vertical
columns (A_v) and slash diagonals (A_s).  Each test pins the oracle to
something other than itself: the row-sum invariant, a closed form, an
explicit-matrix brute force in numpy, and a limit case."""
import math

import numpy as np
import pytest

import oracle


def _bf16_bits(x):
    u = np.ascontiguousarray(x, np.float32).view(np.uint32)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def test_row_sums_give_n():
    rng = np.random.default_rng(0)
    N = 300
    Q = _bf16_bits(2 * rng.standard_normal((N, 4, 32)))
    K = _bf16_bits(2 * rng.standard_normal((N, 2, 32)))
    Av, As = oracle.aggregate(Q, K)
    assert np.allclose(Av.sum(1), N, rtol=0, atol=1e-9)
    assert np.allclose(As.sum(1), N, rtol=0, atol=1e-9)
    assert (Av >= 0).all() and (As >= 0).all()


def test_uniform_attention_harmonic_closed_form():
    # q = 0 makes every causal weight p_ij = 1/(i+1), so
    # A_v[j] = sum_{i>=j} 1/(i+1) = H_N - H_j and A_s[o] = H_N - H_o
    N = 257
    Q = np.zeros((N, 1, 16), np.float32)
    K = np.random.default_rng(1).standard_normal((N, 1, 16)).astype(np.float32)
    Av, As = oracle.aggregate(Q, K)
    H = np.concatenate([[0.0], np.cumsum(1.0 / np.arange(1, N + 1))])
    want = H[N] - H[np.arange(N)]
    assert np.allclose(Av[0], want, rtol=1e-12, atol=1e-12)
    assert np.allclose(As[0], want, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("seed", range(4))
def test_matches_explicit_matrix(seed):
    # numpy: full score matrix, causal mask, row softmax, then column sums and
    # the sums along each sub-diagonal (np.diagonal with offset -o)
    rng = np.random.default_rng(10 + seed)
    N, Hq, Hkv, d = int(rng.integers(1, 90)), 4, 2, 16
    Q = rng.standard_normal((N, Hq, d)).astype(np.float32)
    K = rng.standard_normal((N, Hkv, d)).astype(np.float32)
    scale = float(rng.uniform(0.05, 0.6))
    Av, As = oracle.aggregate(Q, K, scale=scale)
    for h in range(Hq):
        S = scale * (Q[:, h, :].astype(np.float64) @ K[:, h // 2, :].astype(np.float64).T)
        S[np.triu_indices(N, 1)] = -np.inf
        P = np.exp(S - S.max(1, keepdims=True))
        P /= P.sum(1, keepdims=True)
        assert np.allclose(Av[h], P.sum(0), rtol=1e-12, atol=1e-13)
        diag = np.array([np.diagonal(P, offset=-o).sum() for o in range(N)])
        assert np.allclose(As[h], diag, rtol=1e-12, atol=1e-13)


def test_dominant_first_key_limit():
    # k_0 aligned with every query at a huge score: p_i0 -> 1, so A_v -> N e_0
    # and every offset o collects p_{o,0} -> 1
    N, d = 64, 8
    Q = np.zeros((N, 1, d), np.float32)
    Q[:, 0, 0] = 1.0
    K = np.zeros((N, 1, d), np.float32)
    K[0, 0, 0] = 400.0
    Av, As = oracle.aggregate(Q, K, scale=1.0)
    assert abs(Av[0, 0] - N) < 1e-9 and np.abs(Av[0, 1:]).max() < 1e-9
    assert np.allclose(As[0], 1.0, atol=1e-9)


def test_row_range_gives_exact_tail_and_head_subset():
    rng = np.random.default_rng(3)
    N = 200
    Q = _bf16_bits(rng.standard_normal((N, 4, 16)))
    K = _bf16_bits(rng.standard_normal((N, 1, 16)))
    Av, As = oracle.aggregate(Q, K)
    lo = 150
    tv, ts = oracle.aggregate(Q, K, heads=[2, 0], rows=(lo, N))
    assert np.array_equal(tv[0, lo:], Av[2, lo:]) and np.array_equal(ts[1, lo:], As[0, lo:])
    assert (tv[:, :lo] >= 0).all() and tv[:, :lo].sum() < Av[[2, 0], :lo].sum()

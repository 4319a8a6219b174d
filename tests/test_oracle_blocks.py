"""Pins for the oracle's FlashPrefill-style block pattern and block-sparse
attention (CPU only).

FlashPrefill summary page, section 2A (skeleton queries probe key blocks
through their mean keys) and 2B (keep blocks scoring at least alpha times the
best).  Each test pins the oracle to something other than itself: a numpy
restatement, a closed form, limits in alpha, and the dense oracle."""
import math

import numpy as np
import pytest

import oracle


def _np_block_select(Q, K, alpha, scale):
    # independent numpy statement of the definition
    N, Hq, d = Q.shape
    Hkv = K.shape[1]
    T = (N + 127) // 128
    out = np.zeros((Hq, T, T), bool)
    for h in range(Hq):
        k = K[:, h // (Hq // Hkv), :].astype(np.float64)
        kbar = np.stack([k[128 * J:min(N, 128 * J + 128)].mean(0) for J in range(T)])
        for I in range(T):
            out[h, I, I] = True
            if I == 0:
                continue
            probes = [128 * I + 8 * m for m in range(16) if 128 * I + 8 * m < N]
            q = Q[probes, h, :].astype(np.float64)
            s = scale * q @ kbar[:I].T                       # [probes, I]
            p = np.exp(s - s.max(1, keepdims=True))
            p /= p.sum(1, keepdims=True)
            score = p.mean(0)
            out[h, I, :I] = score >= alpha * score.max()
    return out


def _unpack(mask, T):
    bits = np.unpackbits(mask.view(np.uint8), bitorder="little").reshape(mask.shape[0], T, -1)
    return bits[:, :, :T].astype(bool)


@pytest.mark.parametrize("seed", range(3))
def test_matches_numpy_restatement(seed):
    rng = np.random.default_rng(seed)
    N, Hq, Hkv, d = int(rng.integers(129, 1500)), 4, 2, 16
    Q = rng.standard_normal((N, Hq, d)).astype(np.float32)
    K = (rng.standard_normal((N, Hkv, d)) + rng.standard_normal((1, Hkv, d))).astype(np.float32)
    # structure: some key blocks pulled toward the queries' shared direction
    u = rng.standard_normal(d).astype(np.float32)
    Q += 0.8 * u
    for J in rng.choice((N + 127) // 128, 3):
        K[128 * J:128 * J + 128] += 0.6 * u
    alpha = float(rng.uniform(0.05, 0.7))
    scale = 0.4
    mask, margin = oracle.block_select(Q, K, alpha, scale=scale)
    want = _np_block_select(Q, K, alpha, scale)
    got = _unpack(mask, (N + 127) // 128)
    assert (margin > 1e-9).all()
    assert np.array_equal(got, want)


def test_closed_form_constant_blocks():
    # keys constant per block and one query for all rows: every probe gives
    # softmax_J(log a_J) = a_J / sum, so block J < I is kept iff
    # a_J >= alpha * max_{J' < I} a_J'
    T, d = 9, 8
    N = 128 * T
    a = np.array([5.0, 0.3, 1.0, 4.0, 0.05, 2.5, 0.9, 3.0, 1.0])
    q = np.zeros(d)
    q[0] = 1.0
    Q = np.tile(q, (N, 1, 1)).astype(np.float32)
    K = np.zeros((N, 1, d), np.float32)
    for J in range(T):
        K[128 * J:128 * J + 128, 0, 0] = np.log(a[J])
    for alpha in (0.25, 0.55, 0.9):  # no ratio a_J / max lies on a threshold
        mask, margin = oracle.block_select(Q, K, alpha, scale=1.0)
        assert margin[0] > 1e-6
        got = _unpack(mask, T)[0]
        for I in range(T):
            want = np.zeros(T, bool)
            want[I] = True
            if I:
                want[:I] = a[:I] >= alpha * a[:I].max() - 1e-12
            assert np.array_equal(got[I], want), (alpha, I)


def test_closed_form_probe_rows_and_ragged_probe_count():
    # Which rows probe: only rows 128 I + 8 m (m = 0..15, below N) carry the
    # probe queries -- q1 = e1 for even m, q2 = e2 for odd m -- every other
    # row carries -e1, which would invert the preferences if it were read.
    # Keys are constant per block, k_J = ln(a_J) e1 + ln(b_J) e2, so with
    # scale 1 a q1 probe gives softmax weights a_J / sum a and a q2 probe
    # b_J / sum b over J < I.  A full block has 8 probes of each kind: score
    # (P1 + P2) / 2; the last block here holds 20 rows, i.e. probes m = 0,
    # 1, 2 (two q1, one q2): score (2 P1 + P2) / 3.
    T, d = 6, 4
    N = 128 * (T - 1) + 20
    a = np.array([3.0, 0.4, 1.2, 2.0, 0.7, 1.0])
    b = np.array([0.2, 2.5, 1.0, 0.5, 3.0, 1.0])
    K = np.zeros((N, 1, d), np.float32)
    for J in range(T):
        rows = slice(128 * J, min(N, 128 * J + 128))
        K[rows, 0, 1] = np.log(a[J])
        K[rows, 0, 2] = np.log(b[J])
    Q = np.zeros((N, 1, d), np.float32)
    Q[:, 0, 1] = -1.0
    for I in range(T):
        for m in range(16):
            i = 128 * I + 8 * m
            if i < N:
                Q[i, 0, 1], Q[i, 0, 2] = (1.0, 0.0) if m % 2 == 0 else (0.0, 1.0)
    for alpha in (0.3, 0.6, 0.85):
        mask, margin = oracle.block_select(Q, K, alpha, scale=1.0)
        assert margin[0] > 1e-6, alpha
        got = _unpack(mask, T)[0]
        for I in range(T):
            want = np.zeros(T, bool)
            want[I] = True
            if I:
                p1 = a[:I] / a[:I].sum()
                p2 = b[:I] / b[:I].sum()
                score = (2 * p1 + p2) / 3 if I == T - 1 else (p1 + p2) / 2
                want[:I] = score >= alpha * score.max()
            assert np.array_equal(got[I], want), (alpha, I)


def test_alpha_limits_and_monotonicity():
    rng = np.random.default_rng(4)
    N = 1000
    Q = rng.standard_normal((N, 2, 16)).astype(np.float32)
    K = rng.standard_normal((N, 1, 16)).astype(np.float32)
    T = (N + 127) // 128
    every, _ = oracle.block_select(Q, K, 1e-300)
    assert np.array_equal(_unpack(every, T), np.tril(np.ones((T, T), bool))[None].repeat(2, 0))
    prev = _unpack(every, T)
    for alpha in (0.1, 0.3, 0.6, 0.95):
        cur = _unpack(oracle.block_select(Q, K, alpha)[0], T)
        assert (cur <= prev).all()  # a larger alpha keeps a subset
        prev = cur
    top, _ = oracle.block_select(Q, K, 1.0)
    t = _unpack(top, T)
    assert all(t[h, I, :I].sum() == (1 if I else 0) for h in range(2) for I in range(T))


def _full_mask(Hq, T, keep):
    W = (T + 31) // 32
    m = np.zeros((Hq, T, W), np.uint32)
    for h in range(Hq):
        for I in range(T):
            for J in range(T):
                if keep(h, I, J):
                    m[h, I, J >> 5] |= np.uint32(1 << (J & 31))
    return m


def test_block_attention_all_kept_is_dense():
    rng = np.random.default_rng(5)
    N, Hq, d = 700, 2, 32
    Q = rng.standard_normal((N, Hq, d)).astype(np.float32)
    K = rng.standard_normal((N, 1, d)).astype(np.float32)
    V = rng.standard_normal((N, 1, d)).astype(np.float32)
    T = (N + 127) // 128
    mask = _full_mask(Hq, T, lambda h, I, J: J <= I)
    rows = np.array([0, 1, 127, 128, 300, 699])
    for h in range(Hq):
        O, l = oracle.attn_block_rows(Q, K, V, h, rows, mask)
        Od, ld = oracle.attn_rows(Q, K, V, h, rows, dense=True)
        assert np.allclose(O, Od, atol=1e-12) and np.allclose(l, ld, atol=1e-12)


def test_block_attention_matches_numpy_mask():
    rng = np.random.default_rng(6)
    N, Hq, d = 520, 2, 16
    Q = rng.standard_normal((N, Hq, d)).astype(np.float32)
    K = rng.standard_normal((N, 1, d)).astype(np.float32)
    V = rng.standard_normal((N, 1, d)).astype(np.float32)
    T = (N + 127) // 128
    keep = rng.random((Hq, T, T)) < 0.5
    mask = _full_mask(Hq, T, lambda h, I, J: J <= I and (J == I or keep[h, I, J]))
    rows = np.arange(N)
    for h in range(Hq):
        O, l = oracle.attn_block_rows(Q, K, V, h, rows, mask)
        S = (Q[:, h].astype(np.float64) @ K[:, 0].astype(np.float64).T) / math.sqrt(d)
        allowed = np.zeros((N, N), bool)
        for i in range(N):
            for J in range(i // 128 + 1):
                if J == i // 128 or keep[h, i // 128, J]:
                    allowed[i, 128 * J:min(i + 1, 128 * J + 128)] = True
        S[~allowed] = -np.inf
        P = np.exp(S - S.max(1, keepdims=True))
        want = (P / P.sum(1, keepdims=True)) @ V[:, 0].astype(np.float64)
        assert np.allclose(O, want, atol=1e-10)
        assert np.allclose(l, S.max(1) + np.log(np.exp(S - S.max(1, keepdims=True)).sum(1)), atol=1e-10)

"""Pins for the oracle's vertical-slash attention (CPU only).

The key set of query i is the union of the selected columns j <= i and the
keys i - o at the selected offsets o <= i (VSPrefill summary pages,
Technical Summary section 2: vertical lines are key columns, slash lines are
diagonals at relative offset i - j; the fused kernel merges both index lists
so each key is used once).  Pins: a hand-worked example, reduction to
PyTorch's causal SDPA when every column is selected, the closed forms for
S={0} and V={0},S={0}, and brute force over masks at tiny N.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from vs_workloads import gen_qkv

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _sets(v, s, ld=None):
    v = sorted(set(v))
    s = sorted(set(s))
    ld = ld or max(1, len(v), len(s))
    vi = np.full((1, ld), -1, np.int32)
    si = np.full((1, ld), -1, np.int32)
    vi[0, : len(v)] = v
    si[0, : len(s)] = s
    return vi, np.array([len(v)], np.int32), si, np.array([len(s)], np.int32)


def _f32(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_worked_example_fixture():
    g = json.load(open(os.path.join(GOLD, "attn_worked_example.json")))
    N, d = g["N"], g["d"]
    Q = np.array(g["q"], np.float32).reshape(N, 1, d)
    K = np.array(g["k"], np.float32).reshape(N, 1, d)
    V = np.array(g["v"], np.float32).reshape(N, 1, d)
    vi, vc, si, sc = _sets(g["verticals"], g["slashes"])
    for form in ("rows", "mask"):
        if form == "rows":
            O, lse = oracle.attn_rows(Q, K, V, 0, np.arange(N), vi, vc, si, sc, scale=g["scale"])
        else:
            O, lse = oracle.attn_mask(Q, K, V, 0, vi, vc, si, sc, scale=g["scale"])
        np.testing.assert_allclose(O, np.array(g["O"]), rtol=1e-13, atol=1e-13)
        np.testing.assert_allclose(lse, np.array(g["LSE"]), rtol=1e-13, atol=1e-13)
    _, _, M = oracle.attn_mask(Q, K, V, 0, vi, vc, si, sc, scale=g["scale"], return_mask=True)
    for i, ks in enumerate(g["key_sets"]):
        assert list(np.nonzero(M[i])[0]) == ks


@pytest.mark.parametrize("Hq,Hkv,d,N", [(1, 1, 64, 200), (4, 2, 32, 150), (4, 1, 16, 97)])
def test_all_columns_equals_causal_sdpa(Hq, Hkv, d, N):
    Q, K, V = gen_qkv(7, N, Hq, Hkv, d, 10000.0)
    H_sel = Hq
    vi = np.tile(np.arange(N, dtype=np.int32), (H_sel, 1))
    vc = np.full(H_sel, N, np.int32)
    si = np.zeros((H_sel, 1), np.int32)
    sc = np.zeros(H_sel, np.int32)
    q = torch.from_numpy(_f32(Q)).permute(1, 0, 2)
    k = torch.from_numpy(_f32(K)).permute(1, 0, 2).repeat_interleave(Hq // Hkv, 0)
    v = torch.from_numpy(_f32(V)).permute(1, 0, 2).repeat_interleave(Hq // Hkv, 0)
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, is_causal=True).numpy()
    for h in range(Hq):
        O, lse = oracle.attn_rows(Q, K, V, h, np.arange(N), vi, vc, si, sc)
        np.testing.assert_allclose(O, ref[h], rtol=1e-10, atol=1e-12)
        Od, lsed = oracle.attn_rows(Q, K, V, h, np.arange(N), dense=True)
        np.testing.assert_allclose(Od, ref[h], rtol=1e-10, atol=1e-12)
        np.testing.assert_array_equal(lse, lsed)
        # LSE against a direct log-sum-exp of the causal score row (library logsumexp)
        s = (q[h] @ k[h].T) / math.sqrt(d)
        s = s.masked_fill(torch.triu(torch.ones(N, N, dtype=torch.bool), 1), -math.inf)
        np.testing.assert_allclose(lse, torch.logsumexp(s, -1).numpy(), rtol=1e-12, atol=1e-12)


def test_slash_zero_returns_v():
    N, d = 300, 64
    Q, K, V = gen_qkv(3, N, 2, 1, d, 10000.0)
    vi, vc, si, sc = _sets([], [0])
    for h in range(2):
        O, lse = oracle.attn_rows(Q, K, V, h, np.arange(N), vi, vc, si, sc)
        assert np.array_equal(O, _f32(V[:, 0, :]))


def test_two_key_closed_form():
    N, d = 64, 32
    Q, K, V = gen_qkv(4, N, 1, 1, d, 10000.0)
    vi, vc, si, sc = _sets([0], [0])
    O, lse = oracle.attn_rows(Q, K, V, 0, np.arange(N), vi, vc, si, sc)
    q, k, v = _f32(Q[:, 0]), _f32(K[:, 0]), _f32(V[:, 0])
    np.testing.assert_array_equal(O[0], v[0])
    for i in range(1, N):
        s_i0 = q[i] @ k[0] / math.sqrt(d)
        s_ii = q[i] @ k[i] / math.sqrt(d)
        sig = 1.0 / (1.0 + math.exp(s_ii - s_i0))
        np.testing.assert_allclose(O[i], sig * v[0] + (1 - sig) * v[i], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(lse[i], max(s_i0, s_ii) + math.log1p(math.exp(-abs(s_ii - s_i0))),
                                   rtol=1e-12)


def _naive(q, k, v, scale, V, S, N):
    """Per-row loop straight from the element rule j <= i and (j in V or i-j in S)."""
    out, lses = [], []
    for i in range(N):
        keys = [j for j in range(i + 1) if (j in V) or ((i - j) in S)]
        if not keys:
            out.append(np.zeros(q.shape[1]))
            lses.append(-math.inf)
            continue
        s = [scale * float(np.dot(q[i], k[j])) for j in keys]
        m = max(s)
        w = [math.exp(x - m) for x in s]
        l = math.fsum(w)
        out.append(sum(wi * v[j] for wi, j in zip(w, keys)) / l)
        lses.append(m + math.log(l))
    return np.array(out), np.array(lses)


def test_exhaustive_tiny_masks():
    N, d = 6, 4
    Q, K, V = gen_qkv(5, N, 1, 1, d, 10000.0)
    q, k, v = _f32(Q[:, 0]), _f32(K[:, 0]), _f32(V[:, 0])
    scale = 1 / math.sqrt(d)
    for vb, sb in itertools.product(range(1 << N), repeat=2):
        Vs = [j for j in range(N) if vb >> j & 1]
        Ss = [o for o in range(N) if sb >> o & 1]
        vi, vc, si, sc = _sets(Vs, Ss, ld=N)
        O1, l1, M = oracle.attn_mask(Q, K, V, 0, vi, vc, si, sc, return_mask=True)
        want_M = np.array([[(j <= i) and (j in Vs or (i - j) in Ss) for j in range(N)]
                           for i in range(N)], np.uint8)
        assert np.array_equal(M, want_M)
        O2, l2 = oracle.attn_rows(Q, K, V, 0, np.arange(N), vi, vc, si, sc)
        np.testing.assert_array_equal(O1, O2)
        np.testing.assert_array_equal(l1, l2)
        if (vb * 31 + sb) % 17 == 0:  # python brute force on a spread-out subset
            On, ln = _naive(q, k, v, scale, set(Vs), set(Ss), N)
            np.testing.assert_allclose(O1, On, rtol=1e-12, atol=1e-14)
            np.testing.assert_allclose(l1, ln, rtol=1e-12, atol=1e-14)


def test_random_masks_rows_equal_mask_form():
    N, d = 64, 8
    Q, K, V = gen_qkv(6, N, 1, 1, d, 10000.0)
    rng = np.random.default_rng(0)
    for t in range(10000):
        dv, ds = rng.uniform(0, 0.5, 2)
        Vs = np.nonzero(rng.random(N) < dv)[0]
        Ss = np.nonzero(rng.random(N) < ds)[0]
        vi, vc, si, sc = _sets(Vs.tolist(), Ss.tolist(), ld=N)
        O1, l1, M = oracle.attn_mask(Q, K, V, 0, vi, vc, si, sc, return_mask=True)
        O2, l2 = oracle.attn_rows(Q, K, V, 0, np.arange(N), vi, vc, si, sc)
        np.testing.assert_array_equal(O1, O2)
        np.testing.assert_array_equal(l1, l2)
        if t % 500 == 0:
            assert oracle.count_pairs(N, vi[0, : vc[0]], si[0, : sc[0]]) == int(M.sum())


def test_empty_key_set():
    N, d = 16, 8
    Q, K, V = gen_qkv(8, N, 1, 1, d, 10000.0)
    vi, vc, si, sc = _sets([5], [3])
    O, lse = oracle.attn_rows(Q, K, V, 0, np.arange(N), vi, vc, si, sc)
    for i in range(3):  # rows 0..2: column 5 is in the future, offset 3 reaches before 0
        assert np.all(O[i] == 0.0) and lse[i] == -math.inf
    assert np.isfinite(lse[3:]).all()


def test_gqa_and_index_head_mapping():
    # query head h reads KV head h // (Hq/Hkv) and index-set head h*H_sel//Hq:
    # compare against single-head problems carved out by slicing.
    N, d, Hq, Hkv = 80, 16, 4, 2
    Q, K, V = gen_qkv(9, N, Hq, Hkv, d, 10000.0)
    sets = [([0, 3, 17, 40], [0, 1, 5]), ([2, 9], [0, 7, 30, 31])]
    ld = 8
    vi = np.full((2, ld), -1, np.int32)
    si = np.full((2, ld), -1, np.int32)
    vc = np.zeros(2, np.int32)
    sc = np.zeros(2, np.int32)
    for h, (a, b) in enumerate(sets):
        vi[h, : len(a)] = a
        si[h, : len(b)] = b
        vc[h], sc[h] = len(a), len(b)
    for h in range(Hq):
        O, lse = oracle.attn_rows(Q, K, V, h, np.arange(N), vi, vc, si, sc)
        g = h // (Hq // Hkv)
        hs = h * 2 // Hq
        v1, c1, s1, c2 = _sets(*sets[hs])
        O1, l1 = oracle.attn_rows(Q[:, h:h + 1], K[:, g:g + 1], V[:, g:g + 1], 0, np.arange(N),
                                  v1, c1, s1, c2)
        np.testing.assert_array_equal(O, O1)
        np.testing.assert_array_equal(lse, l1)


def test_row_subset_matches_full():
    N, d = 257, 64
    Q, K, V = gen_qkv(10, N, 1, 1, d, 10000.0)
    vi, vc, si, sc = _sets([0, 1, 100, 200], [0, 5, 64, 129])
    O, lse = oracle.attn_rows(Q, K, V, 0, np.arange(N), vi, vc, si, sc)
    rows = np.array([256, 3, 128, 0, 129])
    O2, l2 = oracle.attn_rows(Q, K, V, 0, rows, vi, vc, si, sc)
    np.testing.assert_array_equal(O[rows], O2)
    np.testing.assert_array_equal(lse[rows], l2)

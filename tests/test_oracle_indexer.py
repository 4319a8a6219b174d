"""Pins for the oracle's indexer (CPU only).

The indexer is a shared-weight two-layer linear map on concat(K with RoPE,
V) that predicts a vertical and a slash score per position (VSPrefill
summary pages, Technical Summary section 2, VSIndexer).  Pins: single-weight
probes that expose any index or transposition mistake, and PyTorch fp64
matmuls (library routine).
"""
import numpy as np
import torch

import oracle
from vs_workloads import gen_qkv


def _f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_single_weight_probes():
    N, Hkv, d, hidden = 12, 3, 8, 5
    _, K, V = gen_qkv(1, N, Hkv, Hkv, d, 10000.0)
    k, v = _f64(K), _f64(V)
    for (u, c, r, w1, w2) in [(0, 0, 0, 1.0, 1.0), (3, 2 * d - 1, 1, -2.0, 0.5),
                              (4, d, 0, 1.5, -1.0), (2, d - 1, 1, 1.0, 3.0)]:
        W1 = np.zeros((hidden, 2 * d), np.float32)
        W2 = np.zeros((2, hidden), np.float32)
        W1[u, c] = w1
        W2[r, u] = w2
        lv, ls = oracle.index_scores(K, V, W1, W2)
        x = k[..., c] if c < d else v[..., c - d]  # [N, Hkv]
        want = w2 * np.maximum(w1 * x, 0.0)
        got = lv if r == 0 else ls
        other = ls if r == 0 else lv
        np.testing.assert_array_equal(got, want.T)
        assert np.all(other == 0.0)


def test_matches_torch_fp64():
    N, Hkv, d, hidden = 50, 2, 64, 256
    _, K, V = gen_qkv(2, N, Hkv, Hkv, d, 500000.0)
    rng = np.random.default_rng(3)
    W1 = (0.02 * rng.standard_normal((hidden, 2 * d))).astype(np.float32)
    W2 = (0.02 * rng.standard_normal((2, hidden))).astype(np.float32)
    lv, ls = oracle.index_scores(K, V, W1, W2)
    x = torch.from_numpy(np.concatenate([_f64(K), _f64(V)], -1))  # [N,Hkv,2d]
    h = torch.relu(x @ torch.from_numpy(W1.astype(np.float64)).T)
    out = (h @ torch.from_numpy(W2.astype(np.float64)).T).numpy()  # [N,Hkv,2]
    np.testing.assert_allclose(lv, out[..., 0].T, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(ls, out[..., 1].T, rtol=1e-12, atol=1e-15)
    toks = np.array([49, 0, 17])
    lv2, ls2 = oracle.index_scores(K, V, W1, W2, toks)
    np.testing.assert_array_equal(lv2, lv[:, toks])
    np.testing.assert_array_equal(ls2, ls[:, toks])

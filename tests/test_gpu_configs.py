"""Full-size parity on the five workloads, run exactly as bench.py runs the hot
path (indexer -> select x2 -> sparse attention, same entry points, same
sizes): selected index sets bit-exact against the oracle on the same fp32
scores, attention within tolerance on sampled rows of every head (rows of the
first two tiles and the last tile, rows around every 64th tile boundary,
seeded random rows, and the rows at the first vertical columns)."""
import numpy as np
import pytest
import torch

import oracle
import sparse_attention_long_head_b200 as vs
from vs_testutil import (BF16_MAX_ABS, bf16_to_dev, compare_rows, dev_to_f64, sample_rows)
from vs_workloads import WORKLOADS

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def _pipeline(w):
    Qb, Kb, Vb = w.qkv()
    Q, K, V = bf16_to_dev(Qb), bf16_to_dev(Kb), bf16_to_dev(Vb)
    if w.indexer:
        W1, W2 = w.indexer_weights()
        LV = torch.empty((w.Hkv, w.N), dtype=torch.float32, device="cuda")
        LS = torch.empty_like(LV)
        vs.vs_index_scores(K, V, torch.from_numpy(W1).cuda(), torch.from_numpy(W2).cuda(), LV, LS)
    else:
        lv, ls = w.all_scores()
        LV, LS = torch.from_numpy(lv).cuda(), torch.from_numpy(ls).cuda()
    mode = vs.VS_SELECT_TOPK if w.select_mode == "topk" else vs.VS_SELECT_THRESHOLD
    vi, vc = vs.select(LV, mode, w.k_v, w.tau_v)
    si, sc = vs.select(LS, mode, w.k_s, w.tau_s)
    O, lse = vs.sparse_attention(Q, K, V, vi, vc, si, sc)
    torch.cuda.synchronize()
    return (Qb, Kb, Vb), (LV.cpu().numpy(), LS.cpu().numpy()), \
        tuple(x.cpu().numpy() for x in (vi, vc, si, sc)), O, lse, mode


@pytest.mark.parametrize("name", ["tiny_1k", "llama_8k", "llama_32k", "llama_128k",
                                  "llama_256k_indexer"])
def test_full_size_workload(name, cuda_device):
    w = WORKLOADS[name]
    (Qb, Kb, Vb), (lv, ls), (vi, vc, si, sc), O, lse, mode = _pipeline(w)
    N, Hq = w.N, w.Hq
    if w.indexer:  # indexer on sampled tokens against the fp64 oracle
        W1, W2 = w.indexer_weights()
        toks = np.unique(np.concatenate([np.arange(64), np.arange(N - 64, N),
                                         np.random.default_rng(0).integers(0, N, 512)]))
        rv, rs = oracle.index_scores(Kb, Vb, W1, W2, toks)
        assert np.abs(lv[:, toks] - rv).max() <= 1e-5
        assert np.abs(ls[:, toks] - rs).max() <= 1e-5
    # selection: bit-exact on the same fp32 scores
    ties = []
    for h in range(w.H_sel):
        for scores, idx, cnt, k, tau in ((lv[h], vi[h], vc[h], w.k_v, w.tau_v),
                                         (ls[h], si[h], sc[h], w.k_s, w.tau_s)):
            oi, oc, margin = oracle.select(scores, mode, k, tau)
            if margin < 1e-9:
                ties.append(h)
                continue
            assert cnt == oc and np.array_equal(idx, oi), (name, h)
    assert ties == [], f"tie zones {ties}"
    # attention on sampled rows of every head, with the GPU's index sets
    Od = dev_to_f64(O)
    lsed = lse.cpu().numpy().astype(np.float64)
    n_random = 256 if N <= 32768 else 96
    worst = 0.0
    for h in range(Hq):
        hs = h * w.H_sel // Hq
        rows = sample_rows(N, vi[hs, : vc[hs]], seed=h, n_random=n_random)
        Or, lr = oracle.attn_rows(Qb, Kb, Vb, h, rows, vi, vc, si, sc)
        mx, _ = compare_rows(Od[rows, h], Or, lsed[h, rows], lr, what=f"{name} head {h}")
        worst = max(worst, mx)
    assert worst <= BF16_MAX_ABS


def test_dense_full_size_sampled(cuda_device):
    w = WORKLOADS["llama_8k"]
    Qb, Kb, Vb = w.qkv()
    O, lse = vs.dense_attention(bf16_to_dev(Qb), bf16_to_dev(Kb), bf16_to_dev(Vb))
    Od = dev_to_f64(O)
    lsed = lse.cpu().numpy()
    for h in range(0, w.Hq, 3):
        rows = sample_rows(w.N, seed=100 + h, n_random=128)
        Or, lr = oracle.attn_rows(Qb, Kb, Vb, h, rows, dense=True)
        compare_rows(Od[rows, h], Or, lsed[h, rows], lr, what=f"dense head {h}")

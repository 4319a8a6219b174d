"""Full-size parity on the workloads, run exactly as bench.py runs the hot
path (indexer -> select x2 -> sparse attention, same entry points, same
sizes).  Every expected value comes from the oracle on the seeded inputs:
selected index sets bit-exact against the oracle's selection on the same fp32
scores, attention within tolerance on sampled rows of every head (rows of the
first two tiles and the last tile, rows around every 64th tile boundary,
seeded random rows, and the rows at the first vertical columns) against the
oracle's rows over the oracle's own index sets.

The indexer workload's scores are the oracle's indexer over all tokens
(fp64, rounded to fp32 as the selection's input): the GPU indexer is checked
against them within tolerance, the GPU selection runs on them, and the GPU
pipeline's own sets (from the GPU's fp32 logits) may differ from the oracle's
only in entries whose oracle score lies within the indexer tolerance of the
selection boundary."""
import numpy as np
import pytest
import torch

import oracle
import sparse_attention_long_head_b200 as vs
from vs_testutil import (BF16_MAX_ABS, bf16_to_dev, compare_rows, dev_to_f64, sample_rows)
from vs_workloads import WORKLOADS

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

IDX_TOL = 1e-5  # indexer logits, fp32 GPU vs fp64 oracle


def _oracle_select(w, lv, ls):
    sets = []
    for scores, k, tau in ((lv, w.k_v, w.tau_v), (ls, w.k_s, w.tau_s)):
        idx = np.empty((w.H_sel, k), np.int32)
        cnt = np.empty(w.H_sel, np.int32)
        for h in range(w.H_sel):
            idx[h], cnt[h], margin = oracle.select(scores[h], w.select_mode_id, k, tau)
            assert margin >= 1e-9, f"tie zone at head {h}"
        sets += [idx, cnt]
    return sets


@pytest.mark.parametrize("name", ["tiny_1k", "llama_8k", "llama_32k", "llama_128k",
                                  "llama_128k_S", "llama_128k_maxfrac", "llama_256k_indexer"])
def test_full_size_workload(name, cuda_device):
    w = WORKLOADS[name]
    N, Hq, mode = w.N, w.Hq, w.select_mode_id
    Qb, Kb, Vb = w.qkv()
    Q, K, V = bf16_to_dev(Qb), bf16_to_dev(Kb), bf16_to_dev(Vb)
    if w.indexer:
        W1, W2 = w.indexer_weights()
        rv, rs = oracle.index_scores(Kb, Vb, W1, W2)
        lv, ls = rv.astype(np.float32), rs.astype(np.float32)
    else:
        lv, ls = w.all_scores()
    o_vi, o_vc, o_si, o_sc = _oracle_select(w, lv, ls)

    # the hot path as the benchmark runs it
    if w.indexer:
        LV = torch.empty((w.Hkv, N), dtype=torch.float32, device="cuda")
        LS = torch.empty_like(LV)
        vs.vs_index_scores(K, V, torch.from_numpy(W1).cuda(), torch.from_numpy(W2).cuda(), LV, LS)
    else:
        LV, LS = torch.from_numpy(lv).cuda(), torch.from_numpy(ls).cuda()
    vi, vc = vs.select(LV, mode, w.k_v, w.tau_v)
    si, sc = vs.select(LS, mode, w.k_s, w.tau_s)
    O, lse = vs.sparse_attention(Q, K, V, vi, vc, si, sc)
    torch.cuda.synchronize()
    g_sets = [x.cpu().numpy() for x in (vi, vc, si, sc)]

    if w.indexer:
        assert np.abs(LV.cpu().numpy() - rv).max() <= IDX_TOL
        assert np.abs(LS.cpu().numpy() - rs).max() <= IDX_TOL
        # selection bit-exact on the oracle's scores
        for scores, k, tau, oi, oc in ((lv, w.k_v, w.tau_v, o_vi, o_vc),
                                       (ls, w.k_s, w.tau_s, o_si, o_sc)):
            gi, gc = vs.select(torch.from_numpy(scores).cuda(), mode, k, tau)
            assert np.array_equal(gc.cpu().numpy(), oc) and np.array_equal(gi.cpu().numpy(), oi)
        # the pipeline's own sets: any disagreement sits at the boundary
        for scores, gi, gc, oi, oc in ((lv, g_sets[0], g_sets[1], o_vi, o_vc),
                                       (ls, g_sets[2], g_sets[3], o_si, o_sc)):
            for h in range(w.H_sel):
                a, b = set(gi[h, : gc[h]].tolist()), set(oi[h, : oc[h]].tolist())
                diff = a ^ b
                assert len(diff) <= max(8, len(b) // 100), (h, len(diff))
                if diff:
                    kept_min = min(float(scores[h, j]) for j in b)
                    for j in diff:
                        assert abs(float(scores[h, j]) - kept_min) <= 4 * IDX_TOL, (h, j)
        # attention over the oracle's sets
        O, lse = vs.sparse_attention(Q, K, V, *(torch.from_numpy(x).cuda()
                                                for x in (o_vi, o_vc, o_si, o_sc)))
        torch.cuda.synchronize()
    else:
        for g, o in zip(g_sets, (o_vi, o_vc, o_si, o_sc)):
            assert np.array_equal(g, o), name

    Od = dev_to_f64(O)
    lsed = lse.cpu().numpy().astype(np.float64)
    # 4096 seeded random rows per head (1024 at 256K, where a row has ~32K keys)
    n_random = 4096 if N <= 131072 else 1024
    worst = 0.0
    for h in range(Hq):
        hs = h * w.H_sel // Hq
        rows = sample_rows(N, o_vi[hs, : o_vc[hs]], seed=h, n_random=n_random)
        Or, lr = oracle.attn_rows(Qb, Kb, Vb, h, rows, o_vi, o_vc, o_si, o_sc)
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

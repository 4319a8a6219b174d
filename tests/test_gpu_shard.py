"""Head sharding (one layer split by KV groups over ranks) checked on one GPU:
each rank's slice, as bench.head_shard cuts it and bench.py runs it (its
query heads, KV heads and index-set heads, select x2 then sparse attention,
or indexer -> select x2 -> attention), run one after another, must give
exactly the one-call output: the same index sets, and O and LSE equal bit for
bit.  Heads are independent in every kernel, so nothing may depend on which
other heads share the call."""
import numpy as np
import pytest
import torch

import bench
import sparse_attention_long_head_b200 as vs
from vs_testutil import bf16_to_dev
from vs_workloads import WORKLOADS, small_variant

pytestmark = pytest.mark.gpu


def _pipeline(w, Qb, Kb, Vb, lv, ls, W1=None, W2=None):
    Q, K, V = bf16_to_dev(Qb), bf16_to_dev(Kb), bf16_to_dev(Vb)
    N = Q.shape[0]
    if w.indexer:
        LV = torch.empty((K.shape[1], N), dtype=torch.float32, device="cuda")
        LS = torch.empty_like(LV)
        vs.vs_index_scores(K, V, torch.from_numpy(W1).cuda(), torch.from_numpy(W2).cuda(), LV, LS)
    else:
        LV, LS = torch.from_numpy(np.ascontiguousarray(lv)).cuda(), \
            torch.from_numpy(np.ascontiguousarray(ls)).cuda()
    vi, vc = vs.select(LV, w.select_mode_id, w.k_v, w.tau_v)
    si, sc = vs.select(LS, w.select_mode_id, w.k_s, w.tau_s)
    O, lse = vs.sparse_attention(Q, K, V, vi, vc, si, sc)
    torch.cuda.synchronize()
    return [x.cpu() for x in (LV, LS, vi, vc, si, sc, O, lse)]


@pytest.mark.parametrize("base,N", [("llama_128k", 8192), ("llama_256k_indexer", 4096)])
def test_head_shards_equal_one_call(base, N, cuda_device):
    w = small_variant(WORKLOADS[base], N)
    Qb, Kb, Vb = w.qkv()
    W1 = W2 = lv = ls = None
    if w.indexer:
        W1, W2 = w.indexer_weights()
    else:
        lv, ls = w.all_scores()
    full = _pipeline(w, Qb, Kb, Vb, lv, ls, W1, W2)
    LVf, LSf, vif, vcf, sif, scf, Of, lsef = full
    for world in (2, 4, 8):
        got_O = torch.empty_like(Of)
        got_lse = torch.empty_like(lsef)
        for rank in range(world):
            q0, q1, kv0, kv1, s0, s1 = bench.head_shard(w.Hq, w.Hkv, w.H_sel, world, rank)
            part = _pipeline(
                w, np.ascontiguousarray(Qb[:, q0:q1]), np.ascontiguousarray(Kb[:, kv0:kv1]),
                np.ascontiguousarray(Vb[:, kv0:kv1]),
                None if lv is None else lv[s0:s1], None if ls is None else ls[s0:s1], W1, W2)
            LV, LS, vi, vc, si, sc, O, lse = part
            assert torch.equal(LV, LVf[s0:s1]) and torch.equal(LS, LSf[s0:s1]), (world, rank)
            assert torch.equal(vc, vcf[s0:s1]) and torch.equal(sc, scf[s0:s1]), (world, rank)
            assert torch.equal(vi, vif[s0:s1]) and torch.equal(si, sif[s0:s1]), (world, rank)
            got_O[:, q0:q1] = O
            got_lse[q0:q1] = lse
        assert torch.equal(got_O, Of), world
        assert torch.equal(got_lse, lsef), world

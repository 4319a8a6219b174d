"""Variable-length batched prefill on the GPU: B sequences packed along the
token axis, each attending only to itself, vs the fp64 oracle applied to each
sequence on its own (the pages' per-sequence definition), and vs the
single-sequence entry point run on each sequence (bit-identical)."""
import numpy as np
import pytest
import torch

import oracle
import sparse_attention_long_head_b200 as vs
from vs_testutil import bf16_to_dev, compare_rows, dev_to_f64, sets_to_rows
from vs_workloads import gen_qkv

pytestmark = pytest.mark.gpu


def _batch(lengths, Hq, Hkv, d, seed):
    parts = [gen_qkv(seed + i, n, Hq, Hkv, d, 10000.0) for i, n in enumerate(lengths)]
    Qb, Kb, Vb = (np.concatenate([p[t] for p in parts]) for t in range(3))
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    return Qb, Kb, Vb, cu


def _sets(rng, lengths, H_sel):
    v_all, s_all = [], []
    for n in lengths:
        for _ in range(H_sel):
            v = np.nonzero(rng.random(n) < 0.1)[0]
            s = np.nonzero(rng.random(n) < 0.15)[0]
            if rng.random() < 0.7:
                s = np.union1d(s, [0])
            v_all.append(v)
            s_all.append(s)
    return v_all, s_all


def _run_varlen(Qb, Kb, Vb, cu, v_sets, s_sets, packed=True, max_n=None):
    Q, K, V = (bf16_to_dev(x) for x in (Qb, Kb, Vb))
    T, Hq, d = Q.shape
    B = len(cu) - 1
    H_sel = len(v_sets) // B
    vi, vc = sets_to_rows(v_sets)
    si, sc = sets_to_rows(s_sets)
    cu_d = torch.from_numpy(cu).cuda()
    max_n = max_n or int(np.diff(cu).max())
    ws = vs.workspace(vs.vs_attn_workspace_size_varlen(B, max_n, H_sel, d,
                                                       vi.shape[1] if packed else 0))
    O = torch.empty_like(Q)
    lse = torch.empty((Hq, T), dtype=torch.float32, device="cuda")
    vs.vs_sparse_attn_fwd_varlen(Q, K, V, cu_d, max_n, *(torch.from_numpy(x).cuda()
                                                         for x in (vi, vc, si, sc)), O, lse, ws)
    rc, flags = vs.vs_read_device_status(ws)
    return O, lse, (vi, vc, si, sc), rc, flags


@pytest.mark.parametrize("lengths,d,Hq,Hkv,H_sel", [
    ([1, 300, 1000, 129, 2048], 128, 4, 2, 4),
    ([640, 1, 777], 64, 2, 2, 2),
    ([256, 256, 256, 256], 128, 4, 1, 1),
    ([3000], 128, 2, 1, 2),
])
@pytest.mark.parametrize("packed", [True, False])
def test_sparse_varlen_against_oracle(lengths, d, Hq, Hkv, H_sel, packed, cuda_device):
    rng = np.random.default_rng(sum(lengths) + d)
    Qb, Kb, Vb, cu = _batch(lengths, Hq, Hkv, d, seed=len(lengths))
    v_sets, s_sets = _sets(rng, lengths, H_sel)
    O, lse, _, rc, flags = _run_varlen(Qb, Kb, Vb, cu, v_sets, s_sets, packed)
    assert rc == vs.VS_OK and flags == 0
    Od = dev_to_f64(O)
    lsed = lse.cpu().numpy().astype(np.float64)
    for b, n in enumerate(lengths):
        t0 = cu[b]
        vi, vc = sets_to_rows(v_sets[b * H_sel:(b + 1) * H_sel])
        si, sc = sets_to_rows(s_sets[b * H_sel:(b + 1) * H_sel])
        sl = slice(t0, t0 + n)
        for h in range(Hq):
            Or, lr = oracle.attn_rows(Qb[sl], Kb[sl], Vb[sl], h, np.arange(n), vi, vc, si, sc)
            compare_rows(Od[sl, h], Or, lsed[h, sl], lr, what=f"seq {b} head {h}")


def test_varlen_matches_single_sequence_calls_bitwise(cuda_device):
    lengths = [500, 1, 1300, 128]
    rng = np.random.default_rng(5)
    Qb, Kb, Vb, cu = _batch(lengths, 4, 2, 128, seed=40)
    v_sets, s_sets = _sets(rng, lengths, 2)
    O, lse, _, rc, flags = _run_varlen(Qb, Kb, Vb, cu, v_sets, s_sets)
    assert rc == vs.VS_OK and flags == 0
    for b, n in enumerate(lengths):
        sl = slice(cu[b], cu[b] + n)
        vi, vc = sets_to_rows(v_sets[2 * b:2 * b + 2])
        si, sc = sets_to_rows(s_sets[2 * b:2 * b + 2])
        Q1, K1, V1 = (bf16_to_dev(x[sl]) for x in (Qb, Kb, Vb))
        ws = vs.workspace(vs.vs_attn_workspace_size_ld(n, 4, 2, 128, vi.shape[1]))
        O1, lse1 = vs.sparse_attention(Q1, K1, V1, *(torch.from_numpy(x).cuda()
                                                     for x in (vi, vc, si, sc)), ws=ws)
        assert torch.equal(O[sl], O1), b
        assert torch.equal(lse[:, sl], lse1), b


@pytest.mark.parametrize("lengths,d", [([1, 300, 1000, 129, 2048], 128), ([640, 1, 777], 64)])
def test_dense_varlen_against_oracle(lengths, d, cuda_device):
    Qb, Kb, Vb, cu = _batch(lengths, 2, 1, d, seed=9)
    Q, K, V = (bf16_to_dev(x) for x in (Qb, Kb, Vb))
    T = Q.shape[0]
    O = torch.empty_like(Q)
    lse = torch.empty((2, T), dtype=torch.float32, device="cuda")
    ws = vs.workspace(256)
    vs.vs_dense_attn_fwd_varlen(Q, K, V, torch.from_numpy(cu).cuda(), max(lengths), O, lse, ws)
    rc, flags = vs.vs_read_device_status(ws)
    assert rc == vs.VS_OK and flags == 0
    Od = dev_to_f64(O)
    lsed = lse.cpu().numpy().astype(np.float64)
    for b, n in enumerate(lengths):
        sl = slice(cu[b], cu[b] + n)
        for h in range(2):
            Or, lr = oracle.attn_rows(Qb[sl], Kb[sl], Vb[sl], h, np.arange(n), dense=True)
            compare_rows(Od[sl, h], Or, lsed[h, sl], lr, what=f"dense seq {b} head {h}")


def test_malformed_offsets_are_flagged_and_contained(cuda_device):
    # sequence 1 is longer than max_seqlen: it is skipped and flagged; the
    # others are still correct
    lengths = [300, 500, 300]
    rng = np.random.default_rng(8)
    Qb, Kb, Vb, cu = _batch(lengths, 2, 1, 128, seed=77)
    v_sets, s_sets = _sets(rng, [300, 300, 300], 1)
    O, lse, _, rc, flags = _run_varlen(Qb, Kb, Vb, cu, v_sets, s_sets, max_n=400)
    assert rc == vs.VS_ERR_DEVICE_BOUNDS and flags & vs.VS_DEVFLAG_BOUNDS
    Od = dev_to_f64(O)
    lsed = lse.cpu().numpy().astype(np.float64)
    for b in (0, 2):
        vi, vc = sets_to_rows(v_sets[b:b + 1])
        si, sc = sets_to_rows(s_sets[b:b + 1])
        sl = slice(cu[b], cu[b + 1])
        for h in range(2):
            Or, lr = oracle.attn_rows(Qb[sl], Kb[sl], Vb[sl], h, np.arange(300), vi, vc, si, sc)
            compare_rows(Od[sl, h], Or, lsed[h, sl], lr, what=f"seq {b} head {h}")


@pytest.mark.slow
def test_full_size_batch_workload(cuda_device):
    # the bench's batch pipeline: one batched select per score type, then one
    # batched attention call; selections bit-exact against the oracle, rows of
    # every sequence sampled
    from vs_testutil import sample_rows
    from vs_workloads import BATCH_WORKLOADS
    w = BATCH_WORKLOADS["llama_varlen_mix"]
    Qb, Kb, Vb = w.qkv()
    Q, K, V = (bf16_to_dev(x) for x in (Qb, Kb, Vb))
    B, H_sel, Hq = len(w.lengths), w.H_sel, w.Hq
    cu = w.cu_seqlens
    cu_t = torch.from_numpy(cu).cuda()
    cap_max = w.cap(max(w.lengths))
    caps = torch.tensor([w.cap(n) for n in w.lengths], dtype=torch.int32, device="cuda")
    scores = [w.scores(b) for b in range(B)]
    LV = torch.from_numpy(np.ascontiguousarray(np.concatenate([x[0] for x in scores], 1))).cuda()
    LS = torch.from_numpy(np.ascontiguousarray(np.concatenate([x[1] for x in scores], 1))).cuda()
    vi, vc = vs.select_varlen(LV, cu_t, max(w.lengths), w.select_mode_id, caps, cap_max, w.tau_v)
    si, sc = vs.select_varlen(LS, cu_t, max(w.lengths), w.select_mode_id, caps, cap_max, w.tau_s)
    oracle_sets = []
    for b, n in enumerate(w.lengths):
        lv, ls = scores[b]
        k = w.cap(n)
        ovi, ovc, mv = oracle.select_heads(lv, w.select_mode_id, k, w.tau_v)
        osi, osc, ms = oracle.select_heads(ls, w.select_mode_id, k, w.tau_s)
        assert (mv >= 1e-9).all() and (ms >= 1e-9).all()
        oracle_sets.append((ovi, ovc, osi, osc))
    max_n = max(w.lengths)
    ws = vs.workspace(vs.vs_attn_workspace_size_varlen(B, max_n, H_sel, w.d, cap_max))
    O = torch.empty_like(Q)
    lse = torch.empty((Hq, Q.shape[0]), dtype=torch.float32, device="cuda")
    vs.vs_sparse_attn_fwd_varlen(Q, K, V, cu_t, max_n, vi, vc, si, sc, O, lse, ws)
    rc, flags = vs.vs_read_device_status(ws)
    assert rc == vs.VS_OK and flags == 0
    gvi, gvc, gsi, gsc = (x.cpu().numpy() for x in (vi, vc, si, sc))
    Od = dev_to_f64(O)
    lsed = lse.cpu().numpy().astype(np.float64)
    for b, n in enumerate(w.lengths):
        ovi, ovc, osi, osc = oracle_sets[b]
        k = w.cap(n)
        rows = slice(b * H_sel, (b + 1) * H_sel)
        assert np.array_equal(gvc[rows], ovc) and np.array_equal(gvi[rows, :k], ovi), b
        assert np.array_equal(gsc[rows], osc) and np.array_equal(gsi[rows, :k], osi), b
        sl = slice(cu[b], cu[b] + n)
        for h in range(0, Hq, 5):
            hs = (h * H_sel) // Hq
            rr = sample_rows(n, ovi[hs, : ovc[hs]], seed=b * 100 + h, n_random=32)
            Or, lr = oracle.attn_rows(Qb[sl], Kb[sl], Vb[sl], h, rr, ovi, ovc, osi, osc)
            compare_rows(Od[sl][rr, h], Or, lsed[h, sl][rr], lr, what=f"seq {b} head {h}")

"""Batched (variable-length) selection on the GPU: vs_select_varlen over B
sequences packed along the token axis, in one launch (the budget step of
VSPrefill Technical Summary, section 2, "Dynamic Budgeting", per sequence).

Each row (sequence b, head h) is checked against the oracle on that
sequence's scores alone: bit-exact indices and counts outside tie zones
(threshold decisions within 1e-9 of the boundary), -1 padding up to the
sequence's cap and nothing written past it; and against vs_select on the
same row.  Empty sequences keep nothing; malformed offsets and caps set the
bounds flag and leave the well-formed sequences exact."""
import numpy as np
import pytest
import torch

import oracle
import sparse_attention_long_head_b200 as vs
from vs_workloads import BATCH_WORKLOADS

pytestmark = pytest.mark.gpu

TOPK, THR, MAXF = vs.VS_SELECT_TOPK, vs.VS_SELECT_THRESHOLD, vs.VS_SELECT_MAXFRAC
UNTOUCHED = -7


def _pack(rows_per_seq):
    """[H, n_b] arrays -> ([H, total] packed, cu int32 [B + 1])."""
    lengths = [r.shape[1] for r in rows_per_seq]
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    return np.ascontiguousarray(np.concatenate(rows_per_seq, axis=1)), cu


def _run(packed, cu, caps, mode, tau, cap_max):
    H = packed.shape[0]
    B = len(cu) - 1
    max_n = max(1, int(np.max(np.diff(cu))))
    idx = torch.full((B * H, cap_max), UNTOUCHED, dtype=torch.int32, device="cuda")
    cnt = torch.full((B * H,), UNTOUCHED, dtype=torch.int32, device="cuda")
    ws = vs.workspace(vs.vs_select_workspace_size_varlen(B, H, max_n))
    vs.vs_select_varlen(torch.from_numpy(packed).cuda(), torch.from_numpy(cu).cuda(), max_n, mode,
                        torch.from_numpy(np.asarray(caps, np.int32)).cuda(), cap_max, tau, idx, cnt,
                        ws)
    rc, flags = vs.vs_read_device_status(ws)
    return idx.cpu().numpy(), cnt.cpu().numpy(), rc, flags


def _check_rows(seqs, idx, cnt, caps, mode, tau, skip=()):
    """Every row against the oracle on its sequence alone; returns tie rows."""
    H = seqs[0].shape[0]
    ties = []
    for b, s in enumerate(seqs):
        if b in skip:
            continue
        k = caps[b]
        for h in range(H):
            r = b * H + h
            if s.shape[1] == 0:
                assert cnt[r] == 0 and np.all(idx[r] == UNTOUCHED), (b, h)
                continue
            oi, oc, margin = oracle.select(s[h], mode, k, tau)
            if margin < 1e-9:
                ties.append((b, h))
                assert abs(int(cnt[r]) - oc) <= 1
                continue
            assert cnt[r] == oc, (b, h, cnt[r], oc)
            assert np.array_equal(idx[r, :k], oi), (b, h)
            assert np.all(idx[r, k:] == UNTOUCHED), (b, h)  # nothing past the cap
    return ties


@pytest.mark.parametrize("mode,tau", [(TOPK, 1.0), (THR, 0.9), (THR, 0.5), (THR, 1.0),
                                      (MAXF, 0.05), (MAXF, 1.0)])
def test_batch_against_oracle_and_single_calls(mode, tau, cuda_device):
    rng = np.random.default_rng(11 + mode)
    lengths = (1, 300, 4095, 4096, 4097, 20000, 129, 33000)
    H = 3
    seqs = [(rng.standard_normal((H, n)) * 2).astype(np.float32) for n in lengths]
    seqs[2][:, ::7] = 1.5  # ties inside one sequence
    caps = [max(1, n // 3) for n in lengths]
    caps[1] = 300  # a cap equal to the length
    packed, cu = _pack(seqs)
    cap_max = max(caps) + 5
    idx, cnt, rc, flags = _run(packed, cu, caps, mode, tau, cap_max)
    assert rc == vs.VS_OK and flags == 0
    ties = _check_rows(seqs, idx, cnt, caps, mode, tau)
    assert ties == []
    # the same rows through vs_select, one sequence at a time
    for b, s in enumerate(seqs):
        gi, gc = vs.select(torch.from_numpy(s).cuda(), mode, caps[b], tau)
        gi, gc = gi.cpu().numpy(), gc.cpu().numpy()
        for h in range(H):
            assert cnt[b * H + h] == gc[h], (b, h)
            assert np.array_equal(idx[b * H + h, :caps[b]], gi[h]), (b, h)


def test_empty_sequences_keep_nothing(cuda_device):
    rng = np.random.default_rng(5)
    H = 2
    lengths = (0, 500, 0, 1, 0)
    seqs = [rng.standard_normal((H, n)).astype(np.float32) for n in lengths]
    caps = [7, 100, 3, 1, 9]
    packed, cu = _pack(seqs)
    idx, cnt, rc, flags = _run(packed, cu, caps, THR, 0.9, 128)
    assert rc == vs.VS_OK and flags == 0
    assert _check_rows(seqs, idx, cnt, caps, THR, 0.9) == []


def test_malformed_offsets_and_caps_flag_bounds(cuda_device):
    rng = np.random.default_rng(6)
    H = 2
    lengths = (400, 300, 500, 200)
    seqs = [rng.standard_normal((H, n)).astype(np.float32) for n in lengths]
    packed, cu = _pack(seqs)
    caps = [50, 60, 70, 80]
    # sequence 1 ends before it starts (its offsets are malformed; sequence 2
    # then starts later than its true start, so only 0 and 3 stay checkable)
    bad = cu.copy()
    bad[2] = bad[1] - 10
    idx, cnt, rc, flags = _run(packed, bad, caps, TOPK, 1.0, 128)
    assert rc == vs.VS_ERR_DEVICE_BOUNDS and flags & vs.VS_DEVFLAG_BOUNDS
    assert np.all(cnt[H:2 * H] == 0) and np.all(idx[H:2 * H] == UNTOUCHED)
    _check_rows(seqs, idx, cnt, caps, TOPK, 1.0, skip=(1, 2))
    # a cap above its sequence's length, and a zero cap
    for badcap in ([50, 301, 70, 80], [50, 60, 0, 80]):
        idx, cnt, rc, flags = _run(packed, cu, badcap, TOPK, 1.0, 400)
        assert rc == vs.VS_ERR_DEVICE_BOUNDS and flags & vs.VS_DEVFLAG_BOUNDS
        b = 1 if badcap[1] == 301 else 2
        assert np.all(cnt[b * H:(b + 1) * H] == 0)
        assert np.all(idx[b * H:(b + 1) * H] == UNTOUCHED)
        _check_rows(seqs, idx, cnt, badcap, TOPK, 1.0, skip=(b,))


@pytest.mark.slow
def test_full_size_batch_workload_scores(cuda_device):
    # the batch workload's score vectors (17 sequences of 256-32768 tokens, 32
    # heads, threshold 0.90 / 0.95, caps 1/8 of each length): one launch per
    # score type, every row equal to the oracle's selection
    w = BATCH_WORKLOADS["llama_varlen_mix"]
    caps = [w.cap(n) for n in w.lengths]
    cap_max = w.cap(max(w.lengths))
    sv, ss = zip(*(w.scores(b) for b in range(len(w.lengths))))
    for seqs, tau in ((sv, w.tau_v), (ss, w.tau_s)):
        packed, cu = _pack(list(seqs))
        idx, cnt, rc, flags = _run(packed, cu, caps, w.select_mode_id, tau, cap_max)
        assert rc == vs.VS_OK and flags == 0
        assert _check_rows(list(seqs), idx, cnt, caps, w.select_mode_id, tau) == []


def test_many_long_rows_two_cta_clusters(cuda_device):
    # rows longer than one CTA's key cache (32768 keys) and more rows than a
    # wave of SMs holds at 8 CTAs per row: the launch takes 2-CTA clusters
    rng = np.random.default_rng(8)
    H = 4
    lengths = tuple(int(x) for x in rng.integers(30000, 40001, 20))
    seqs = [(rng.standard_normal((H, n)) * 2).astype(np.float32) for n in lengths]
    caps = [n // 8 for n in lengths]
    packed, cu = _pack(seqs)
    for mode, tau in ((THR, 0.9), (TOPK, 1.0)):
        idx, cnt, rc, flags = _run(packed, cu, caps, mode, tau, max(caps))
        assert rc == vs.VS_OK and flags == 0
        assert _check_rows(seqs, idx, cnt, caps, mode, tau) == []

"""Helpers shared by the GPU parity tests (marshalling and comparison only)."""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
import sparse_attention_long_head_b200 as vs

# Tolerances against the fp64 oracle on identical inputs and index sets.
BF16_MAX_ABS = 2e-2
BF16_MEAN_ABS = 2e-3
FP32_MAX_ABS = 1e-3
LSE_MAX_ABS = 1e-3


def bf16_to_dev(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def dev_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


def sets_to_rows(sets, ld=None):
    """list of index lists -> (idx int32 [H, ld] padded -1, cnt int32 [H])"""
    H = len(sets)
    ld = ld or max(1, max(len(s) for s in sets))
    idx = np.full((H, ld), -1, np.int32)
    cnt = np.zeros(H, np.int32)
    for h, s in enumerate(sets):
        s = np.asarray(s, np.int32)
        idx[h, : s.size] = s
        cnt[h] = s.size
    return idx, cnt


def check_select(scores: np.ndarray, mode: int, k: int, tau: float = 1.0, ld_scores=None,
                 ld_idx=None):
    """GPU vs oracle on the same fp32 scores. Returns the list of tie-zone heads."""
    H, N = scores.shape
    s = torch.full((H, ld_scores or N), float("nan"), dtype=torch.float32, device="cuda")
    s[:, :N] = torch.from_numpy(scores).cuda()
    idx = torch.full((H, ld_idx or k), -7, dtype=torch.int32, device="cuda")
    cnt = torch.empty(H, dtype=torch.int32, device="cuda")
    ws = vs.workspace(vs.vs_select_workspace_size(H, N))
    vs.vs_select(s[:, :N] if ld_scores is None else s.as_strided((H, N), (ld_scores, 1)), mode, k,
                 tau, idx, cnt, ws)
    rc, flags = vs.vs_read_device_status(ws)
    assert rc == vs.VS_OK and flags == 0
    gi = idx.cpu().numpy()
    gc = cnt.cpu().numpy()
    ties = []
    for h in range(H):
        oi, oc, margin = oracle.select(scores[h], mode, k, tau)
        if margin < 1e-9:
            ties.append(h)
            assert abs(int(gc[h]) - oc) <= 1
            continue
        assert gc[h] == oc, (h, gc[h], oc)
        assert np.array_equal(gi[h, :k], oi), h
        if ld_idx and ld_idx > k:
            assert np.all(gi[h, k:] == -7)  # untouched past k_or_cap
    return ties


def compare_rows(O_gpu: np.ndarray, O_ref: np.ndarray, lse_gpu, lse_ref, fp32=False, what=""):
    err = np.abs(O_gpu - O_ref)
    mx = float(err.max()) if err.size else 0.0
    mean = float(err.mean()) if err.size else 0.0
    if fp32:
        assert mx <= FP32_MAX_ABS, f"{what}: fp32 max-abs {mx}"
    else:
        assert mx <= BF16_MAX_ABS, f"{what}: max-abs {mx}"
        assert mean <= BF16_MEAN_ABS, f"{what}: mean-abs {mean}"
    if lse_gpu is not None:
        inf_ref = np.isneginf(lse_ref)
        assert np.array_equal(np.isneginf(lse_gpu), inf_ref), what
        if (~inf_ref).any():
            le = float(np.abs(lse_gpu[~inf_ref] - lse_ref[~inf_ref]).max())
            assert le <= LSE_MAX_ABS, f"{what}: lse max-abs {le}"
    return mx, mean


def run_sparse(Qb, Kb, Vb, v_sets, s_sets, fp32=False, vld=None, sld=None):
    """Runs the GPU sparse kernel on numpy inputs; returns (O f64 [N,Hq,d], lse [Hq,N], ws)."""
    vi, vc = sets_to_rows(v_sets, vld)
    si, sc = sets_to_rows(s_sets, sld)
    if fp32:
        Q, K, V = (torch.from_numpy(x).cuda() for x in (Qb, Kb, Vb))
    else:
        Q, K, V = (bf16_to_dev(x) for x in (Qb, Kb, Vb))
    N, Hq, d = Q.shape
    ws = vs.workspace(vs.vs_attn_workspace_size(N, Hq, len(v_sets), d))
    O, lse = vs.sparse_attention(Q, K, V, torch.from_numpy(vi).cuda(), torch.from_numpy(vc).cuda(),
                                 torch.from_numpy(si).cuda(), torch.from_numpy(sc).cuda(), ws=ws)
    rc, flags = vs.vs_read_device_status(ws)
    assert rc == vs.VS_OK, (rc, flags)
    return dev_to_f64(O), lse.cpu().numpy().astype(np.float64), (vi, vc, si, sc)


def oracle_rows(Qb, Kb, Vb, h, rows, sets=None, dense=False):
    if dense:
        return oracle.attn_rows(Qb, Kb, Vb, h, rows, dense=True)
    vi, vc, si, sc = sets
    return oracle.attn_rows(Qb, Kb, Vb, h, rows, vi, vc, si, sc)


def sample_rows(N: int, v_first=(), seed=0, n_random=256):
    """Rows of tiles 0, 1 and the last; rows 127/128 of every 64th tile boundary;
    seeded random rows; the rows at the first vertical columns."""
    T = (N + 127) // 128
    rows = set(range(0, min(N, 256)))
    rows |= set(range(max(0, (T - 1) * 128), N))
    for t in range(0, T, 64):
        for r in (128 * t - 1, 128 * t, 128 * t + 127, 128 * t + 128):
            if 0 <= r < N:
                rows.add(r)
    rng = np.random.default_rng(seed)
    rows |= set(int(x) for x in rng.integers(0, N, n_random))
    rows |= set(int(j) for j in list(v_first)[:16] if 0 <= j < N)
    return np.array(sorted(rows), np.int64)


def pairs_from_sets(N, vlist, slist):
    return oracle.count_pairs(N, np.asarray(vlist, np.int32), np.asarray(slist, np.int32))

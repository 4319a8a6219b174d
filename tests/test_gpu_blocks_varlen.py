"""Batched (variable-length) FlashPrefill-style block path on the GPU: block
discovery and block-sparse attention over B sequences packed along the token
axis (FlashPrefill summary page, sections 2A, 2B and 3, per sequence).

Each sequence's kept-block mask is bit-exact against the oracle run on that
sequence alone, rows past its block count are zero, and both its mask and
its attention output are bit-identical to the single-sequence calls on the
same sequence; attention rows are within the bf16 tolerances of the oracle
over the oracle's masks."""
import numpy as np
import pytest
import torch

import oracle
import sparse_attention_long_head_b200 as vs
from vs_testutil import bf16_to_dev, compare_rows, dev_to_f64, sample_rows
from vs_workloads import gen_qkv, plant_block_structure

pytestmark = pytest.mark.gpu


def _batch(lengths, Hq, Hkv, d, seed):
    parts = []
    for b, n in enumerate(lengths):
        Qb, Kb, Vb = gen_qkv(seed * 100 + b, n, Hq, Hkv, d, 500000.0)
        Qb, Kb = plant_block_structure(Qb, Kb, seed=seed * 100 + b)
        parts.append((Qb, Kb, Vb))
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    cat = tuple(np.concatenate([p[t] for p in parts]) for t in range(3))
    return parts, cu, cat


@pytest.mark.parametrize("lengths,Hq,Hkv,d,alpha", [
    ((300, 1000, 129, 2048, 1), 4, 2, 128, 0.2),
    ((3000, 700, 128, 1500), 8, 2, 64, 0.3),
    ((4097, 257), 4, 4, 128, 0.05),
])
def test_block_varlen_against_oracle_and_single_calls(lengths, Hq, Hkv, d, alpha, cuda_device):
    parts, cu, (Qc, Kc, Vc) = _batch(lengths, Hq, Hkv, d, seed=len(lengths) + d)
    Q, K, V = bf16_to_dev(Qc), bf16_to_dev(Kc), bf16_to_dev(Vc)
    cu_t = torch.from_numpy(cu).cuda()
    maxN = max(lengths)
    O, lse, mask = vs.block_prefill_varlen(Q, K, V, cu_t, maxN, alpha)
    torch.cuda.synchronize()
    m = mask.cpu().numpy().view(np.uint32)  # [B, Hq, T, W]
    Od = dev_to_f64(O)
    lsed = lse.cpu().numpy().astype(np.float64)
    for b, (Qb, Kb, Vb) in enumerate(parts):
        n = lengths[b]
        t0, t1 = int(cu[b]), int(cu[b + 1])
        Tb = (n + 127) // 128
        Wb = (Tb + 31) // 32
        ref, margin = oracle.block_select(Qb, Kb, alpha)
        assert (margin > 1e-9).all(), margin
        got = m[b, :, :Tb, :Wb]
        assert np.array_equal(got, ref), b
        assert not m[b, :, :Tb, Wb:].any() and not m[b, :, Tb:, :].any(), b
        # the single-sequence calls on the same sequence: identical bits
        O1, lse1, m1 = vs.block_prefill(*(bf16_to_dev(x) for x in (Qb, Kb, Vb)), alpha)
        torch.cuda.synchronize()
        assert np.array_equal(m1.cpu().numpy().view(np.uint32), got), b
        assert torch.equal(O[t0:t1], O1), b
        assert torch.equal(lse[:, t0:t1], lse1), b
        rows = sample_rows(n, seed=b, n_random=128)
        for h in range(Hq):
            Or, lr = oracle.attn_block_rows(Qb, Kb, Vb, h, rows, ref)
            compare_rows(Od[t0 + rows, h], Or, lsed[h, t0 + rows], lr, what=f"seq {b} head {h}")


def test_block_varlen_malformed_offsets_flag_bounds(cuda_device):
    # a decreasing offset empties that sequence and sets the bounds flag; the
    # well-formed sequences are still selected exactly
    lengths = (400, 300, 500)
    parts, cu, (Qc, Kc, _) = _batch(lengths, 2, 1, 128, seed=9)
    bad = cu.copy()
    bad[2] = bad[1] - 50  # sequence 1 ends before it starts
    Q, K = bf16_to_dev(Qc), bf16_to_dev(Kc)
    maxN = max(lengths)
    T = (maxN + 127) // 128
    mask = torch.full((3, 2, T, (T + 31) // 32), -1, dtype=torch.int32, device="cuda")
    ws = vs.workspace(vs.vs_block_select_workspace_size_varlen(3, maxN, 1, 128))
    vs.vs_block_select_varlen(Q, K, torch.from_numpy(bad).cuda(), maxN, 0.3, mask, ws)
    rc, flags = vs.vs_read_device_status(ws)
    assert rc == vs.VS_ERR_DEVICE_BOUNDS and flags & vs.VS_DEVFLAG_BOUNDS
    m = mask.cpu().numpy().view(np.uint32)
    assert not m[1].any()  # the emptied sequence keeps nothing
    ref, _ = oracle.block_select(*parts[0][:2], 0.3)
    Tb = (lengths[0] + 127) // 128
    assert np.array_equal(m[0, :, :Tb, :1], ref)

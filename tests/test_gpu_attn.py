"""Sparse / dense attention on the GPU vs the fp64 oracle on identical inputs
and index sets: bf16 max-abs <= 2e-2 and mean-abs <= 2e-3, fp32 max-abs
<= 1e-3, LSE max-abs <= 1e-3 (-inf exactly where the key set is empty)."""
import numpy as np
import pytest
import torch

import oracle
import sparse_attention_long_head_b200 as vs
from vs_testutil import (bf16_to_dev, compare_rows, dev_to_f64, oracle_rows, run_sparse,
                         sets_to_rows)
from vs_workloads import bf16_bits_to_f32, gen_qkv, gen_qkv_f32

pytestmark = pytest.mark.gpu


def _all_rows_check(Qb, Kb, Vb, v_sets, s_sets, fp32=False, what=""):
    O, lse, sets = run_sparse(Qb, Kb, Vb, v_sets, s_sets, fp32=fp32)
    N, Hq, d = Qb.shape
    for h in range(Hq):
        Or, lr = oracle_rows(Qb, Kb, Vb, h, np.arange(N), sets)
        compare_rows(O[:, h], Or, lse[h], lr, fp32=fp32, what=f"{what} head {h}")
    return O, lse


def _random_sets(rng, N, H, dv, ds, force0=True):
    vs_, ss = [], []
    for _ in range(H):
        v = np.nonzero(rng.random(N) < dv)[0]
        s = np.nonzero(rng.random(N) < ds)[0]
        if force0:
            v = np.union1d(v, [0])
            s = np.union1d(s, [0])
        vs_.append(v)
        ss.append(s)
    return vs_, ss


@pytest.mark.parametrize("N,d", [(1000, 128), (1000, 64), (128, 128), (129, 64), (1, 128),
                                 (300, 128), (640, 64)])
def test_scattered_sets(N, d, cuda_device):
    rng = np.random.default_rng(N + d)
    Qb, Kb, Vb = gen_qkv(N, N, 4, 2, d, 10000.0)
    v_sets, s_sets = _random_sets(rng, N, 4, 0.1, 0.2)
    _all_rows_check(Qb, Kb, Vb, v_sets, s_sets, what=f"scattered N={N} d={d}")


@pytest.mark.parametrize("N,d", [(1000, 128), (2000, 64), (777, 128)])
def test_clustered_sets_split_path(N, d, cuda_device):
    # few verticals, short contiguous slash band: most units take the gathered
    # vertical chunks + touched block-diagonals
    rng = np.random.default_rng(7)
    Qb, Kb, Vb = gen_qkv(3 + N, N, 4, 1, d, 10000.0)
    v_sets = [np.array([0, 1, 2, 3]), np.sort(rng.choice(N, 300, replace=False)),
              np.sort(rng.choice(N, 5, replace=False)), np.array([], np.int64)]
    s_sets = [np.arange(0, 50), np.arange(0, 4), np.array([0, 200, 201, 202]), np.arange(10, 30)]
    _all_rows_check(Qb, Kb, Vb, v_sets, s_sets, what=f"clustered N={N} d={d}")


def test_vertical_heavy_gather(cuda_device):
    # many vertical chunks (gather4 path) with chunks straddling the diagonal
    N, d = 1536, 128
    rng = np.random.default_rng(8)
    Qb, Kb, Vb = gen_qkv(9, N, 2, 1, d, 500000.0)
    v_sets = [np.sort(rng.choice(N, 700, replace=False)), np.sort(rng.choice(N, 129, replace=False))]
    s_sets = [np.array([0, 1]), np.array([0])]
    _all_rows_check(Qb, Kb, Vb, v_sets, s_sets, what="vertical heavy")


def test_slash_zero_returns_v_exactly(cuda_device):
    N, d = 700, 128
    Qb, Kb, Vb = gen_qkv(10, N, 2, 2, d, 10000.0)
    O, lse, _ = run_sparse(Qb, Kb, Vb, [[], []], [[0], [0]])
    Vf = bf16_bits_to_f32(Vb).astype(np.float64)
    assert np.array_equal(O[:, 0], Vf[:, 0]) and np.array_equal(O[:, 1], Vf[:, 1])


def test_empty_sets_and_empty_rows(cuda_device):
    N, d = 400, 64
    Qb, Kb, Vb = gen_qkv(11, N, 2, 1, d, 10000.0)
    # head 0: nothing selected at all; head 1: column 300 and offset 250 only
    O, lse = _all_rows_check(Qb, Kb, Vb, [[], [300]], [[], [250]], what="empty")
    assert np.all(O[:, 0] == 0) and np.all(np.isneginf(lse[0]))
    assert np.all(O[:250, 1] == 0) and np.isneginf(lse[1, :250]).all()


def test_all_columns_equals_dense(cuda_device):
    N, d = 900, 128
    Qb, Kb, Vb = gen_qkv(12, N, 4, 2, d, 500000.0)
    O, lse, _ = run_sparse(Qb, Kb, Vb, [np.arange(N)] * 4, [[N - 1]] * 4)
    for h in range(4):
        Or, lr = oracle_rows(Qb, Kb, Vb, h, np.arange(N), dense=True)
        compare_rows(O[:, h], Or, lse[h], lr, what=f"all-columns head {h}")


def test_gqa_shared_index_sets(cuda_device):
    # H_sel = Hkv: each index set shared by its group of query heads
    N, d = 1100, 128
    rng = np.random.default_rng(13)
    Qb, Kb, Vb = gen_qkv(14, N, 8, 2, d, 500000.0)
    v_sets, s_sets = _random_sets(rng, N, 2, 0.05, 0.1)
    _all_rows_check(Qb, Kb, Vb, v_sets, s_sets, what="gqa H_sel=Hkv")


def test_unsorted_duplicate_indices_are_sets(cuda_device):
    N, d = 500, 64
    Qb, Kb, Vb = gen_qkv(15, N, 1, 1, d, 10000.0)
    v = [0, 100, 3, 100, 77]
    s = [5, 0, 5, 64, 1]
    O1, l1, _ = run_sparse(Qb, Kb, Vb, [v], [s])
    O2, l2, _ = run_sparse(Qb, Kb, Vb, [sorted(set(v))], [sorted(set(s))])
    assert np.array_equal(O1, O2) and np.array_equal(l1, l2)


def test_out_of_range_indices_flag_bounds(cuda_device):
    N, d = 256, 64
    Qb, Kb, Vb = gen_qkv(16, N, 1, 1, d, 10000.0)
    vi, vc = sets_to_rows([[0, 5, N + 3, -2]])
    si, sc = sets_to_rows([[0, 1, 10 * N]])
    Q, K, V = (bf16_to_dev(x) for x in (Qb, Kb, Vb))
    ws = vs.workspace(vs.vs_attn_workspace_size(N, 1, 1, d))
    O, lse = vs.sparse_attention(Q, K, V, torch.from_numpy(vi).cuda(), torch.from_numpy(vc).cuda(),
                                 torch.from_numpy(si).cuda(), torch.from_numpy(sc).cuda(), ws=ws)
    rc, flags = vs.vs_read_device_status(ws)
    assert rc == vs.VS_ERR_DEVICE_BOUNDS and flags & vs.VS_DEVFLAG_BOUNDS
    # the in-range entries are still honoured
    Or, lr = oracle.attn_rows(Qb, Kb, Vb, 0, np.arange(N), *sets_to_rows([[0, 5]]),
                              *sets_to_rows([[0, 1]]))
    compare_rows(dev_to_f64(O)[:, 0], Or, lse.cpu().numpy()[0], lr, what="bounds")


@pytest.mark.parametrize("N,d,Hq,Hkv", [(1000, 128, 4, 2), (333, 64, 2, 2), (2048, 128, 2, 1)])
def test_dense_api(N, d, Hq, Hkv, cuda_device):
    Qb, Kb, Vb = gen_qkv(17, N, Hq, Hkv, d, 500000.0)
    Q, K, V = (bf16_to_dev(x) for x in (Qb, Kb, Vb))
    O, lse = vs.dense_attention(Q, K, V)
    O = dev_to_f64(O)
    lse = lse.cpu().numpy()
    for h in range(Hq):
        Or, lr = oracle_rows(Qb, Kb, Vb, h, np.arange(N), dense=True)
        compare_rows(O[:, h], Or, lse[h], lr, what=f"dense head {h}")


def test_fp32_path(cuda_device):
    N, d = 1024, 64
    rng = np.random.default_rng(18)
    Qf, Kf, Vf = gen_qkv_f32(19, N, 2, 1, d, 10000.0)
    v_sets, s_sets = _random_sets(rng, N, 2, 0.03, 0.03)
    _all_rows_check(Qf, Kf, Vf, v_sets, s_sets, fp32=True, what="fp32")
    Q, K, V = (torch.from_numpy(x).cuda() for x in (Qf, Kf, Vf))
    O, lse = vs.dense_attention(Q, K, V)
    for h in range(2):
        Or, lr = oracle.attn_rows(Qf, Kf, Vf, h, np.arange(N), dense=True)
        compare_rows(O[:, h].cpu().numpy().astype(np.float64), Or, lse[h].cpu().numpy(), lr,
                     fp32=True, what="fp32 dense")


def test_custom_scale_and_strided_tokens(cuda_device):
    N, d, Hq, Hkv = 600, 128, 2, 1
    Qb, Kb, Vb = gen_qkv(20, N, Hq, Hkv, d, 10000.0)
    # token rows padded: stride 2 * H * d
    Qp = torch.zeros((N, 2 * Hq * d), dtype=torch.bfloat16, device="cuda")
    Kp = torch.zeros((N, 2 * Hkv * d), dtype=torch.bfloat16, device="cuda")
    Vp = torch.zeros((N, 2 * Hkv * d), dtype=torch.bfloat16, device="cuda")
    Qp[:, : Hq * d] = bf16_to_dev(Qb).reshape(N, -1)
    Kp[:, : Hkv * d] = bf16_to_dev(Kb).reshape(N, -1)
    Vp[:, : Hkv * d] = bf16_to_dev(Vb).reshape(N, -1)
    Q = Qp.as_strided((N, Hq, d), (2 * Hq * d, d, 1))
    K = Kp.as_strided((N, Hkv, d), (2 * Hkv * d, d, 1))
    V = Vp.as_strided((N, Hkv, d), (2 * Hkv * d, d, 1))
    O = torch.zeros_like(Qp).as_strided((N, Hq, d), (2 * Hq * d, d, 1))
    lse = torch.empty((Hq, N), dtype=torch.float32, device="cuda")
    vi, vc = sets_to_rows([[0, 7, 400], [1]])
    si, sc = sets_to_rows([[0, 3], [0, 1, 2, 300]])
    ws = vs.workspace(vs.vs_attn_workspace_size(N, Hq, 2, d))
    vs.vs_sparse_attn_fwd(Q, K, V, torch.from_numpy(vi).cuda(), torch.from_numpy(vc).cuda(),
                          torch.from_numpy(si).cuda(), torch.from_numpy(sc).cuda(), O, lse, ws,
                          softmax_scale=0.05)
    Od = dev_to_f64(O)
    for h in range(Hq):
        Or, lr = oracle.attn_rows(Qb, Kb, Vb, h, np.arange(N), vi, vc, si, sc, scale=0.05)
        compare_rows(Od[:, h], Or, lse[h].cpu().numpy(), lr, what=f"strided head {h}")


def test_packed_and_gathered_vertical_paths_agree(cuda_device):
    # same call with the plan-only workspace (row gathers) and with room to
    # pack the vertical rows (tile loads): identical outputs
    N, d = 3000, 128
    rng = np.random.default_rng(21)
    Qb, Kb, Vb = gen_qkv(22, N, 4, 2, d, 500000.0)
    v_sets = [np.sort(rng.choice(N, n, replace=False)) for n in (700, 129, 1, 0)]
    s_sets = [np.array([0, 1, 2]), np.arange(0, 40), np.array([0]), np.array([5, 900])]
    vi, vc = sets_to_rows(v_sets, 1000)
    si, sc = sets_to_rows(s_sets)
    Q, K, V = (bf16_to_dev(x) for x in (Qb, Kb, Vb))
    args = [torch.from_numpy(x).cuda() for x in (vi, vc, si, sc)]
    outs = []
    for nbytes in (vs.vs_attn_workspace_size(N, 4, 4, d),
                   vs.vs_attn_workspace_size_ld(N, 4, 4, d, vi.shape[1])):
        ws = vs.workspace(nbytes)
        O, lse = vs.sparse_attention(Q, K, V, *args, ws=ws)
        assert vs.vs_read_device_status(ws)[0] == vs.VS_OK
        outs.append((O.clone(), lse.clone()))
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
    Od = dev_to_f64(outs[1][0])
    for h in range(4):
        Or, lr = oracle.attn_rows(Qb, Kb, Vb, h, np.arange(N), vi, vc, si, sc)
        compare_rows(Od[:, h], Or, outs[1][1][h].cpu().numpy(), lr, what=f"packed head {h}")


@pytest.mark.slow
def test_maximum_sequence_length(cuda_device):
    # N = 2^22, the largest vs_sparse_attn_fwd accepts: one head, d = 64, few
    # keys per row; sampled rows (first / last tiles, tile boundaries, rows
    # at and after the selected columns and offsets)
    from vs_testutil import sample_rows
    N, d = 1 << 22, 64
    Qb, Kb, Vb = gen_qkv(22, N, 1, 1, d, 500000.0)
    v = np.array([0, 5, 130, 1_000_000, 4_000_000])
    s = np.array([0, 1, 2, 100, 127, 128, 3_000_000])
    vi, vc = sets_to_rows([v])
    si, sc = sets_to_rows([s])
    Q, K, V = (bf16_to_dev(x) for x in (Qb, Kb, Vb))
    ws = vs.workspace(vs.vs_attn_workspace_size_ld(N, 1, 1, d, vi.shape[1]))
    O, lse = vs.sparse_attention(Q, K, V, *(torch.from_numpy(x).cuda() for x in (vi, vc, si, sc)),
                                 ws=ws)
    rc, flags = vs.vs_read_device_status(ws)
    assert rc == vs.VS_OK and flags == 0
    rows = np.unique(np.concatenate([sample_rows(N, v, seed=1, n_random=200),
                                     v, v + 1, s, s + 1, s + 3_000_000 - s.min()]))
    rows = rows[rows < N]
    Or, lr = oracle.attn_rows(Qb, Kb, Vb, 0, rows, vi, vc, si, sc)
    compare_rows(dev_to_f64(O)[rows, 0], Or, lse.cpu().numpy().astype(np.float64)[0, rows], lr,
                 what="N = 2^22")


def _unit_plan(N, v, s, p):
    """The attention kernel's per-unit choice for the 256-row unit at pair p,
    restated from the plan's definition (key blocks on block-diagonals touched
    by an offset, 128-column chunks of the columns <= the unit's last row):
    returns (vertical chunks, slash key blocks, dense key blocks)."""
    T = (N + 127) // 128
    touched = set()
    for o in s:
        touched.add(int(o) >> 7)
        if (int(o) & 127) and (int(o) >> 7) + 1 < T:
            touched.add((int(o) >> 7) + 1)
    d1 = touched | {t + 1 for t in touched}
    last_b = min(2 * p + 1, T - 1)
    nslash = sum(1 for x in d1 if 2 * p + 1 - last_b <= x <= 2 * p + 1)
    nvc = (int(np.count_nonzero(np.asarray(v) <= min(256 * p + 255, N - 1))) + 127) // 128
    return nvc, nslash, last_b + 1


@pytest.mark.slow
def test_split_path_many_vertical_chunks(cuda_device):
    # N = 32768: the last units stream 64-128 vertical chunks each (split
    # mode), the chunks at the diagonal straddle it (columns above some rows
    # of the unit), and many columns also lie on selected diagonals (counted
    # once).  Run with the plan-only workspace (row gathers) and with room
    # for the packed rows (tile loads): identical outputs, checked against
    # the oracle on the last two units' rows and sampled rows of every head.
    from vs_testutil import sample_rows
    N, d, Hq, Hkv = 32768, 128, 4, 2
    rng = np.random.default_rng(31)
    Qb, Kb, Vb = gen_qkv(32, N, Hq, Hkv, d, 500000.0)
    v_sets = [np.sort(rng.choice(N, 9000, replace=False)),
              np.arange(0, N, 4)[:8200],
              np.sort(rng.choice(N, 16384, replace=False)),
              np.sort(rng.choice(np.arange(3 * N // 4, N), 8192, replace=False))]
    s_sets = [np.concatenate([np.arange(0, 50), [300, 1000, 5000]]),
              np.concatenate([np.arange(0, 64), [127, 128, 129]]),
              np.array([0, 1, 2]),
              np.concatenate([np.arange(0, 10), [20000]])]
    P = (N // 128 + 1) // 2
    for v, s in zip(v_sets, s_sets):
        for p in (P - 1, P - 2):
            nvc, nslash, ndense = _unit_plan(N, v, s, p)
            assert nvc + nslash < ndense and (p < P - 1 or nvc >= 64), (nvc, nslash, ndense)
        assert np.intersect1d(v, N - 1 - s).size > 0  # a column on a selected diagonal
    vi, vc = sets_to_rows(v_sets)
    si, sc = sets_to_rows(s_sets)
    Q, K, V = (bf16_to_dev(x) for x in (Qb, Kb, Vb))
    args = [torch.from_numpy(x).cuda() for x in (vi, vc, si, sc)]
    outs = []
    for nbytes in (vs.vs_attn_workspace_size(N, Hq, Hq, d),
                   vs.vs_attn_workspace_size_ld(N, Hq, Hq, d, vi.shape[1])):
        ws = vs.workspace(nbytes)
        O, lse = vs.sparse_attention(Q, K, V, *args, ws=ws)
        rc, flags = vs.vs_read_device_status(ws)
        assert rc == vs.VS_OK and flags == 0
        outs.append((O.clone(), lse.clone()))
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])
    Od = dev_to_f64(outs[1][0])
    lsed = outs[1][1].cpu().numpy().astype(np.float64)
    for h in range(Hq):
        rows = np.union1d(np.arange(N - 512, N), sample_rows(N, v_sets[h], seed=h, n_random=1024))
        Or, lr = oracle.attn_rows(Qb, Kb, Vb, h, rows, vi, vc, si, sc)
        compare_rows(Od[rows, h], Or, lsed[h, rows], lr, what=f"many chunks head {h}")

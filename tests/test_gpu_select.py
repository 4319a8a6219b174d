"""vs_select on the GPU vs the oracle: bit-exact index sets and counts on the
same fp32 scores (ties to the smaller index; threshold decisions within 1e-9
of the boundary are reported as tie zones)."""
import numpy as np
import pytest

import sparse_attention_long_head_b200 as vs
from vs_testutil import check_select
from vs_workloads import WORKLOADS

pytestmark = pytest.mark.gpu

TOPK, THR, MAXF = vs.VS_SELECT_TOPK, vs.VS_SELECT_THRESHOLD, vs.VS_SELECT_MAXFRAC


@pytest.mark.parametrize("name", ["tiny_1k", "llama_8k", "llama_32k", "llama_128k", "llama_128k_S"])
def test_workload_scores(name, cuda_device):
    w = WORKLOADS[name]
    lv, ls = w.all_scores()
    mode = w.select_mode_id
    ties = check_select(lv, mode, w.k_v, w.tau_v)
    ties += check_select(ls, mode, w.k_s, w.tau_s)
    assert ties == [], f"tie zones at heads {ties}"


@pytest.mark.parametrize("N", [1, 2, 100, 4095, 4096, 4097, 33000, 131071])
@pytest.mark.parametrize("mode,tau", [(TOPK, 1.0), (THR, 0.5), (THR, 0.95), (THR, 1.0),
                                      (MAXF, 0.5), (MAXF, 1e-3), (MAXF, 1.0)])
def test_sizes_and_modes(N, mode, tau, cuda_device):
    rng = np.random.default_rng(N)
    s = (rng.standard_normal((3, N)) * 2).astype(np.float32)
    for k in sorted({1, max(1, N // 3), N}):
        check_select(s, mode, k, tau)


def test_ties_nan_inf_signed_zero(cuda_device):
    rng = np.random.default_rng(1)
    N = 20000
    s = rng.integers(-3, 4, (4, N)).astype(np.float32)  # heavy ties
    s[0, rng.integers(0, N, 500)] = np.nan
    s[1, rng.integers(0, N, 500)] = -np.inf
    s[2, :] = -0.0
    s[2, rng.integers(0, N, 300)] = 0.0
    s[3, rng.integers(0, N, 50)] = np.inf
    for k in (1, 7, 1000, N):
        check_select(s, TOPK, k)
    for tau in (0.3, 0.9, 1.0):
        check_select(s, THR, N, tau)
        check_select(s, THR, 100, tau)
    allnan = np.full((1, 5000), np.nan, np.float32)
    check_select(allnan, THR, 10, 0.5)
    check_select(allnan, TOPK, 10)
    allneg = np.full((1, 5000), -np.inf, np.float32)
    check_select(allneg, THR, 5000, 0.5)
    for alpha in (1.0, 0.2, 1e-30):
        check_select(s, MAXF, N, alpha)
        check_select(s, MAXF, 100, alpha)
    check_select(allnan, MAXF, 10, 0.5)
    check_select(allneg, MAXF, 5000, 0.5)
    check_select(allneg, MAXF, 17, 0.5)


def test_all_equal_closed_form(cuda_device):
    import torch
    s = torch.zeros((2, 1024), dtype=torch.float32, device="cuda")
    idx, cnt = vs.select(s, THR, 1024, 0.9)
    assert cnt.tolist() == [922, 922]
    assert idx[0, :922].tolist() == list(range(922))
    assert (idx[:, 922:] == -1).all()


def test_strided_rows_and_untouched_tail(cuda_device):
    rng = np.random.default_rng(2)
    s = rng.standard_normal((5, 3000)).astype(np.float32)
    check_select(s, TOPK, 64, ld_scores=3072, ld_idx=100)
    check_select(s, THR, 64, 0.7, ld_scores=3001, ld_idx=65)


def test_large_n_without_shared_cache(cuda_device):
    rng = np.random.default_rng(3)
    N = 300000  # more keys per CTA than the shared-memory cache holds
    s = rng.standard_normal((2, N)).astype(np.float32)
    check_select(s, TOPK, 12345)
    check_select(s, THR, N, 0.95)


@pytest.mark.parametrize("name", ["llama_8k", "llama_128k"])
@pytest.mark.parametrize("alpha", [0.3, 0.01])
def test_maxfrac_on_workload_scores(name, alpha, cuda_device):
    # FlashPrefill's max-based rule on the workloads' score vectors, with the
    # workload's budgets as caps (binding for some heads, not for others)
    w = WORKLOADS[name]
    lv, ls = w.all_scores()
    assert check_select(lv, MAXF, w.k_v, alpha) == []
    assert check_select(ls, MAXF, w.k_s, alpha) == []
    assert check_select(lv, MAXF, w.N, alpha) == []


def test_maxfrac_exact_boundary_is_kept(cuda_device):
    import math
    rows = []
    for q in range(1, 200):
        d = -q / 8.0
        if math.log(math.exp(d)) == d:
            rows.append((d, math.exp(d)))
    assert len(rows) > 20
    for d, alpha in rows[:8]:
        s = np.array([[0.0, d, d - 0.125] + [-1e3] * 5000], np.float32)
        check_select(s, MAXF, 5003, alpha)
        check_select(s, MAXF, 1, alpha)


def test_maxfrac_near_uniform_long_rows(cuda_device):
    # the indexer workload's shape: 8 heads x 262144 near-uniform logits
    # (std 0.06); alpha decides between a binding cap and a short list
    rng = np.random.default_rng(7)
    s = (0.06 * rng.standard_normal((8, 262144))).astype(np.float32)
    check_select(s, MAXF, 16384, 0.5)   # ~all entries pass: the cap binds
    check_select(s, MAXF, 16384, 0.9)  # a few hundred entries pass: no search
    big = rng.standard_normal((2, 300000)).astype(np.float32)  # beyond the shared cache
    check_select(big, MAXF, 300000, 0.05)
    check_select(big, MAXF, 1000, 0.05)


@pytest.mark.slow
def test_maximum_row_length(cuda_device):
    # N = 2^20, the largest vs_select accepts
    rng = np.random.default_rng(20)
    N = 1 << 20
    s = rng.standard_normal((2, N)).astype(np.float32)
    check_select(s, TOPK, 1000)
    check_select(s, THR, N, 0.5)
    check_select(s, MAXF, 5000, 0.02)


@pytest.mark.parametrize("H,N", [(32, 131072), (8, 262144), (3, 5000)])
def test_threshold_repeatable_bit_for_bit(H, N, cuda_device):
    # the fp64 mass sums have a fixed order (per-warp histograms, warp-order
    # and rank-order merges): repeated calls of one shape give identical
    # selections; each of the three shapes below runs on its own cluster size
    # (4, 16 and 2 CTAs), and the order differs from one size to another
    import torch
    rng = np.random.default_rng(N + H)
    s = torch.from_numpy((rng.standard_normal((H, N)) * 3.0).astype(np.float32)).cuda()
    k = N  # no cap: the mass sums alone decide
    ws = vs.workspace(vs.vs_select_workspace_size(H, N))
    outs = []
    for _ in range(3):
        idx = torch.empty((H, k), dtype=torch.int32, device="cuda")
        cnt = torch.empty(H, dtype=torch.int32, device="cuda")
        vs.vs_select(s, vs.VS_SELECT_THRESHOLD, k, 0.9, idx, cnt, ws)
        outs.append((idx.cpu().numpy(), cnt.cpu().numpy()))
    rc, flags = vs.vs_read_device_status(ws)
    assert rc == vs.VS_OK and flags == 0
    for o in outs[1:]:
        assert np.array_equal(o[0], outs[0][0]) and np.array_equal(o[1], outs[0][1])

"""vs_select on the GPU vs the oracle: bit-exact index sets and counts on the
same fp32 scores (ties to the smaller index; threshold decisions within 1e-9
of the boundary are reported as tie zones)."""
import numpy as np
import pytest

import sparse_attention_long_head_b200 as vs
from vs_testutil import check_select
from vs_workloads import WORKLOADS

pytestmark = pytest.mark.gpu

TOPK, THR = vs.VS_SELECT_TOPK, vs.VS_SELECT_THRESHOLD


@pytest.mark.parametrize("name", ["tiny_1k", "llama_8k", "llama_32k", "llama_128k", "llama_128k_S"])
def test_workload_scores(name, cuda_device):
    w = WORKLOADS[name]
    lv, ls = w.all_scores()
    mode = TOPK if w.select_mode == "topk" else THR
    ties = check_select(lv, mode, w.k_v, w.tau_v)
    ties += check_select(ls, mode, w.k_s, w.tau_s)
    assert ties == [], f"tie zones at heads {ties}"


@pytest.mark.parametrize("N", [1, 2, 100, 4095, 4096, 4097, 33000, 131071])
@pytest.mark.parametrize("mode,tau", [(TOPK, 1.0), (THR, 0.5), (THR, 0.95), (THR, 1.0)])
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

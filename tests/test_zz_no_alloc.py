"""The allocation-free entry point vs_sparse_attn_fwd_static_scratch, called
through the C ABI, against the workspace-based vs_sparse_attn_fwd.

It serves callers that cannot allocate device memory (plain-C hosts without a
memory manager, plug-ins inside engines that own the whole device pool).  Calls in a
row with different index sets check that the shared static scratch carries
nothing over from the previous call: the same index sets give the same bits
before and after a call with other sets.  Collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

import sparse_attention_long_head_b200 as vs
from vs_testutil import BF16_MAX_ABS, BF16_MEAN_ABS, bf16_to_dev
from vs_workloads import WORKLOADS

pytestmark = pytest.mark.gpu


def _c(t):
    return ctypes.c_void_p(t.data_ptr())


def _static_call(Q, K, V, vi, vc, si, sc, O, lse):
    L = vs.lib()
    N, Hq, d = Q.shape
    return L.vs_sparse_attn_fwd_static_scratch(
        _c(Q), _c(K), _c(V), vs.VS_BF16, N, Hq, K.shape[1], d, Q.stride(0), K.stride(0), 0.0,
        vi.shape[0], _c(vi), vi.stride(0), _c(vc), _c(si), si.stride(0), _c(sc), _c(O), _c(lse),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_static_scratch_matches_workspace_entry_point(cuda_device):
    w = WORKLOADS["llama_8k"]  # 32 index sets at N = 8192: plan fits in 16 MiB
    assert vs.vs_attn_workspace_size(w.N, w.Hq, w.H_sel, w.d) <= 16 << 20
    Qb, Kb, Vb = w.qkv()
    Q, K, V = bf16_to_dev(Qb), bf16_to_dev(Kb), bf16_to_dev(Vb)
    lv, ls = w.all_scores()
    sets = []
    for shift in (0, 1):  # two different index-set pairs, one per call
        sv = torch.from_numpy(np.roll(lv, shift, axis=1)).cuda()
        ss = torch.from_numpy(np.roll(ls, 37 * shift, axis=1)).cuda()
        vi, vc = vs.select(sv, vs.VS_SELECT_TOPK, w.k_v)
        si, sc = vs.select(ss, vs.VS_SELECT_TOPK, w.k_s)
        sets.append((vi, vc, si, sc))
    outs = []
    for vi, vc, si, sc in (sets[1], sets[0], sets[1]):  # three calls in a row
        O = torch.empty_like(Q)
        lse = torch.empty((w.Hq, w.N), dtype=torch.float32, device="cuda")
        assert _static_call(Q, K, V, vi, vc, si, sc, O, lse) == vs.VS_OK
        Oref, lref = vs.sparse_attention(Q, K, V, vi, vc, si, sc)
        torch.cuda.synchronize()
        err = (O.float() - Oref.float()).abs()
        assert err.max().item() <= BF16_MAX_ABS and err.mean().item() <= BF16_MEAN_ABS
        assert torch.allclose(lse, lref, atol=1e-3, rtol=0)
        outs.append((O, lse))
    # the second index-set pair gives the same bits whether the scratch was
    # last used by nothing or by the first pair: no state carries over
    assert torch.equal(outs[0][0], outs[2][0]) and torch.equal(outs[0][1], outs[2][1])


def test_static_scratch_rejects_oversized_plans(cuda_device):
    N, Hq = 131072, 32  # needs ~35 MB of plan data
    assert vs.vs_attn_workspace_size(N, Hq, Hq, 128) > 16 << 20
    L = vs.lib()
    nul = ctypes.c_void_p(0x1000)
    rc = L.vs_sparse_attn_fwd_static_scratch(nul, nul, nul, vs.VS_BF16, N, Hq, 8, 128, Hq * 128,
                                             8 * 128, 0.0, Hq, nul, 8192, nul, nul, 8192, nul,
                                             nul, None, None)
    assert rc == vs.VS_ERR_UNSUPPORTED

"""Device-side failure reporting without faulting the GPU: a bounded wait on
an mbarrier that nothing arrives at gives up and reports a timeout through
the workspace status word; the context stays usable afterwards."""
import time

import pytest
import torch

import sparse_attention_long_head_b200 as vs

pytestmark = pytest.mark.gpu


def test_wait_timeout_reported_and_context_usable(cuda_device):
    ws = vs.workspace(256)
    t0 = time.time()
    vs.vs_selftest_wait_timeout(ws, 20_000_000)  # 20 ms
    rc, flags = vs.vs_read_device_status(ws)
    assert rc == vs.VS_ERR_DEVICE_TIMEOUT and flags & vs.VS_DEVFLAG_TIMEOUT
    assert time.time() - t0 < 30
    # the context still works: a normal call succeeds and clears the status
    s = torch.randn(2, 1000, device="cuda")
    idx, cnt = vs.select(s, vs.VS_SELECT_TOPK, 10, ws=ws)
    rc, flags = vs.vs_read_device_status(ws)
    assert rc == vs.VS_OK and flags == 0
    assert cnt.tolist() == [10, 10]


def test_host_errors_raise(cuda_device):
    s = torch.randn(2, 100, device="cuda")
    with pytest.raises(vs.VsError) as e:
        vs.select(s, vs.VS_SELECT_TOPK, 101)
    assert e.value.code == vs.VS_ERR_INVALID_ARG
    q = torch.randn(10, 1, 96, device="cuda").bfloat16()
    with pytest.raises(vs.VsError) as e:
        vs.dense_attention(q, q, q)
    assert e.value.code == vs.VS_ERR_UNSUPPORTED

"""vs_attn_aggregate on the GPU vs the oracle: column sums A_v and diagonal
sums A_s of the full causal attention weights (the VSPrefill pages'
distillation target, Technical Summary section 2, Distillation Training).

Tolerance: the weights come from a bf16 MMA with fp32 accumulation, a
hardware exp2 (relative error ~2^-22) and the dense kernel's fp32 LSE, and
are summed in fp32 (A_s with atomics), so each entry is within
2e-4 relative + 2e-5 absolute of the fp64 oracle, and each head's row of A_v
and of A_s sums to N within 1e-4 N."""
import math

import numpy as np
import pytest
import torch

import oracle
import sparse_attention_long_head_b200 as vs
from vs_testutil import bf16_to_dev
from vs_workloads import WORKLOADS, gen_qkv

pytestmark = pytest.mark.gpu

RTOL, ATOL = 2e-4, 2e-5


def _gpu_aggregate(Qb, Kb, Vb):
    Q, K, V = bf16_to_dev(Qb), bf16_to_dev(Kb), bf16_to_dev(Vb)
    ws = vs.workspace(256)
    A_v, A_s = vs.aggregate(Q, K, V, ws=ws)
    torch.cuda.synchronize()
    rc, flags = vs.vs_read_device_status(ws)
    assert rc == vs.VS_OK and flags == 0
    return A_v.cpu().numpy().astype(np.float64), A_s.cpu().numpy().astype(np.float64)


def _check(got, want, what):
    err = np.abs(got - want)
    bound = RTOL * np.abs(want) + ATOL
    bad = np.argwhere(err > bound)
    assert bad.size == 0, f"{what}: {len(bad)} entries off, worst {err.max():.3g} at {bad[:3]}"


@pytest.mark.parametrize("N,d,Hq,Hkv", [(1, 128, 1, 1), (100, 128, 2, 1), (128, 64, 1, 1),
                                        (129, 128, 4, 2), (1000, 64, 2, 2), (2049, 128, 4, 1)])
def test_small_cases_against_oracle(N, d, Hq, Hkv, cuda_device):
    Qb, Kb, Vb = gen_qkv(N + d, N, Hq, Hkv, d, 10000.0)
    A_v, A_s = _gpu_aggregate(Qb, Kb, Vb)
    R_v, R_s = oracle.aggregate(Qb, Kb)
    _check(A_v, R_v, "A_v")
    _check(A_s, R_s, "A_s")
    assert np.allclose(A_v.sum(1), N, rtol=1e-4) and np.allclose(A_s.sum(1), N, rtol=1e-4)


def test_uniform_attention_closed_form(cuda_device):
    # q = 0: every causal weight is 1/(i+1), A_v[j] = A_s[j] = H_N - H_j
    N, d = 3000, 128
    rng = np.random.default_rng(4)
    Qb = np.zeros((N, 2, d), np.uint16)
    Kb = (rng.integers(0x3c00, 0x3f80, (N, 1, d))).astype(np.uint16)
    Vb = Kb.copy()
    A_v, A_s = _gpu_aggregate(Qb, Kb, Vb)
    H = np.concatenate([[0.0], np.cumsum(1.0 / np.arange(1, N + 1))])
    want = H[N] - H[np.arange(N)]
    for h in range(2):
        _check(A_v[h], want, "A_v uniform")
        _check(A_s[h], want, "A_s uniform")


@pytest.mark.slow
@pytest.mark.parametrize("name", ["llama_32k", "llama_128k"])
def test_full_size_tail_and_row_sums(name, cuda_device):
    # exact tail: A_v[j] and A_s[o] for j, o >= N - R involve rows i >= N - R only
    w = WORKLOADS[name]
    Qb, Kb, Vb = w.qkv()
    A_v, A_s = _gpu_aggregate(Qb, Kb, Vb)
    N = w.N
    assert np.allclose(A_v.sum(1), N, rtol=1e-4) and np.allclose(A_s.sum(1), N, rtol=1e-4)
    assert (A_v >= 0).all() and (A_s >= 0).all()
    R = 128
    heads = [0, 13, 31]
    R_v, R_s = oracle.aggregate(Qb, Kb, heads=heads, rows=(N - R, N))
    for x, h in enumerate(heads):
        _check(A_v[h, N - R:], R_v[x, N - R:], f"{name} A_v tail head {h}")
        _check(A_s[h, N - R:], R_s[x, N - R:], f"{name} A_s tail head {h}")


@pytest.mark.parametrize("lengths,d,Hq,Hkv", [((300, 1, 1000, 129, 2049), 128, 4, 2),
                                              ((700, 256, 1500), 64, 2, 1)])
def test_batched_sequences_against_oracle(lengths, d, Hq, Hkv, cuda_device):
    # sequences packed along the token axis: each sequence's sums against the
    # oracle on that sequence alone, and A_v equal bit for bit to the
    # single-sequence call (A_v has no atomics)
    parts = [gen_qkv(7 * n + b, n, Hq, Hkv, d, 10000.0) for b, n in enumerate(lengths)]
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    Qc, Kc, Vc = (np.concatenate([p[t] for p in parts]) for t in range(3))
    Q, K, V = bf16_to_dev(Qc), bf16_to_dev(Kc), bf16_to_dev(Vc)
    ws = vs.workspace(256)
    A_v, A_s = vs.aggregate_varlen(Q, K, V, torch.from_numpy(cu).cuda(), max(lengths), ws=ws)
    torch.cuda.synchronize()
    rc, flags = vs.vs_read_device_status(ws)
    assert rc == vs.VS_OK and flags == 0
    Av = A_v.cpu().numpy().astype(np.float64)
    As = A_s.cpu().numpy().astype(np.float64)
    for b, (Qb, Kb, Vb) in enumerate(parts):
        t0, t1 = int(cu[b]), int(cu[b + 1])
        n = t1 - t0
        R_v, R_s = oracle.aggregate(Qb, Kb)
        _check(Av[:, t0:t1], R_v, f"seq {b} A_v")
        _check(As[:, t0:t1], R_s, f"seq {b} A_s")
        assert np.allclose(Av[:, t0:t1].sum(1), n, rtol=1e-4)
        assert np.allclose(As[:, t0:t1].sum(1), n, rtol=1e-4)
        S_v, _ = _gpu_aggregate(Qb, Kb, Vb)
        assert np.array_equal(S_v, Av[:, t0:t1]), b

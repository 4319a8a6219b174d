"""vs_index_scores on the GPU vs the fp64 oracle: max-abs <= 1e-5 (logits of
std ~0.06 at the 0.02-std weights).  bf16 inputs with d in {64, 128}, hidden
in {128, 256} and 16-byte aligned rows take the tensor-core kernel (W1 split
into two bf16 parts, fp32 accumulation); other layouts take the fp32
CUDA-core kernels."""
import numpy as np
import pytest
import torch

import oracle
import sparse_attention_long_head_b200 as vs
from vs_testutil import bf16_to_dev
from vs_workloads import WORKLOADS, gen_qkv, gen_qkv_f32, small_variant

pytestmark = pytest.mark.gpu

TOL = 1e-5


def _run(K, V, W1, W2):
    N, Hkv, _ = K.shape
    lv = torch.empty((Hkv, N), dtype=torch.float32, device="cuda")
    ls = torch.empty_like(lv)
    vs.vs_index_scores(K, V, torch.from_numpy(W1).cuda(), torch.from_numpy(W2).cuda(), lv, ls)
    return lv.cpu().numpy().astype(np.float64), ls.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("N,Hkv,d,hidden", [(1000, 8, 128, 256), (333, 2, 64, 256),
                                            (257, 3, 128, 300), (64, 1, 128, 1),
                                            (1, 1, 64, 128), (129, 4, 128, 128),
                                            (5000, 2, 64, 128)])
def test_matches_oracle(N, Hkv, d, hidden, cuda_device):
    _, Kb, Vb = gen_qkv(N, N, Hkv, Hkv, d, 500000.0)
    rng = np.random.default_rng(hidden)
    W1 = (0.02 * rng.standard_normal((hidden, 2 * d))).astype(np.float32)
    W2 = (0.02 * rng.standard_normal((2, hidden))).astype(np.float32)
    lv, ls = _run(bf16_to_dev(Kb), bf16_to_dev(Vb), W1, W2)
    rv, rs = oracle.index_scores(Kb, Vb, W1, W2)
    assert np.abs(lv - rv).max() <= TOL and np.abs(ls - rs).max() <= TOL


def test_fp32_inputs(cuda_device):
    N, Hkv, d = 500, 2, 128
    _, Kf, Vf = gen_qkv_f32(3, N, Hkv, Hkv, d, 500000.0)
    rng = np.random.default_rng(4)
    W1 = (0.02 * rng.standard_normal((256, 2 * d))).astype(np.float32)
    W2 = (0.02 * rng.standard_normal((2, 256))).astype(np.float32)
    lv, ls = _run(torch.from_numpy(Kf).cuda(), torch.from_numpy(Vf).cuda(), W1, W2)
    rv, rs = oracle.index_scores(Kf, Vf, W1, W2)
    assert np.abs(lv - rv).max() <= TOL and np.abs(ls - rs).max() <= TOL


def test_indexer_workload_then_select(cuda_device):
    # the 256K indexer workload's generators at N=8192: logits -> select bit-exact
    w = small_variant(WORKLOADS["llama_256k_indexer"], 8192, 32, 8)
    _, Kb, Vb = w.qkv()
    W1, W2 = w.indexer_weights()
    lv, ls = _run(bf16_to_dev(Kb), bf16_to_dev(Vb), W1, W2)
    rv, rs = oracle.index_scores(Kb, Vb, W1, W2)
    assert np.abs(lv - rv).max() <= TOL and np.abs(ls - rs).max() <= TOL
    from vs_testutil import check_select
    ties = check_select(lv.astype(np.float32), vs.VS_SELECT_THRESHOLD, w.k_v, w.tau_v)
    ties += check_select(ls.astype(np.float32), vs.VS_SELECT_THRESHOLD, w.k_s, w.tau_s)
    assert ties == []


@pytest.mark.parametrize("d,pad", [(40, 0), (128, 3)])
def test_general_layout_path(d, pad, cuda_device):
    # d not a multiple of 16, or a token stride off the 16-byte grid: the
    # kernel for arbitrary strides
    N, Hkv, hidden = 300, 2, 256
    _, Kb, Vb = gen_qkv(d + pad, N, Hkv, Hkv, d, 500000.0)
    rng = np.random.default_rng(d)
    W1 = (0.02 * rng.standard_normal((hidden, 2 * d))).astype(np.float32)
    W2 = (0.02 * rng.standard_normal((2, hidden))).astype(np.float32)

    def padded(bits):
        buf = torch.zeros((N, Hkv * d + pad), dtype=torch.int16)
        buf[:, : Hkv * d] = torch.from_numpy(bits.reshape(N, Hkv * d).view(np.int16))
        return buf.cuda().view(torch.bfloat16)[:, : Hkv * d].view(N, Hkv, d) if pad == 0 else \
            buf.cuda().view(torch.bfloat16).as_strided((N, Hkv, d), (Hkv * d + pad, d, 1))

    lv, ls = _run(padded(Kb), padded(Vb), W1, W2)
    rv, rs = oracle.index_scores(Kb, Vb, W1, W2)
    assert np.abs(lv - rv).max() <= TOL and np.abs(ls - rs).max() <= TOL


@pytest.mark.parametrize("d,hidden", [(128, 256), (64, 128)])
def test_tensor_core_path_padded_rows(d, hidden, cuda_device):
    # token stride Hkv*d + 8 bf16 (still on the 16-byte grid): the tensor-core
    # kernel must follow the stride, not assume packed rows
    N, Hkv, pad = 700, 3, 8
    _, Kb, Vb = gen_qkv(d + hidden, N, Hkv, Hkv, d, 500000.0)
    rng = np.random.default_rng(d + hidden)
    W1 = (0.02 * rng.standard_normal((hidden, 2 * d))).astype(np.float32)
    W2 = (0.02 * rng.standard_normal((2, hidden))).astype(np.float32)

    def padded(bits):
        buf = torch.zeros((N, Hkv * d + pad), dtype=torch.int16)
        buf[:, : Hkv * d] = torch.from_numpy(bits.reshape(N, Hkv * d).view(np.int16))
        return buf.cuda().view(torch.bfloat16).as_strided((N, Hkv, d), (Hkv * d + pad, d, 1))

    lv, ls = _run(padded(Kb), padded(Vb), W1, W2)
    rv, rs = oracle.index_scores(Kb, Vb, W1, W2)
    assert np.abs(lv - rv).max() <= TOL and np.abs(ls - rs).max() <= TOL


def test_deterministic_across_runs(cuda_device):
    # two hidden slices add into each logit: with exactly two addends onto
    # zero the result does not depend on their order
    N, Hkv, d, hidden = 4096, 8, 128, 256
    _, Kb, Vb = gen_qkv(11, N, Hkv, Hkv, d, 500000.0)
    rng = np.random.default_rng(12)
    W1 = (0.02 * rng.standard_normal((hidden, 2 * d))).astype(np.float32)
    W2 = (0.02 * rng.standard_normal((2, hidden))).astype(np.float32)
    K, V = bf16_to_dev(Kb), bf16_to_dev(Vb)
    first = _run(K, V, W1, W2)
    for _ in range(3):
        again = _run(K, V, W1, W2)
        assert np.array_equal(first[0], again[0]) and np.array_equal(first[1], again[1])


@pytest.mark.parametrize("d,hidden", [(128, 256), (64, 128)])
def test_tensor_core_single_weight_probes(d, hidden, cuda_device):
    # one nonzero bf16-representable weight: the split has no low part, the
    # MMA sums a single exact product, so the logits are exact -- any slip in
    # the swizzled operand layout or the hidden-slice split moves the weight
    # to another feature or unit
    N, Hkv = 300, 2
    _, Kb, Vb = gen_qkv(5, N, Hkv, Hkv, d, 500000.0)
    k = (Kb.astype(np.uint32) << 16).view(np.float32)
    v = (Vb.astype(np.uint32) << 16).view(np.float32)
    K, V = bf16_to_dev(Kb), bf16_to_dev(Vb)
    for (u, c, r, w1, w2) in [(0, 0, 0, 1.0, 1.0), (hidden - 1, 2 * d - 1, 1, -2.0, 0.5),
                              (hidden // 2 + 3, d, 0, 1.5, -1.0), (77 % hidden, d - 1, 1, 1.0, 3.0),
                              (hidden // 2 - 1, 37, 0, 0.25, 2.0)]:
        W1 = np.zeros((hidden, 2 * d), np.float32)
        W2 = np.zeros((2, hidden), np.float32)
        W1[u, c] = w1
        W2[r, u] = w2
        lv, ls = _run(K, V, W1, W2)
        x = k[..., c] if c < d else v[..., c - d]  # [N, Hkv]
        want = (np.float32(w2) * np.maximum(np.float32(w1) * x, np.float32(0))).T.astype(np.float64)
        got, other = (lv, ls) if r == 0 else (ls, lv)
        np.testing.assert_array_equal(got, want)
        assert np.all(other == 0.0)

"""FlashPrefill-style block pattern discovery and block-sparse attention on
the GPU vs the oracle (FlashPrefill summary page, sections 2A, 2B and 3).

Selection: bit-exact kept-block masks on the same inputs (both sides decide
in fp64; a decision within 1e-9 of its threshold would be a tie zone, and the
seeds give none).  Attention: bf16 tolerances as for the other kernels, on
the oracle's own masks."""
import numpy as np
import pytest
import torch

import oracle
import sparse_attention_long_head_b200 as vs
from vs_testutil import bf16_to_dev, compare_rows, dev_to_f64
from vs_workloads import gen_qkv, plant_block_structure

pytestmark = pytest.mark.gpu


def _gpu_mask(Q, K, alpha):
    N, Hq, d = Q.shape
    T = (N + 127) // 128
    mask = torch.zeros((Hq, T, (T + 31) // 32), dtype=torch.int32, device="cuda")
    ws = vs.workspace(vs.vs_block_select_workspace_size(N, K.shape[1], d))
    vs.vs_block_select(Q, K, alpha, mask, ws)
    rc, flags = vs.vs_read_device_status(ws)
    assert rc == vs.VS_OK and flags == 0
    return mask.cpu().numpy().view(np.uint32)


@pytest.mark.parametrize("N,d,Hq,Hkv,alpha", [(128, 128, 2, 1, 0.5), (1000, 128, 4, 2, 0.2),
                                              (3000, 64, 4, 1, 0.05), (4097, 128, 2, 2, 0.6),
                                              (2500, 128, 8, 2, 1.0)])
def test_block_select_against_oracle(N, d, Hq, Hkv, alpha, cuda_device):
    Qb, Kb, _ = gen_qkv(N + 3, N, Hq, Hkv, d, 10000.0)
    Qb, Kb = plant_block_structure(Qb, Kb, seed=N)
    ref, margin = oracle.block_select(Qb, Kb, alpha)
    assert (margin > 1e-9).all(), margin
    got = _gpu_mask(bf16_to_dev(Qb), bf16_to_dev(Kb), alpha)
    assert np.array_equal(got, ref)


@pytest.mark.slow
def test_block_select_long_rows_recompute_path(cuda_device):
    # T > 1024 blocks: the dot products are recomputed instead of kept
    N = 140000
    Qb, Kb, _ = gen_qkv(21, N, 1, 1, 64, 500000.0)
    Qb, Kb = plant_block_structure(Qb, Kb, seed=21)
    ref, margin = oracle.block_select(Qb, Kb, 0.3)
    assert (margin > 1e-9).all(), margin
    got = _gpu_mask(bf16_to_dev(Qb), bf16_to_dev(Kb), 0.3)
    assert np.array_equal(got, ref)


def _gpu_block_attn(Qb, Kb, Vb, mask):
    Q, K, V = (bf16_to_dev(x) for x in (Qb, Kb, Vb))
    N, Hq, d = Q.shape
    O = torch.empty_like(Q)
    lse = torch.empty((Hq, N), dtype=torch.float32, device="cuda")
    ws = vs.workspace(vs.vs_block_attn_workspace_size(N, Hq))
    vs.vs_block_sparse_attn_fwd(Q, K, V, torch.from_numpy(mask.view(np.int32)).cuda(), O, lse, ws)
    rc, flags = vs.vs_read_device_status(ws)
    assert rc == vs.VS_OK and flags == 0
    return O, lse


@pytest.mark.parametrize("N,d,Hq,Hkv,alpha", [(1000, 128, 4, 2, 0.2), (129, 64, 2, 1, 0.5),
                                              (3000, 128, 2, 1, 0.05), (2049, 64, 4, 4, 0.9)])
def test_block_attention_against_oracle(N, d, Hq, Hkv, alpha, cuda_device):
    Qb, Kb, Vb = gen_qkv(N + 7, N, Hq, Hkv, d, 10000.0)
    Qb, Kb = plant_block_structure(Qb, Kb, seed=N + 1)
    mask, _ = oracle.block_select(Qb, Kb, alpha)
    O, lse = _gpu_block_attn(Qb, Kb, Vb, mask)
    Od = dev_to_f64(O)
    lsed = lse.cpu().numpy().astype(np.float64)
    rows = np.arange(N)
    for h in range(Hq):
        Or, lr = oracle.attn_block_rows(Qb, Kb, Vb, h, rows, mask)
        compare_rows(Od[:, h], Or, lsed[h], lr, what=f"block N={N} head {h}")


def test_all_blocks_kept_equals_dense_kernel_bitwise(cuda_device):
    N, Hq = 1500, 4
    Qb, Kb, Vb = gen_qkv(11, N, Hq, 2, 128, 10000.0)
    T = (N + 127) // 128
    W = (T + 31) // 32
    mask = np.zeros((Hq, T, W), np.uint32)
    for I in range(T):
        for J in range(I + 1):
            mask[:, I, J >> 5] |= np.uint32(1 << (J & 31))
    O, lse = _gpu_block_attn(Qb, Kb, Vb, mask)
    Od, lsed = vs.dense_attention(*(bf16_to_dev(x) for x in (Qb, Kb, Vb)))
    assert torch.equal(O, Od) and torch.equal(lse, lsed)


def test_unkept_rows_and_ignored_upper_bits(cuda_device):
    # row I keeps nothing (not even its diagonal) -> O = 0, LSE = -inf there;
    # bits above the diagonal are ignored
    N, Hq = 700, 2
    Qb, Kb, Vb = gen_qkv(12, N, Hq, 1, 128, 10000.0)
    T = (N + 127) // 128
    mask = np.full((Hq, T, 1), 0xFFFFFFFF, np.uint32)
    mask[0, 2, 0] = 0
    O, lse = _gpu_block_attn(Qb, Kb, Vb, mask)
    clean = mask.copy()
    for I in range(T):
        clean[:, I, 0] &= np.uint32((1 << (I + 1)) - 1)
    Od = dev_to_f64(O)
    lsed = lse.cpu().numpy().astype(np.float64)
    for h in range(Hq):
        Or, lr = oracle.attn_block_rows(Qb, Kb, Vb, h, np.arange(N), clean)
        compare_rows(Od[:, h], Or, lsed[h], lr, what=f"head {h}")
    assert np.all(Od[256:384, 0] == 0) and np.all(np.isneginf(lsed[0, 256:384]))


def test_block_prefill_pipeline(cuda_device):
    N, Hq, Hkv, d, alpha = 4000, 4, 2, 128, 0.1
    Qb, Kb, Vb = gen_qkv(13, N, Hq, Hkv, d, 500000.0)
    Qb, Kb = plant_block_structure(Qb, Kb, seed=3)
    O, lse, mask = vs.block_prefill(*(bf16_to_dev(x) for x in (Qb, Kb, Vb)), alpha)
    ref, margin = oracle.block_select(Qb, Kb, alpha)
    assert (margin > 1e-9).all()
    assert np.array_equal(mask.cpu().numpy().view(np.uint32), ref)
    Od = dev_to_f64(O)
    lsed = lse.cpu().numpy().astype(np.float64)
    rows = np.unique(np.concatenate([np.arange(0, 300), np.arange(N - 300, N),
                                     np.random.default_rng(0).integers(0, N, 300)]))
    for h in range(Hq):
        Or, lr = oracle.attn_block_rows(Qb, Kb, Vb, h, rows, ref)
        compare_rows(Od[rows, h], Or, lsed[h, rows], lr, what=f"pipeline head {h}")


@pytest.mark.slow
def test_maximum_length_block_path(cuda_device):
    # N = 2^18, the largest the block calls accept (2048 blocks: the
    # recompute path of the scores)
    from vs_testutil import sample_rows
    N = 1 << 18
    Qb, Kb, Vb = gen_qkv(23, N, 1, 1, 64, 500000.0)
    Qb, Kb = plant_block_structure(Qb, Kb, seed=23)
    ref, margin = oracle.block_select(Qb, Kb, 0.3)
    assert (margin > 1e-9).all(), margin
    assert np.array_equal(_gpu_mask(bf16_to_dev(Qb), bf16_to_dev(Kb), 0.3), ref)
    O, lse = _gpu_block_attn(Qb, Kb, Vb, ref)
    rows = sample_rows(N, seed=2, n_random=200)
    Or, lr = oracle.attn_block_rows(Qb, Kb, Vb, 0, rows, ref)
    compare_rows(dev_to_f64(O)[rows, 0], Or, lse.cpu().numpy().astype(np.float64)[0, rows], lr,
                 what="block N = 2^18")


@pytest.mark.slow
def test_flashprefill_32k_workload_full_size(cuda_device):
    # the bench's configuration: 32 query heads over 8 KV heads (four query
    # heads share a CTA), N = 32768; bit-exact masks for every head, and the
    # block-sparse rows of two heads sampled
    from vs_testutil import sample_rows
    from vs_workloads import BLOCK_WORKLOADS
    w = BLOCK_WORKLOADS["flashprefill_32k"]
    Qb, Kb, Vb = w.qkv()
    ref, margin = oracle.block_select(Qb, Kb, w.alpha)
    assert (margin > 1e-9).all(), margin
    got = _gpu_mask(bf16_to_dev(Qb), bf16_to_dev(Kb), w.alpha)
    assert np.array_equal(got, ref)
    O, lse = _gpu_block_attn(Qb, Kb, Vb, ref)
    rows = sample_rows(w.N, seed=3, n_random=150)
    for h in (0, 29):
        Or, lr = oracle.attn_block_rows(Qb, Kb, Vb, h, rows, ref)
        compare_rows(dev_to_f64(O)[rows, h], Or, lse[h].cpu().numpy().astype(np.float64)[rows], lr,
                     what=f"flashprefill_32k head {h}")


@pytest.mark.slow
def test_flashprefill_128k_workload_full_size(cuda_device):
    # the bench's block workload itself: 32 query heads over 8 KV heads,
    # N = 131072 (1024 query blocks); bit-exact kept-block masks for every
    # head, then the block-sparse rows of every head sampled against the
    # oracle over the oracle's masks
    from vs_testutil import sample_rows
    from vs_workloads import BLOCK_WORKLOADS
    w = BLOCK_WORKLOADS["flashprefill_128k"]
    Qb, Kb, Vb = w.qkv()
    ref, margin = oracle.block_select(Qb, Kb, w.alpha)
    assert (margin > 1e-9).all(), margin
    got = _gpu_mask(bf16_to_dev(Qb), bf16_to_dev(Kb), w.alpha)
    assert np.array_equal(got, ref)
    O, lse = _gpu_block_attn(Qb, Kb, Vb, ref)
    Od = dev_to_f64(O)
    lsed = lse.cpu().numpy().astype(np.float64)
    for h in range(w.Hq):
        rows = sample_rows(w.N, seed=40 + h, n_random=512)
        Or, lr = oracle.attn_block_rows(Qb, Kb, Vb, h, rows, ref)
        compare_rows(Od[rows, h], Or, lsed[h, rows], lr, what=f"flashprefill_128k head {h}")


@pytest.mark.parametrize("N,d,Hq,Hkv,alpha", [(3000, 128, 8, 2, 0.3), (2100, 64, 2, 2, 0.15)])
def test_block_select_fp32_inputs(N, d, Hq, Hkv, alpha, cuda_device):
    # fp32 Q/K (off the bf16 grid) through the same selection; the oracle
    # reads the same fp32 values
    from vs_workloads import bf16_bits_to_f32
    Qb, Kb, _ = gen_qkv(N + 11, N, Hq, Hkv, d, 10000.0)
    Qb, Kb = plant_block_structure(Qb, Kb, seed=N + 11)
    rng = np.random.default_rng(N)
    Qf = (bf16_bits_to_f32(Qb) * (1 + 1e-3 * rng.standard_normal(Qb.shape))).astype(np.float32)
    Kf = (bf16_bits_to_f32(Kb) * (1 + 1e-3 * rng.standard_normal(Kb.shape))).astype(np.float32)
    ref, margin = oracle.block_select(Qf, Kf, alpha)
    assert (margin > 1e-9).all(), margin
    got = _gpu_mask(torch.from_numpy(Qf).cuda(), torch.from_numpy(Kf).cuda(), alpha)
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("N,d,Hq,Hkv,dens,seed", [(2049, 128, 2, 1, 0.15, 1), (1500, 64, 2, 2, 0.5, 2),
                                                  (3000, 128, 4, 2, 0.05, 3)])
def test_random_masks_per_sub_tile(N, d, Hq, Hkv, dens, seed, cuda_device):
    # each query block keeps its own random set (the two query blocks of a
    # pair differ; some drop their diagonal; one keeps nothing)
    Qb, Kb, Vb = gen_qkv(seed + 30, N, Hq, Hkv, d, 10000.0)
    T = (N + 127) // 128
    W = (T + 31) // 32
    rng = np.random.default_rng(seed)
    bits = rng.random((Hq, T, T)) < dens
    bits |= np.eye(T, dtype=bool)[None] & (rng.random((Hq, T, 1)) < 0.8)
    bits[0, T // 2, :] = False
    mask = np.zeros((Hq, T, W), np.uint32)
    for J in range(T):
        mask[:, :, J // 32] |= (bits[:, :, J].astype(np.uint32) << np.uint32(J % 32))
    O, lse = _gpu_block_attn(Qb, Kb, Vb, mask)
    Od = dev_to_f64(O)
    lsed = lse.cpu().numpy().astype(np.float64)
    for h in range(Hq):
        Or, lr = oracle.attn_block_rows(Qb, Kb, Vb, h, np.arange(N), mask)
        compare_rows(Od[:, h], Or, lsed[h], lr, what=f"head {h}")
    r0 = 128 * (T // 2)
    assert np.all(Od[r0:r0 + 128, 0] == 0) and np.all(np.isneginf(lsed[0, r0:r0 + 128]))

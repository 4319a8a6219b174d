"""The seeded input generators: determinism, bf16 rounding and RoPE."""
import numpy as np

from vs_workloads import (WORKLOADS, bf16_bits_to_f32, f64_to_bf16_bits, gen_qkv,
                          gen_tensor_bf16, small_variant)


def test_bf16_round_to_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 1.0 + 2 ** -8 + 2 ** -30, 3.0e-3])
    got = bf16_bits_to_f32(f64_to_bf16_bits(x)).astype(np.float64)
    # 1+2^-8 is halfway between 1 and 1+2^-7 -> even (1.0); 1+3*2^-8 -> 1+2^-6
    assert got[0] == 1.0 and got[1] == 1.0 and got[2] == 1.0 + 2 ** -6
    assert got[3] == -2.5 and got[4] == 1.0 + 2 ** -7
    assert abs(got[5] - 3.0e-3) <= 3.0e-3 * 2 ** -8


def test_bf16_matches_torch_for_fp32_exact_values():
    import torch
    rng = np.random.default_rng(0)
    x = rng.standard_normal(10000).astype(np.float32).astype(np.float64)  # exact in fp32
    ours = f64_to_bf16_bits(x)
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy()
    assert np.array_equal(ours, ref.view(np.uint16))


def test_deterministic_and_chunk_independent():
    a = gen_tensor_bf16(5, 1, 9000, 2, 64, 10000.0, threads=1)
    b = gen_tensor_bf16(5, 1, 9000, 2, 64, 10000.0, threads=4)
    assert np.array_equal(a, b)
    c = gen_tensor_bf16(5, 1, 5000, 2, 64, 10000.0)
    assert np.array_equal(a[:4096], c[:4096])


def test_rope_preserves_pair_norms():
    N, d = 100, 64
    Q, _, _ = gen_qkv(1, N, 1, 1, d, 10000.0)
    rng = np.random.default_rng([1, 0, 0])
    x = rng.standard_normal((N, 1, d))
    q = bf16_bits_to_f32(Q).astype(np.float64)
    half = d // 2
    n_raw = x[..., :half] ** 2 + x[..., half:] ** 2
    n_rot = q[..., :half] ** 2 + q[..., half:] ** 2
    np.testing.assert_allclose(n_rot, n_raw, rtol=2e-2, atol=1e-2)
    np.testing.assert_allclose(q[0], x[0], rtol=1e-2, atol=1e-2)  # position 0: no rotation


def test_workload_registry_shapes():
    w = WORKLOADS["llama_128k"]
    assert (w.N, w.Hq, w.Hkv, w.d, w.H_sel) == (131072, 32, 8, 128, 32)
    assert WORKLOADS["llama_256k_indexer"].H_sel == 8
    s = small_variant(w, 4096, 4, 1)
    lv, ls = s.all_scores()
    assert lv.shape == (4, 4096) and lv.dtype == np.float32
    assert np.isfinite(lv).all() and np.isfinite(ls).all()
    lv2, _ = s.all_scores()
    assert np.array_equal(lv, lv2)

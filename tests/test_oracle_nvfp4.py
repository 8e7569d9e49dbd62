"""Pins of the oracle's NVFP4 comparison codec (no GPU).

NVFP4 is named by the llm-compressor page (ai-insight.org/news/11771) and the
llama.cpp quantizer page (bittide.aicompass.dev: "NVFP4 weight and input tensor
scales"); neither prints a bit recipe.  The oracle takes the plainest reading
(E2M1 values, 16-element blocks, E4M3 block scale, fp32 tensor scale
amax / (6 * 448)); these tests pin its pieces against library conversions,
brute force and exact round trips.
"""
import numpy as np
import torch

E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def test_e4m3_decode_matches_torch(oracle_mod):
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)  # skip NaN codes
    ref = torch.tensor(codes).view(torch.float8_e4m3fn).float().numpy()
    np.testing.assert_array_equal(oracle_mod.e4m3_to_f32(codes), ref)


def test_e4m3_encode_matches_torch_in_range(oracle_mod):
    rng = np.random.default_rng(21)
    x = np.concatenate([
        rng.uniform(0, 448, 3000), 2.0 ** rng.uniform(-12, 8.8, 3000),
        oracle_mod.e4m3_to_f32(np.arange(1, 126, dtype=np.uint8)),  # exact codes
    ]).astype(np.float32)
    # midpoints between neighbours exercise ties-to-even
    v = oracle_mod.e4m3_to_f32(np.arange(0, 127, dtype=np.uint8)).astype(np.float64)
    mids = ((v[1:] + v[:-1]) / 2).astype(np.float32)
    x = np.concatenate([x, mids[np.isclose(mids.astype(np.float64), (v[1:] + v[:-1]) / 2, rtol=0, atol=0)]])
    ref = torch.tensor(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(oracle_mod.e4m3_from_f32(x), ref)
    assert oracle_mod.e4m3_from_f32([448.0, 500.0, 1e9])[0] == 0x7E
    assert np.all(oracle_mod.e4m3_from_f32([448.0, 500.0, 1e9]) == 0x7E)  # saturating


def test_e2m1_is_nearest_with_ties_to_even(oracle_mod):
    x = np.concatenate([np.linspace(-8, 8, 4001), (E2M1[1:] + E2M1[:-1]) / 2, -(E2M1[1:] + E2M1[:-1]) / 2])
    got = oracle_mod.e2m1_from_f32(x)
    vals = oracle_mod.e2m1_to_f32(got).astype(np.float64)
    for xi, code, v in zip(x, got, vals):
        a = min(abs(xi), 6.0)
        d = np.abs(E2M1 - a)
        best = np.flatnonzero(d == d.min())
        idx = best[0] if len(best) == 1 else [b for b in best if b % 2 == 0][0]  # tie -> even code
        assert abs(v) == E2M1[idx], (xi, code)
        if E2M1[idx] != 0:
            assert (v < 0) == (xi < 0)
        else:
            assert code == 0  # zero carries no sign


def test_nvfp4_exact_roundtrip_on_representable_weights(oracle_mod):
    rng = np.random.default_rng(22)
    n, k = 5, 64
    g = np.float32(2.0 ** -12)
    # block scales: powers of two (exact in E4M3); the first block holds the amax
    s = 2.0 ** rng.integers(-3, 8, (n, k // 16))
    s[0, 0] = 448.0
    q = E2M1[rng.integers(0, 8, (n, k))] * np.where(rng.random((n, k)) < 0.5, -1, 1)
    q[:, ::16] = 6.0  # every block reaches its maximum magnitude
    W = (q * np.repeat(s, 16, axis=1) * g).astype(np.float32)
    codes, scales, g_out = oracle_mod.nvfp4_quantize(W)
    assert np.float32(g_out) == g
    np.testing.assert_array_equal(oracle_mod.nvfp4_dequantize(codes, scales, g_out, n, k), W.astype(np.float64))


def test_nvfp4_reconstruction_and_gemm(oracle_mod):
    rng = np.random.default_rng(23)
    n, k, m = 40, 256, 3
    W = (rng.standard_normal((n, k)) * 0.02).astype(np.float32)
    codes, scales, g = oracle_mod.nvfp4_quantize(W)
    assert abs(g - np.abs(W).max() / 2688) <= 1e-7 * g
    Wd = oracle_mod.nvfp4_dequantize(codes, scales, g, n, k)
    rel = np.linalg.norm(Wd - W) / np.linalg.norm(W)
    assert 0.07 < rel < 0.12, rel
    X = rng.standard_normal((m, k))
    np.testing.assert_allclose(oracle_mod.nvfp4_gemm(codes, scales, g, n, k, X), X @ Wd.T, rtol=1e-12, atol=1e-14)
    # the global maximum maps to +-6 on a 448 block scale
    r, c = np.unravel_index(np.abs(W).argmax(), W.shape)
    assert abs(Wd[r, c] - W[r, c]) <= 1e-6 * abs(W[r, c])

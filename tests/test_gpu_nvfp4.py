"""GPU parity of the NVFP4 comparison codec against the oracle.

NVFP4 is named by the llm-compressor page (ai-insight.org/news/11771) and the
llama.cpp quantizer page (bittide.aicompass.dev: "NVFP4 weight and input tensor
scales"); the format read here is E2M1 values, 16-element blocks, an E4M3 block
scale and an fp32 tensor scale amax / (6 * 448), no rotation.

Bars:
  * quantise: codes, E4M3 scale bytes and the fp32 tensor scale identical;
  * dequantise: |w_gpu - w64| <= |w64| (2 u32 + u_out) + floor (two fp32
    products, then rounding to the output type);
  * GEMM: relative L2 error <= 1e-3 per output row against the fp64 product
    over the oracle's own reconstruction.
"""
import numpy as np
import pytest
import torch

import oracle
from dequant_gemv_tq4_b200 import inputs

pytestmark = pytest.mark.gpu

REL_L2_TOL = 1e-3
DEV = "cuda:0"
F32, BF16, F16 = torch.float32, torch.bfloat16, torch.float16


def _w(n, k, dtype, seed=0, std=0.02):
    return inputs.gaussian_matrix(seed, n * 7907 + k, n, k, std, dtype)


def _host_f32(t):
    return t.detach().to("cpu").float().numpy()


def _rel_l2(y, ref):
    y = np.atleast_2d(y).astype(np.float64)
    ref = np.atleast_2d(ref)
    return np.linalg.norm(y - ref, axis=1) / np.maximum(np.linalg.norm(ref, axis=1), 1e-300)


def _gpu_quantize(tq, W):
    codes, scales, tensor = tq.nvfp4_quantize(W.to(DEV))
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy(), tensor.cpu().numpy()


def _assert_same_encoding(got, ref):
    c, s, t = got
    c_ref, s_ref, g_ref = ref
    assert np.float32(t[0]).view(np.uint32) == np.float32(g_ref).view(np.uint32)
    np.testing.assert_array_equal(s, s_ref)
    np.testing.assert_array_equal(c, c_ref)


SHAPES = [(1, 32), (3, 64), (17, 96), (16, 128), (33, 160), (5, 4096), (64, 1056), (100, 384)]


@pytest.mark.parametrize("dtype", [F32, BF16, F16])
@pytest.mark.parametrize("n,k", SHAPES)
def test_nvfp4_quantize_bit_exact(cuda_lib, n, k, dtype):
    W = _w(n, k, dtype)
    ref = oracle.nvfp4_quantize(_host_f32(W))
    got = _gpu_quantize(cuda_lib, W)
    _assert_same_encoding(got, ref)
    assert got[2][1] == np.abs(_host_f32(W)).max()  # amax word of the tensor block


def test_nvfp4_quantize_special_values(cuda_lib):
    n, k = 10, 256
    W = _w(n, k, F32, seed=3)
    W[0] = 0.0                          # zero row: scales 0, codes 0
    W[1] = -0.0                         # negative zeros carry no sign
    W[2, :16] = 1e-9                    # block scale below the E4M3 range -> 0
    W[2, 16:32] = 5e-5                  # subnormal E4M3 block scales
    W[2, 32:48] = 1.2e-5                # rounds up to the smallest subnormal
    W[3] = 5.0                          # the tensor amax: every code saturates at 6 * 448 * g
    W[4, ::2] = -5.0
    W[5, :32] = torch.tensor([(-1) ** i * 0.25 * (i % 7) for i in range(32)])  # E2M1 midpoints after scaling
    ref = oracle.nvfp4_quantize(W.numpy().copy())
    _assert_same_encoding(_gpu_quantize(cuda_lib, W), ref)


def test_nvfp4_all_zero_matrix(cuda_lib):
    W = torch.zeros((16, 128), dtype=BF16)
    c, s, t = _gpu_quantize(cuda_lib, W)
    assert t[0] == 0.0 and np.all(c == 0) and np.all(s == 0)
    out = cuda_lib.nvfp4_dequantize(*[torch.tensor(a, device=DEV) for a in (c, s, t)], 16, 128, dtype=F32)
    torch.cuda.synchronize()
    assert torch.count_nonzero(out).item() == 0


def test_nvfp4_quantize_strided(cuda_lib):
    n, k, ld = 12, 256, 264
    base = torch.full((n, ld), 123.0, dtype=F32)   # the padding holds the largest values
    base[:, :k] = _w(n, k, F32, seed=4)
    ref = oracle.nvfp4_quantize(base[:, :k].numpy().copy())
    codes, scales, tensor = cuda_lib.nvfp4_quantize(base.to(DEV)[:, :k])
    torch.cuda.synchronize()
    _assert_same_encoding((codes.cpu().numpy(), scales.cpu().numpy(), tensor.cpu().numpy()), ref)


@pytest.mark.parametrize("out_dtype", [F32, BF16, F16])
@pytest.mark.parametrize("n,k", [(3, 64), (17, 96), (33, 160), (64, 1056)])
def test_nvfp4_dequantize_within_bound(cuda_lib, n, k, out_dtype):
    W = _w(n, k, BF16, seed=5)
    c_ref, s_ref, g = oracle.nvfp4_quantize(_host_f32(W))
    w64 = oracle.nvfp4_dequantize(c_ref, s_ref, g, n, k)
    tensor = torch.tensor([g, 0.0, 0.0, 0.0], dtype=F32, device=DEV)
    out = cuda_lib.nvfp4_dequantize(torch.tensor(c_ref, device=DEV), torch.tensor(s_ref, device=DEV), tensor, n, k,
                                    dtype=out_dtype)
    torch.cuda.synchronize()
    got = out.float().cpu().numpy().astype(np.float64)
    u_out = {F32: 2.0 ** -24, BF16: 2.0 ** -8, F16: 2.0 ** -11}[out_dtype]
    floor = {F32: 2.0 ** -149, BF16: 2.0 ** -133, F16: 2.0 ** -25}[out_dtype]
    bound = np.abs(w64) * (2 * 2.0 ** -24 * (1 + u_out) + u_out) + floor
    err = np.abs(got - w64)
    assert np.all(err <= bound), float((err / bound).max())


GEMM_CASES = [(1, 1, 32), (1, 17, 4096), (1, 1024, 4096), (2, 33, 256), (5, 40, 1024), (8, 16, 8192),
              (16, 100, 384), (16, 300, 1056), (31, 17, 1024), (32, 64, 2048),
              (2, 40, 4096), (3, 100, 2048), (4, 17, 8192)]


@pytest.mark.parametrize("m,n,k", GEMM_CASES)
def test_nvfp4_gemm_rel_l2(cuda_lib, m, n, k):
    W = _w(n, k, BF16, seed=8)
    X = _w(m, k, BF16, seed=9, std=1.0)
    c_ref, s_ref, g = oracle.nvfp4_quantize(_host_f32(W))
    Y_ref = oracle.nvfp4_gemm(c_ref, s_ref, g, n, k, _host_f32(X))
    codes, scales, tensor = cuda_lib.nvfp4_quantize(W.to(DEV))
    Y = cuda_lib.nvfp4_gemm(codes, scales, tensor, n, k, X.to(DEV))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(codes.cpu().numpy(), c_ref)
    assert _rel_l2(Y.cpu().numpy(), Y_ref).max() <= REL_L2_TOL


def test_nvfp4_gemm_rejects_large_m(cuda_lib):
    n, k, m = 32, 128, 33
    codes, scales, tensor = cuda_lib.nvfp4_quantize(_w(n, k, BF16).to(DEV))
    X = torch.zeros((m, k), dtype=BF16, device=DEV)
    Y = torch.zeros((m, n), dtype=F32, device=DEV)
    ws = cuda_lib.workspace(32, n, k)
    st = cuda_lib.tq_nvfp4_gemm(codes.data_ptr(), scales.data_ptr(), tensor.data_ptr(), n, k, X.data_ptr(), 1, m, k,
                                Y.data_ptr(), 0, n, ws.data_ptr(), ws.numel(), torch.cuda.current_stream().cuda_stream)
    assert st == 2  # TQ_ERR_SHAPE


def test_nvfp4_batch_matches_single(cuda_lib):
    m = 3
    shapes = [(256, 1024, "a"), (64, 1024, "a"), (300, 512, "b")]
    Xs = {"a": _w(m, 1024, BF16, seed=40, std=1.0).to(DEV), "b": _w(m, 512, BF16, seed=41, std=1.0).to(DEV)}
    items, singles, refs = [], [], []
    for i, (n, k, name) in enumerate(shapes):
        W = _w(n, k, BF16, seed=50 + i)
        c_ref, s_ref, g = oracle.nvfp4_quantize(_host_f32(W))
        refs.append(oracle.nvfp4_gemm(c_ref, s_ref, g, n, k, _host_f32(Xs[name])))
        codes, scales, tensor = cuda_lib.nvfp4_quantize(W.to(DEV))
        Y = torch.empty((m, n), dtype=F32, device=DEV)
        items.append((codes, scales, tensor, n, k, Xs[name], Y))
        singles.append(cuda_lib.nvfp4_gemm(codes, scales, tensor, n, k, Xs[name]))
    cuda_lib.nvfp4_gemm_batch(items, m=m)
    torch.cuda.synchronize()
    for it, single, ref in zip(items, singles, refs):
        np.testing.assert_allclose(it[6].cpu().numpy(), single.cpu().numpy(), rtol=1e-5, atol=1e-6)
        assert _rel_l2(it[6].cpu().numpy(), ref).max() <= REL_L2_TOL


def _sample_rows(n, count, seed, must):
    rng = np.random.default_rng(seed + n)
    return np.unique(np.concatenate(([0, n - 1, must], rng.choice(n, count, replace=False))))


@pytest.mark.parametrize("m", [1, 16])
def test_nvfp4_llama3_8b_layer_full_size(cuda_lib, m):
    """The Llama-3-8B layer shapes at M = 1 and 16: codes/scales of sampled rows
    bit-exact, products within 1e-3.  The sample includes the row holding the
    tensor's largest |w|, so the oracle derives the same tensor scale."""
    weights, _ = inputs.llama3_8b_layer(device=DEV)
    for name, W in weights.items():
        n, k = W.shape
        X = inputs.gaussian_matrix(1, 200 + m, m, k, 1.0, BF16, DEV)
        codes, scales, tensor = cuda_lib.nvfp4_quantize(W)
        Y = cuda_lib.nvfp4_gemm(codes, scales, tensor, n, k, X)
        torch.cuda.synchronize()
        arg_row = int(W.abs().flatten().argmax().item()) // k
        rows = _sample_rows(n, 12, m, arg_row)
        Wr = _host_f32(W[torch.tensor(rows, device=DEV)])
        c_ref, s_ref, g = oracle.nvfp4_quantize(Wr)
        assert np.float32(tensor[0].item()) == np.float32(g), name
        gc, gs = oracle.row_view(codes.cpu().numpy(), scales.cpu().numpy(), n, k)
        rc, rs = oracle.row_view(c_ref, s_ref, len(rows), k)
        np.testing.assert_array_equal(gc[rows], rc, err_msg=name)
        np.testing.assert_array_equal(gs[rows], rs, err_msg=name)
        Y_ref = oracle.nvfp4_gemm(c_ref, s_ref, g, len(rows), k, _host_f32(X))
        assert _rel_l2(Y.cpu().numpy()[:, rows], Y_ref).max() <= REL_L2_TOL, name

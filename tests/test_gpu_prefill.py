"""GPU parity of the tensor-core prefill product (tq_gemm_prefill, and tq_gemm
for m > 32) against the CPU oracle.

TQ4_1S page ("企业官网建设流程全解析"), section 解码速度：分硬件汇总: the
activation is rotated once, after which every weight contributes
centroid * scale.  The prefill kernel applies this to a whole activation
matrix on tcgen05 tensor cores (fp16 operands, fp32 accumulation).

Bar: relative L2 error <= 1e-3 per output row against the fp64 product over
the oracle's own dequantised weights (the same bar as the skinny product; the
prefill path rounds each weight to fp16(c * d) once more, relative 2^-11).
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
    return inputs.gaussian_matrix(seed, n * 7919 + k, n, k, std, dtype)


def _host_f32(t):
    return t.detach().to("cpu").float().numpy()


def _rel_l2(y, ref):
    y = np.atleast_2d(y).astype(np.float64)
    ref = np.atleast_2d(ref)
    return np.linalg.norm(y - ref, axis=1) / np.maximum(np.linalg.norm(ref, axis=1), 1e-300)


# (m, n, k): single tile, ragged n / m / k (k not a multiple of 64 or 128),
# several tiles in both directions, long k
CASES = [(1, 16, 32), (33, 20, 256), (40, 64, 128), (64, 128, 128), (256, 128, 512), (300, 130, 224),
         (257, 300, 1056), (512, 256, 4096), (100, 1000, 96)]


@pytest.mark.parametrize("m,n,k", CASES)
def test_prefill_rel_l2(cuda_lib, m, n, k):
    W = _w(n, k, BF16, seed=61)
    X = _w(m, k, BF16, seed=62, std=1.0)
    c_ref, s_ref = oracle.quantize(_host_f32(W))
    Y_ref = oracle.gemm(c_ref, s_ref, n, k, _host_f32(X))
    codes, scales = cuda_lib.quantize(W.to(DEV))
    Y = cuda_lib.gemm_prefill(codes, scales, n, k, X.to(DEV))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(codes.cpu().numpy(), c_ref)
    assert _rel_l2(Y.cpu().numpy(), Y_ref).max() <= REL_L2_TOL


@pytest.mark.parametrize("out_dtype", [BF16, F16])
def test_prefill_low_precision_outputs(cuda_lib, out_dtype):
    m, n, k = 260, 200, 1024
    W = _w(n, k, BF16, seed=63)
    X = _w(m, k, F32, seed=64, std=1.0)
    c_ref, s_ref = oracle.quantize(_host_f32(W))
    Y_ref = oracle.gemm(c_ref, s_ref, n, k, _host_f32(X))
    codes, scales = cuda_lib.quantize(W.to(DEV))
    Y = cuda_lib.gemm_prefill(codes, scales, n, k, X.to(DEV), dtype=out_dtype)
    torch.cuda.synchronize()
    u = {BF16: 2.0 ** -8, F16: 2.0 ** -11}[out_dtype]
    assert _rel_l2(Y.float().cpu().numpy(), Y_ref).max() <= REL_L2_TOL + u * (1 + REL_L2_TOL)


def test_gemm_dispatches_large_m_to_prefill(cuda_lib):
    m, n, k = 96, 144, 512
    W = _w(n, k, BF16, seed=65)
    X = _w(m, k, BF16, seed=66, std=1.0).to(DEV)
    codes, scales = cuda_lib.quantize(W.to(DEV))
    a = cuda_lib.gemm(codes, scales, n, k, X)
    b = cuda_lib.gemm_prefill(codes, scales, n, k, X)
    b2 = cuda_lib.gemm_prefill(codes, scales, n, k, X)
    torch.cuda.synchronize()
    assert torch.equal(a, b) and torch.equal(b, b2)  # same kernel, deterministic


def test_prefill_strided_operands(cuda_lib):
    m, n, k, ldx, ldy = 70, 48, 256, 264, 56
    W = _w(n, k, BF16, seed=67)
    Xb = torch.zeros((m, ldx), dtype=BF16)
    Xb[:, :k] = _w(m, k, BF16, seed=68, std=1.0)
    c_ref, s_ref = oracle.quantize(_host_f32(W))
    Y_ref = oracle.gemm(c_ref, s_ref, n, k, _host_f32(Xb[:, :k]))
    codes, scales = cuda_lib.quantize(W.to(DEV))
    Yb = torch.full((m, ldy), 5.0, dtype=F32, device=DEV)
    cuda_lib.gemm_prefill(codes, scales, n, k, Xb.to(DEV)[:, :k], out=Yb[:, :n])
    torch.cuda.synchronize()
    Yh = Yb.cpu().numpy()
    assert np.all(Yh[:, n:] == 5.0)  # nothing written past n
    assert _rel_l2(Yh[:, :n], Y_ref).max() <= REL_L2_TOL


def test_prefill_workspace_errors(cuda_lib):
    m, n, k = 64, 32, 128
    codes, scales = cuda_lib.quantize(_w(n, k, BF16).to(DEV))
    X = torch.zeros((m, k), dtype=BF16, device=DEV)
    Y = torch.zeros((m, n), dtype=F32, device=DEV)
    need = cuda_lib.tq_gemm_prefill_workspace_bytes(m, k)
    assert need == 256 + ((m * k * 2 + 255) // 256) * 256
    ws = torch.zeros(need, dtype=torch.uint8, device=DEV)
    stream = torch.cuda.current_stream().cuda_stream
    st = cuda_lib.tq_gemm_prefill(codes.data_ptr(), scales.data_ptr(), n, k, X.data_ptr(), 1, m, k, Y.data_ptr(), 0,
                                  n, ws.data_ptr(), need - 1, stream)
    assert st == 5  # TQ_ERR_WORKSPACE
    st = cuda_lib.tq_gemm_prefill(codes.data_ptr(), scales.data_ptr(), n, k, X.data_ptr(), 1, m, k, Y.data_ptr(), 0,
                                  n, ws.data_ptr(), need, stream)
    assert st == 0
    torch.cuda.synchronize()
    assert cuda_lib.workspace_status(ws) == 0


def test_prefill_full_size_sampled(cuda_lib):
    """8192 x 8192 weight (bf16 source ~N(0, 0.02^2)) times a 2048-row bf16
    activation ~N(0, 1): every output column of a row sample of the weights
    (including the first and the last row) against the oracle."""
    n = k = 8192
    m = 2048
    W = inputs.gaussian_matrix(0, 40, n, k, 0.02, BF16, DEV)
    X = inputs.gaussian_matrix(1, 41, m, k, 1.0, BF16, DEV)
    codes, scales = cuda_lib.quantize(W)
    Y = cuda_lib.gemm_prefill(codes, scales, n, k, X)
    torch.cuda.synchronize()
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate(([0, n - 1, 127, 128], rng.choice(n, 12, replace=False))))
    c_ref, s_ref = oracle.quantize(_host_f32(W[torch.tensor(rows, device=DEV)]))
    Y_ref = oracle.gemm(c_ref, s_ref, len(rows), k, _host_f32(X))  # [m, rows]
    got = Y.cpu().numpy()[:, rows]
    # per activation row over the sampled outputs, and per sampled output over all rows
    assert _rel_l2(got, Y_ref).max() <= REL_L2_TOL
    assert _rel_l2(got.T, Y_ref.T).max() <= REL_L2_TOL


@pytest.mark.parametrize("m,k", [(1, 32), (3, 160), (2, 4096)])
def test_prerotate_plain_values(cuda_lib, m, k):
    """Row-major fp16 H(s .* x)/32 per 32-block, within one fp16 ulp of the
    fp64 rotation."""
    X = _w(m, k, BF16, seed=69, std=1.0)
    xr = cuda_lib.prerotate_plain(X.to(DEV))
    torch.cuda.synchronize()
    assert xr.dtype == F16 and tuple(xr.shape) == (m, k)
    got = xr.cpu().numpy().astype(np.float64)
    s = oracle.sign(np.arange(k)).astype(np.float64)
    ref = (oracle.fwht32((_host_f32(X).astype(np.float64) * s).reshape(m, k // 32, 32)) / 32).reshape(m, k)
    ulp = np.spacing(np.abs(ref.astype(np.float16))).astype(np.float64)
    assert np.all(np.abs(got - ref) <= ulp + 1e-12)


def test_prefill_xrot_shared_by_three_matrices(cuda_lib):
    """One plain pre-rotation serves three weight matrices of different n
    (q/k/v-like); each product equals tq_gemm_prefill's bit for bit."""
    m, k = 300, 512
    X = _w(m, k, BF16, seed=70, std=1.0).to(DEV)
    xr = cuda_lib.prerotate_plain(X)
    ws = torch.zeros(256, dtype=torch.uint8, device=DEV)
    for i, n in enumerate((256, 64, 130)):
        W = _w(n, k, BF16, seed=71 + i)
        codes, scales = cuda_lib.quantize(W.to(DEV))
        a = cuda_lib.gemm_prefill_xrot(codes, scales, n, k, xr, ws=ws)
        b = cuda_lib.gemm_prefill(codes, scales, n, k, X)
        torch.cuda.synchronize()
        assert torch.equal(a, b)
        assert cuda_lib.workspace_status(ws) == 0
        c_ref, s_ref = oracle.quantize(_host_f32(W))
        Y_ref = oracle.gemm(c_ref, s_ref, n, k, _host_f32(X))
        assert _rel_l2(a.cpu().numpy(), Y_ref).max() <= REL_L2_TOL


def test_prefill_xrot_argument_errors(cuda_lib):
    m, n, k = 64, 32, 128
    codes, scales = cuda_lib.quantize(_w(n, k, BF16).to(DEV))
    xr = torch.zeros((m * k + 8,), dtype=F16, device=DEV)
    Y = torch.zeros((m, n), dtype=F32, device=DEV)
    ws = torch.zeros(256, dtype=torch.uint8, device=DEV)
    stream = torch.cuda.current_stream().cuda_stream
    assert cuda_lib.tq_prefill_xrot_bytes(m, k) == m * k * 2
    call = lambda x, nbytes: cuda_lib.tq_gemm_prefill_xrot(codes.data_ptr(), scales.data_ptr(), n, k, x, m,
                                                            Y.data_ptr(), 0, n, ws.data_ptr(), nbytes, stream)
    assert call(xr.data_ptr(), 255) == 5          # TQ_ERR_WORKSPACE
    assert call(xr.data_ptr() + 2, 256) == 3      # TQ_ERR_ALIGNMENT (xrot not 16-byte aligned)
    assert call(0, 256) == 1                      # TQ_ERR_INVALID_ARG
    assert call(xr.data_ptr(), 256) == 0
    torch.cuda.synchronize()
    assert cuda_lib.workspace_status(ws) == 0


def test_prefill_timeout_path_reports_and_recovers(cuda_lib):
    """Test hook bit 1: the first CTA never issues its second activation-tile
    copy (nor counts its bytes).  Its bounded waits (5 ms under the hook)
    expire, the status word reports TQ_ERR_TIMEOUT, every tensor-memory column
    is released (the next launch allocates them again) and the next call is
    bit-identical to a clean one."""
    m, n, k = 300, 512, 1024  # several CTAs in both directions, 16 stages of 64 columns
    W = _w(n, k, BF16, seed=71)
    X = _w(m, k, BF16, seed=72, std=1.0).to(DEV)
    codes, scales = cuda_lib.quantize(W.to(DEV))
    ws = cuda_lib.prefill_workspace(m, k)
    Y_good = cuda_lib.gemm_prefill(codes, scales, n, k, X, ws=ws).clone()
    assert cuda_lib.workspace_status(ws) == 0
    try:
        cuda_lib.tq_debug_set_flags(2)
        cuda_lib.gemm_prefill(codes, scales, n, k, X, ws=ws)
        assert cuda_lib.workspace_status(ws) == 8  # TQ_ERR_TIMEOUT
    finally:
        cuda_lib.tq_debug_set_flags(0)
    for _ in range(2):
        Y = cuda_lib.gemm_prefill(codes, scales, n, k, X, ws=ws)
        assert cuda_lib.workspace_status(ws) == 0
        assert torch.equal(Y, Y_good)


def test_prefill_writes_nothing_past_its_outputs(cuda_lib):
    """Guard bands: Y rows of a larger buffer (ldy > n) and the rows past m
    keep their sentinel; only the m x n block changes."""
    m, n, k = 40, 130, 256
    W = _w(n, k, BF16, seed=73)
    X = _w(m, k, BF16, seed=74, std=1.0)
    c_ref, s_ref = oracle.quantize(_host_f32(W))
    Y_ref = oracle.gemm(c_ref, s_ref, n, k, _host_f32(X))
    codes, scales = cuda_lib.quantize(W.to(DEV))
    ldy = n + 14
    big = torch.full((m + 3, ldy), 12345.0, dtype=F32, device=DEV)
    ws = cuda_lib.prefill_workspace(m, k)
    st = cuda_lib.tq_gemm_prefill(codes.data_ptr(), scales.data_ptr(), n, k, X.to(DEV).data_ptr(), 1, m, k,
                                  big.data_ptr(), 0, ldy, ws.data_ptr(), ws.numel(),
                                  torch.cuda.current_stream().cuda_stream)
    assert st == 0
    torch.cuda.synchronize()
    got = big.cpu().numpy()
    assert _rel_l2(got[:m, :n], Y_ref).max() <= REL_L2_TOL
    assert np.all(got[:m, n:] == 12345.0)
    assert np.all(got[m:] == 12345.0)

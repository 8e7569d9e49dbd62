"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs.

Bars (TQ4_1S page "企业官网建设流程全解析": 格式原理 items 1-3, 解码速度 section):
  * quantise: codes and fp16 scale bits identical (integer / byte work);
  * dequantise: within a bound derived from the fp32 arithmetic (product
    rounding + five butterfly stages, plus rounding to the output type);
  * pre-rotation: fp16 values within 1 ulp of the fp64 transform;
  * GEMV / GEMM: relative L2 error <= 1e-3 per output row against the fp64
    product over the oracle's own dequantised weights.
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


USE_TMEM = 4  # tq_debug_set_flags bit 2: every m <= 32 on the tensor-memory kernel
USE_MMA_SYNC = 8  # bit 3: every m <= 32 on the mma.sync kernel


@pytest.fixture(params=["mma_sync", "tmem"])
def kernel(request, cuda_lib):
    """Runs a test on each fused-product kernel (m <= 32), whatever m: the
    mma.sync kernel (the default up to 8 rows) and the tcgen05 kernel with the
    weights in tensor memory (the default from 9 rows)."""
    cuda_lib.tq_debug_set_flags(USE_TMEM if request.param == "tmem" else USE_MMA_SYNC)
    try:
        yield request.param
    finally:
        cuda_lib.tq_debug_set_flags(0)


def _w(n, k, dtype, seed=0, std=0.02):
    return inputs.gaussian_matrix(seed, n * 7919 + k, n, k, std, dtype)


def _host_f32(t):
    return t.detach().to("cpu").float().numpy()


def _oracle_quantize(W):
    return oracle.quantize(_host_f32(W))


def _gpu_quantize(tq, W):
    codes, scales = tq.quantize(W.to(DEV))
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy().view(np.uint16)


def _rel_l2(y, ref):
    y = np.atleast_2d(y).astype(np.float64)
    ref = np.atleast_2d(ref)
    num = np.linalg.norm(y - ref, axis=1)
    den = np.maximum(np.linalg.norm(ref, axis=1), 1e-300)
    return num / den


QUANT_SHAPES = [(1, 32), (3, 64), (17, 96), (16, 128), (33, 160), (5, 4096), (64, 1056), (100, 384)]


@pytest.mark.parametrize("dtype", [F32, BF16, F16])
@pytest.mark.parametrize("n,k", QUANT_SHAPES)
def test_quantize_bit_exact(cuda_lib, n, k, dtype):
    W = _w(n, k, dtype)
    c_ref, s_ref = _oracle_quantize(W)
    c, s = _gpu_quantize(cuda_lib, W)
    np.testing.assert_array_equal(s, s_ref)
    np.testing.assert_array_equal(c, c_ref)


def test_quantize_strided_and_special_values(cuda_lib):
    n, k, ld = 12, 256, 264
    base = torch.zeros((n, ld), dtype=F32)
    base[:, :k] = _w(n, k, F32, seed=3)
    base[0, :k] = 0.0                                   # all-zero row
    base[1, :k] = 1e-30                                 # scale underflows to 0
    base[2, :k] = 1000.0 * torch.sign(_w(1, k, F32)[0]) # large values
    s = torch.tensor(oracle.sign(np.arange(k)).astype(np.float32))
    base[3, :k] = -0.5 * s                              # worked block, every block
    base[4, :k] = 3.0                                   # constant row
    base[5, :k] = -0.0
    W = base[:, :k]
    c_ref, s_ref = oracle.quantize(W.numpy().copy())
    Wd = base.to(DEV)
    codes, scales = cuda_lib.quantize(Wd[:, :k])
    torch.cuda.synchronize()
    np.testing.assert_array_equal(codes.cpu().numpy(), c_ref)
    np.testing.assert_array_equal(scales.cpu().numpy().view(np.uint16), s_ref)


def _dequant_bound(codes, scales, n, k, w64, out_dtype):
    code, d = oracle.unpack(codes, scales, n, k)
    M32, _, _ = oracle.codebook()
    absc = M32[code & 7].astype(np.float64) * np.repeat(d.view(np.float16).astype(np.float64), 16, axis=2).reshape(n, k)
    blk = absc.reshape(n, k // 32, 32).sum(axis=2, keepdims=True) / 32
    arith = 8 * 2.0 ** -24 * np.broadcast_to(blk, (n, k // 32, 32)).reshape(n, k)
    rel = {F32: 2.0 ** -24, BF16: 2.0 ** -8, F16: 2.0 ** -11}[out_dtype]
    floor = {F32: 2.0 ** -149, BF16: 2.0 ** -133, F16: 2.0 ** -25}[out_dtype]
    return arith * (1 + rel) + np.abs(w64) * rel + floor


@pytest.mark.parametrize("out_dtype", [F32, BF16, F16])
@pytest.mark.parametrize("n,k", [(3, 64), (17, 96), (33, 160), (64, 1056)])
def test_dequantize_within_arithmetic_bound(cuda_lib, n, k, out_dtype):
    W = _w(n, k, BF16, seed=5)
    c_ref, s_ref = _oracle_quantize(W)
    w64 = oracle.dequantize(c_ref, s_ref, n, k)
    codes = torch.tensor(c_ref, device=DEV)
    scales = torch.tensor(s_ref.view(np.int16), device=DEV)
    out = cuda_lib.dequantize(codes, scales, n, k, dtype=out_dtype)
    torch.cuda.synchronize()
    got = out.float().cpu().numpy().astype(np.float64)
    bound = _dequant_bound(c_ref, s_ref, n, k, w64, out_dtype)
    err = np.abs(got - w64)
    assert np.all(err <= bound), float((err / bound).max())


def test_dequantize_strided_output(cuda_lib):
    n, k, ld = 9, 128, 136
    W = _w(n, k, F32, seed=6)
    c_ref, s_ref = _oracle_quantize(W)
    codes = torch.tensor(c_ref, device=DEV)
    scales = torch.tensor(s_ref.view(np.int16), device=DEV)
    out = torch.full((n, ld), 7.0, device=DEV)
    cuda_lib.dequantize(codes, scales, n, k, out=out[:, :k])
    torch.cuda.synchronize()
    o = out.cpu().numpy()
    assert np.all(o[:, k:] == 7.0)  # nothing written past k
    w64 = oracle.dequantize(c_ref, s_ref, n, k)
    assert np.all(np.abs(o[:, :k] - w64) <= _dequant_bound(c_ref, s_ref, n, k, w64, F32))


@pytest.mark.parametrize("out_dtype", [BF16, F32, F16])
def test_dequantize_batch_matches_single_launches(cuda_lib, out_dtype):
    """tq_dequantize_batch (one launch over several matrices, work items
    spread over persistent CTAs) writes exactly what one tq_dequantize per
    matrix writes: ragged k, rows not a multiple of 8 or 16, an empty matrix,
    strided outputs whose padding columns stay untouched."""
    shapes = [(64, 1056), (17, 96), (0, 128), (300, 4160), (33, 160), (1000, 1024), (9, 32)]
    items, expect = [], []
    for i, (n, k) in enumerate(shapes):
        W = _w(max(n, 1), k, BF16, seed=120 + i)[:n]
        codes, scales = cuda_lib.quantize(W.to(DEV).contiguous())
        ld = k + (8 if i % 2 else 0)
        out = torch.full((n, ld), 7.0, dtype=out_dtype, device=DEV)
        items.append((codes, scales, n, k, out[:, :k]))
        expect.append(cuda_lib.dequantize(codes, scales, n, k, dtype=out_dtype) if n else None)
    cuda_lib.dequantize_batch(items)
    torch.cuda.synchronize()
    for (codes, scales, n, k, o), ref in zip(items, expect):
        if n == 0:
            continue
        assert torch.equal(o, ref), (n, k)
        full = o.as_strided((n, o.stride(0)), (o.stride(0), 1))
        assert bool((full[:, k:] == 7.0).all()), (n, k)


def test_dequantize_batch_layer_against_oracle(cuda_lib):
    """Eight matrices (the batch limit) in one launch; sampled rows checked
    against the oracle within the arithmetic bound."""
    shapes = [(256, 1024), (64, 1024), (64, 1024), (256, 1024), (512, 1024), (512, 1024), (256, 3584), (40, 2080)]
    items, packed = [], []
    for i, (n, k) in enumerate(shapes):
        W = _w(n, k, BF16, seed=140 + i)
        c_ref, s_ref = _oracle_quantize(W)
        codes = torch.tensor(c_ref, device=DEV)
        scales = torch.tensor(s_ref.view(np.int16), device=DEV)
        items.append((codes, scales, n, k, torch.empty((n, k), dtype=F32, device=DEV)))
        packed.append((c_ref, s_ref))
    cuda_lib.dequantize_batch(items)
    torch.cuda.synchronize()
    for (codes, scales, n, k, o), (c_ref, s_ref) in zip(items, packed):
        w64 = oracle.dequantize(c_ref, s_ref, n, k)
        got = o.cpu().numpy().astype(np.float64)
        bound = _dequant_bound(c_ref, s_ref, n, k, w64, F32)
        assert np.all(np.abs(got - w64) <= bound), (n, k)


@pytest.mark.parametrize("m,k", [(1, 32), (1, 4096), (3, 96), (5, 160)])
def test_prerotate_values_and_layout(cuda_lib, m, k):
    X = _w(m, k, BF16, seed=7, std=1.0)
    xr = cuda_lib.prerotate(X.to(DEV))
    torch.cuda.synchronize()
    got = xr.cpu().numpy().view(np.float16).astype(np.float64)
    nsb = (k // 32 + 3) // 4
    got = got.reshape(m, nsb * 4, 4, 8)  # [row][block][t][q]
    s = oracle.sign(np.arange(k)).astype(np.float64)
    ref = oracle.fwht32((_host_f32(X).astype(np.float64) * s).reshape(m, k // 32, 32)) / 32
    # entry [t][q] of a block is element (q//2)*8 + 2t + q%2
    t_idx, q_idx = np.meshgrid(np.arange(4), np.arange(8), indexing="ij")
    elem = (q_idx // 2) * 8 + 2 * t_idx + q_idx % 2
    unperm = np.zeros((m, nsb * 4, 32))
    unperm[:, :, elem] = got
    assert np.all(unperm[:, k // 32:, :] == 0)  # padding blocks
    r16 = ref.astype(np.float16).astype(np.float64)
    ulp = np.spacing(np.abs(r16).astype(np.float16)).astype(np.float64)
    assert np.all(np.abs(unperm[:, : k // 32, :] - ref) <= ulp + 1e-12)


GEMM_CASES = [
    (1, 1, 32), (1, 15, 96), (1, 16, 128), (1, 17, 4096), (1, 1024, 4096), (2, 33, 256), (3, 64, 160),
    (5, 40, 1024), (8, 16, 8192), (9, 48, 512), (16, 100, 384), (31, 17, 1024), (32, 64, 2048),
    (33, 20, 256), (40, 64, 128), (4, 3, 16384), (20, 50, 640), (24, 33, 1056), (17, 300, 4096),
    # two to four rows: the half-block-combination kernels, with split tiles and ragged edges
    (2, 1, 32), (2, 40, 4096), (3, 100, 2048), (4, 17, 8192), (4, 300, 640), (3, 2000, 160),
]


@pytest.mark.parametrize("m,n,k", GEMM_CASES)
def test_gemm_rel_l2(cuda_lib, kernel, m, n, k):
    W = _w(n, k, BF16, seed=8)
    X = _w(m, k, BF16, seed=9, std=1.0)
    c_ref, s_ref = _oracle_quantize(W)
    Y_ref = oracle.gemm(c_ref, s_ref, n, k, _host_f32(X))
    codes, scales = cuda_lib.quantize(W.to(DEV))
    Y = cuda_lib.gemm(codes, scales, n, k, X.to(DEV))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(codes.cpu().numpy(), c_ref)
    assert _rel_l2(Y.cpu().numpy(), Y_ref).max() <= REL_L2_TOL


@pytest.mark.parametrize("out_dtype", [BF16, F16])
def test_gemv_low_precision_outputs(cuda_lib, kernel, out_dtype):
    n, k = 300, 1024
    W = _w(n, k, BF16, seed=10)
    x = _w(1, k, F32, seed=11, std=1.0)[0]
    c_ref, s_ref = _oracle_quantize(W)
    y_ref = oracle.gemm(c_ref, s_ref, n, k, _host_f32(x)[None])[0]
    codes, scales = cuda_lib.quantize(W.to(DEV))
    y = cuda_lib.gemv(codes, scales, n, k, x.to(DEV), dtype=out_dtype)
    torch.cuda.synchronize()
    # ||round(y) - y64|| <= u ||y|| + ||y - y64||: the output type's unit
    # roundoff u adds to the product's 1e-3 bar
    u = {BF16: 2.0 ** -8, F16: 2.0 ** -11}[out_dtype]
    assert _rel_l2(y.float().cpu().numpy(), y_ref).max() <= REL_L2_TOL + u * (1 + REL_L2_TOL)


def test_gemv_single_matrix_workload(cuda_lib):
    """2048x2048 fp32 ~N(0, 0.02^2), x fp32 ~N(0,1): quantise, dequantise, GEMV."""
    W, x = inputs.single_matrix()
    n, k = W.shape
    c_ref, s_ref = oracle.quantize(W.numpy())
    Wd = W.to(DEV)
    codes, scales = cuda_lib.quantize(Wd)
    deq = cuda_lib.dequantize(codes, scales, n, k, dtype=F32)
    y = cuda_lib.gemv(codes, scales, n, k, x.to(DEV))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(codes.cpu().numpy(), c_ref)
    np.testing.assert_array_equal(scales.cpu().numpy().view(np.uint16), s_ref)
    w64 = oracle.dequantize(c_ref, s_ref, n, k)
    assert np.all(np.abs(deq.cpu().numpy() - w64) <= _dequant_bound(c_ref, s_ref, n, k, w64, F32))
    y_ref = oracle.gemm(c_ref, s_ref, n, k, x.numpy()[None])[0]
    assert _rel_l2(y.cpu().numpy(), y_ref)[0] <= REL_L2_TOL


def test_gemv_deterministic_and_workspace_reuse(cuda_lib, kernel):
    n, k = 4096, 4096
    W = inputs.gaussian_matrix(0, 1, n, k, 0.02, BF16, DEV)
    x = inputs.gaussian_matrix(1, 1, 1, k, 1.0, BF16, DEV)[0]
    codes, scales = cuda_lib.quantize(W)
    ws = cuda_lib.workspace(1, n, k)
    y1 = cuda_lib.gemv(codes, scales, n, k, x, ws=ws).clone()
    for _ in range(3):
        y2 = cuda_lib.gemv(codes, scales, n, k, x, ws=ws)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)


def test_shared_prerotation_matches_gemm(cuda_lib):
    """One pre-rotated activation shared by three matrices (q/k/v style).
    tq_gemm_xrot takes the mma.sync kernel's fragment-ordered activation, so
    it is compared bit for bit with tq_gemm on that (default) kernel, and with
    the tensor-memory kernel within the product's bar."""
    k = 1024
    x = _w(1, k, BF16, seed=12, std=1.0).to(DEV)
    xr = cuda_lib.prerotate(x)
    for n in (256, 64, 64):
        W = _w(n, k, BF16, seed=n).to(DEV)
        codes, scales = cuda_lib.quantize(W)
        ws = cuda_lib.workspace(1, n, k)
        a = cuda_lib.gemm_xrot(codes, scales, n, k, xr, 1, ws=ws)
        b = cuda_lib.gemm(codes, scales, n, k, x)  # one row: the mma.sync kernel
        try:
            cuda_lib.tq_debug_set_flags(USE_TMEM)
            c = cuda_lib.gemm(codes, scales, n, k, x)
        finally:
            cuda_lib.tq_debug_set_flags(0)
        torch.cuda.synchronize()
        assert torch.equal(a, b)
        assert _rel_l2(a.cpu().numpy(), c.cpu().numpy().astype(np.float64)).max() <= REL_L2_TOL


def test_workspace_errors(cuda_lib):
    n, k = 64, 256
    codes, scales = cuda_lib.quantize(_w(n, k, BF16).to(DEV))
    x = torch.zeros(k, dtype=BF16, device=DEV)
    y = torch.zeros(n, dtype=F32, device=DEV)
    need = cuda_lib.tq_gemm_workspace_bytes(1, n, k)
    ws = torch.zeros(need + 512, dtype=torch.uint8, device=DEV)
    st = cuda_lib.tq_gemv(codes.data_ptr(), scales.data_ptr(), n, k, x.data_ptr(), 1, y.data_ptr(), 0,
                          ws.data_ptr(), 255, torch.cuda.current_stream().cuda_stream)
    assert st == 5  # smaller than the header alone
    st = cuda_lib.tq_gemv(codes.data_ptr(), scales.data_ptr(), n, k, x.data_ptr(), 1, y.data_ptr(), 0,
                          ws.data_ptr() + 16, need, torch.cuda.current_stream().cuda_stream)
    assert st == 5
    st = cuda_lib.tq_gemv(codes.data_ptr(), scales.data_ptr(), n, k, x.data_ptr(), 1, y.data_ptr(), 0,
                          0, need, torch.cuda.current_stream().cuda_stream)
    assert st == 5


# ---------------------------------------------------------------------------
# full-size workloads, checked on sampled rows (rows are independent)
# ---------------------------------------------------------------------------
def _sample_rows(n, count=24, seed=0):
    rng = np.random.default_rng(seed + n)
    rows = np.unique(np.concatenate(([0, n - 1], rng.choice(n, count, replace=False))))
    return rows


def test_llama3_8b_layer_full_size(cuda_lib, kernel):
    weights, acts = inputs.llama3_8b_layer(device=DEV)
    for name, W in weights.items():
        n, k = W.shape
        x = acts[inputs.LLAMA3_8B_INPUTS[name]]
        codes, scales = cuda_lib.quantize(W)
        y = cuda_lib.gemv(codes, scales, n, k, x)
        torch.cuda.synchronize()
        rows = _sample_rows(n)
        Wr = W[torch.tensor(rows, device=DEV)]
        c_ref, s_ref = oracle.quantize(_host_f32(Wr))
        gc, gs = oracle.row_view(codes.cpu().numpy(), scales.cpu().numpy().view(np.uint16), n, k)
        rc, rs = oracle.row_view(c_ref, s_ref, len(rows), k)
        np.testing.assert_array_equal(gc[rows], rc, err_msg=name)
        np.testing.assert_array_equal(gs[rows], rs, err_msg=name)
        y_ref = oracle.gemm(c_ref, s_ref, len(rows), k, _host_f32(x)[None])[0]
        assert _rel_l2(y.cpu().numpy()[rows], y_ref)[0] <= REL_L2_TOL, name


@pytest.mark.parametrize("m", [1, 2, 4, 8, 16, 24, 32])
def test_ffn_70b_skinny_sweep_full_size(cuda_lib, kernel, m):
    n, k = inputs.FFN_70B["gate"]
    W = inputs.gaussian_matrix(2, 0, n, k, 0.015, BF16, DEV)
    X = inputs.gaussian_matrix(1, 100 + m, m, k, 1.0, BF16, DEV)
    codes, scales = cuda_lib.quantize(W)
    Y = cuda_lib.gemm(codes, scales, n, k, X)
    torch.cuda.synchronize()
    rows = _sample_rows(n, 12)
    c_ref, s_ref = oracle.quantize(_host_f32(W[torch.tensor(rows, device=DEV)]))
    Y_ref = oracle.gemm(c_ref, s_ref, len(rows), k, _host_f32(X))
    assert _rel_l2(Y.cpu().numpy()[:, rows], Y_ref).max() <= REL_L2_TOL


@pytest.mark.parametrize("m", [1, 2, 3, 4, 5])
def test_gemm_batch_shares_prerotation(cuda_lib, kernel, m):
    """Six matrices with three distinct inputs in one batch (q/k/v-style and
    gate/up-style sharing) against the oracle and the one-matrix path."""
    shapes = [(256, 1024, "a"), (64, 1024, "a"), (64, 1024, "a"), (300, 512, "b"), (300, 512, "b"), (40, 2048, "c")]
    Xs = {name: _w(m, k, BF16, seed=20 + i, std=1.0) for i, (_, k, name) in enumerate(shapes)}
    items, refs, singles = [], [], []
    for i, (n, k, name) in enumerate(shapes):
        W = _w(n, k, BF16, seed=30 + i)
        c_ref, s_ref = _oracle_quantize(W)
        refs.append(oracle.gemm(c_ref, s_ref, n, k, _host_f32(Xs[name])))
        codes, scales = cuda_lib.quantize(W.to(DEV))
        X = Xs[name]
        Xd = X.to(DEV) if name not in [it[6] for it in items] else [it[4] for it in items if it[6] == name][0]
        Y = torch.empty((m, n), dtype=F32, device=DEV)
        items.append((codes, scales, n, k, Xd, Y, name))
        singles.append(cuda_lib.gemm(codes, scales, n, k, Xd))
    cuda_lib.gemm_batch([it[:6] for it in items], m=m)
    torch.cuda.synchronize()
    for (codes, scales, n, k, Xd, Y, name), ref, single in zip(items, refs, singles):
        assert _rel_l2(Y.cpu().numpy(), ref).max() <= REL_L2_TOL
        np.testing.assert_allclose(Y.cpu().numpy(), single.cpu().numpy(), rtol=1e-5, atol=1e-6)


def test_timeout_path_reports_and_recovers(cuda_lib, kernel):
    """Fault injection on the host side of the contract: one bulk copy is never
    issued, the kernel's bounded wait (5 ms under injection) expires, it sets
    the workspace status word and returns; the context stays usable."""
    n, k = 4096, 4096
    W = inputs.gaussian_matrix(0, 3, n, k, 0.02, BF16, DEV)
    x = inputs.gaussian_matrix(1, 3, 1, k, 1.0, BF16, DEV)[0]
    codes, scales = cuda_lib.quantize(W)
    ws = cuda_lib.workspace(1, n, k)
    y_good = cuda_lib.gemv(codes, scales, n, k, x, ws=ws).clone()
    assert cuda_lib.workspace_status(ws) == 0
    base = USE_TMEM if kernel == "tmem" else USE_MMA_SYNC
    try:
        cuda_lib.tq_debug_set_flags(base | 1)
        cuda_lib.gemv(codes, scales, n, k, x, ws=ws)
        assert cuda_lib.workspace_status(ws) == 8  # TQ_ERR_TIMEOUT
    finally:
        cuda_lib.tq_debug_set_flags(base)
    y = cuda_lib.gemv(codes, scales, n, k, x, ws=ws)
    assert cuda_lib.workspace_status(ws) == 0
    assert torch.equal(y, y_good)


def test_gemv_correct_while_another_stream_holds_the_sms(cuda_lib):
    """The fused product relies on its whole grid being resident (a split
    tile's first warp polls for the partial sums of later CTAs); it is launched
    cooperatively, so a long kernel on another stream that occupies the SMs
    delays it but cannot make that poll run out.  Status TQ_OK and output
    identical to the solo run."""
    n, k = 14336, 4096
    W = inputs.gaussian_matrix(0, 5, n, k, 0.02, BF16, DEV)
    x = inputs.gaussian_matrix(1, 5, 1, k, 1.0, BF16, DEV)[0]
    codes, scales = cuda_lib.quantize(W)
    ws = cuda_lib.workspace(1, n, k)
    y_solo = cuda_lib.gemv(codes, scales, n, k, x, ws=ws).clone()
    A = torch.randn(8192, 8192, dtype=BF16, device=DEV)
    B = torch.randn(8192, 8192, dtype=BF16, device=DEV)
    C = torch.empty(8192, 8192, dtype=BF16, device=DEV)
    torch.cuda.synchronize()
    busy = torch.cuda.Stream()
    with torch.cuda.stream(busy):
        for _ in range(40):  # a few tens of ms of dense matmuls on every SM
            torch.matmul(A, B, out=C)
    for _ in range(5):
        y = cuda_lib.gemv(codes, scales, n, k, x, ws=ws)
    assert cuda_lib.workspace_status(ws) == 0
    torch.cuda.synchronize()
    assert torch.equal(y, y_solo)


@pytest.mark.parametrize("m", [1, 3, 17])
def test_gemm_writes_nothing_past_its_outputs(cuda_lib, kernel, m):
    """Guard bands: with n inside the last 16-row tile (rows past n exist in
    the packed planes) and ldy > n, every column past n and every row past m
    keeps its sentinel."""
    n, k = 77, 640
    W = _w(n, k, BF16, seed=40)
    X = _w(m, k, BF16, seed=41, std=1.0)
    c_ref, s_ref = _oracle_quantize(W)
    Y_ref = oracle.gemm(c_ref, s_ref, n, k, _host_f32(X))
    codes, scales = cuda_lib.quantize(W.to(DEV))
    ldy = 96
    big = torch.full((m + 2, ldy), -777.0, dtype=F32, device=DEV)
    ws = cuda_lib.workspace(m, n, k)
    st = cuda_lib.tq_gemm(codes.data_ptr(), scales.data_ptr(), n, k, X.to(DEV).data_ptr(), 1, m, k, big.data_ptr(),
                          0, ldy, ws.data_ptr(), ws.numel(), torch.cuda.current_stream().cuda_stream)
    assert st == 0
    torch.cuda.synchronize()
    got = big.cpu().numpy()
    assert _rel_l2(got[:m, :n], Y_ref).max() <= REL_L2_TOL
    assert np.all(got[:m, n:] == -777.0)
    assert np.all(got[m:] == -777.0)


@pytest.mark.parametrize("m", [1, 8, 32])
def test_gemm_small_weights(cuda_lib, kernel, m):
    """Weights of std 1e-4: half-block scales d around 6e-4, so the products
    fp16(c * d) of the smallest centroid fall near the bottom of the fp16
    normal range (6.1e-5), and some below it."""
    n, k = 256, 2048
    W = _w(n, k, F32, seed=42, std=1e-4)
    X = _w(m, k, BF16, seed=43, std=1.0)
    c_ref, s_ref = _oracle_quantize(W)
    Y_ref = oracle.gemm(c_ref, s_ref, n, k, _host_f32(X))
    codes, scales = cuda_lib.quantize(W.to(DEV))
    Y = cuda_lib.gemm(codes, scales, n, k, X.to(DEV))
    torch.cuda.synchronize()
    assert _rel_l2(Y.cpu().numpy(), Y_ref).max() <= REL_L2_TOL


STEAL_ALL = 16  # tq_debug_set_flags bit 4: split tiles' first warps compute every later contribution


@pytest.mark.parametrize("m", [1, 2, 3, 4, 5, 8, 16, 24, 32])
def test_split_tiles_recomputed_contributions_are_bit_identical(cuda_lib, m):
    """The mma.sync kernel needs no co-resident grid: a split tile's first
    warp computes a later contribution that does not arrive in time from the
    packed weights.  Forced on every split tile (test hook), the products are
    bit-identical to the normal path, which reads those contributions."""
    shapes = [(4096, 4096), (300, 14336), (1000, 1056)]
    for n, k in shapes:
        W = _w(n, k, BF16, seed=50 + m)
        X = _w(m, k, BF16, seed=51 + m, std=1.0)
        codes, scales = cuda_lib.quantize(W.to(DEV))
        try:
            cuda_lib.tq_debug_set_flags(USE_MMA_SYNC)
            ref = cuda_lib.gemm(codes, scales, n, k, X.to(DEV)).clone()
            cuda_lib.tq_debug_set_flags(USE_MMA_SYNC | STEAL_ALL)
            got = cuda_lib.gemm(codes, scales, n, k, X.to(DEV))
        finally:
            cuda_lib.tq_debug_set_flags(0)
        torch.cuda.synchronize()
        assert torch.equal(got, ref), (m, n, k)


def test_split_tiles_recomputed_nvfp4(cuda_lib):
    """The same for the NVFP4 product (its tensor scale applies to the
    recomputed contributions too)."""
    for m in (1, 16):
        n, k = 4096, 4096
        W = _w(n, k, BF16, seed=60 + m)
        X = _w(m, k, BF16, seed=61 + m, std=1.0).to(DEV)
        c, s, t = cuda_lib.nvfp4_quantize(W.to(DEV))
        ref = cuda_lib.nvfp4_gemm(c, s, t, n, k, X).clone()
        try:
            cuda_lib.tq_debug_set_flags(STEAL_ALL)
            got = cuda_lib.nvfp4_gemm(c, s, t, n, k, X)
        finally:
            cuda_lib.tq_debug_set_flags(0)
        torch.cuda.synchronize()
        assert torch.equal(got, ref), m

"""The workspace-free GEMV entry point (tq_gemv_static_scratch).

It serves callers that cannot allocate device memory (allocator callbacks,
plugins that only receive an operation's tensors, fully reserved devices): its
scratch is a fixed array inside the library instead of a caller workspace.
This file is collected last so that a failure here stops a run only after
every other test has run; it must pass alone in a fresh process as well.
"""
import numpy as np
import pytest
import torch

import oracle
from dequant_gemv_tq4_b200 import inputs

pytestmark = pytest.mark.gpu

REL_L2_TOL = 1e-3
TQ_ERR_TIMEOUT = 8


def _rel_l2(a, b):
    a = a.astype(np.float64)
    b = b.astype(np.float64)
    return np.linalg.norm(a - b) / np.linalg.norm(b)


def _static_gemv(tq, codes, scales, n, k, x):
    y = torch.full((n,), float("nan"), dtype=torch.float32, device="cuda")
    st = tq.tq_gemv_static_scratch(codes.data_ptr(), scales.data_ptr(), n, k, x.data_ptr(), tq.TQ_BF16,
                                   y.data_ptr(), tq.TQ_F32, torch.cuda.current_stream().cuda_stream)
    assert st == 0, tq.status_string(st)
    return y


def test_static_scratch_gemv_matches_workspace_gemv_and_oracle(cuda_lib):
    tq = cuda_lib
    oracle.build()
    # three calls in a row: a large problem, a smaller one, then the large one
    # again, which reuses partial-sum slots that the first call left tagged;
    # none may depend on what an earlier call left in the shared scratch
    for seed, (n, k) in enumerate(((4096, 4096), (1000, 1056), (4096, 4096))):
        W = inputs.gaussian_matrix(seed, 11, n, k, 0.02, torch.bfloat16, "cuda")
        x = inputs.gaussian_matrix(seed, 12, 1, k, 1.0, torch.bfloat16, "cuda")[0]
        codes, scales = tq.quantize(W)
        y_ref = tq.gemv(codes, scales, n, k, x)  # the entry point with a caller workspace
        y = _static_gemv(tq, codes, scales, n, k, x)
        torch.cuda.synchronize()
        assert tq.tq_static_scratch_status(1, torch.cuda.current_stream().cuda_stream) == 0
        got = y.cpu().numpy()
        assert _rel_l2(got, y_ref.cpu().numpy()) <= REL_L2_TOL
        # and against the CPU oracle (fp64 product over its own dequantised weights)
        c_or, s_or = oracle.quantize(W.float().cpu().numpy())
        y_or = oracle.gemm(c_or, s_or, n, k, x.float().cpu().numpy()[None].astype(np.float64))[0]
        assert _rel_l2(got, y_or) <= REL_L2_TOL


def test_static_scratch_on_a_second_stream(cuda_lib):
    """Calls on two streams, ordered by an event: the supported pattern."""
    tq = cuda_lib
    n, k = 2048, 2048
    W = inputs.gaussian_matrix(5, 11, n, k, 0.02, torch.bfloat16, "cuda")
    x = inputs.gaussian_matrix(5, 12, 1, k, 1.0, torch.bfloat16, "cuda")[0]
    codes, scales = tq.quantize(W)
    y_ref = tq.gemv(codes, scales, n, k, x)
    y1 = _static_gemv(tq, codes, scales, n, k, x)
    done = torch.cuda.Event()
    done.record()
    side = torch.cuda.Stream()
    side.wait_event(done)
    with torch.cuda.stream(side):
        y2 = _static_gemv(tq, codes, scales, n, k, x)
    torch.cuda.synchronize()
    for y in (y1, y2):
        assert _rel_l2(y.cpu().numpy(), y_ref.cpu().numpy()) <= REL_L2_TOL


def test_static_scratch_timeout_is_reported_and_recovers(cuda_lib):
    """A bounded wait that runs out (test hook: one bulk copy is never issued,
    5 ms limit) shows in tq_static_scratch_status; the next call is correct."""
    tq = cuda_lib
    stream = torch.cuda.current_stream().cuda_stream
    n, k = 4096, 4096
    W = inputs.gaussian_matrix(7, 11, n, k, 0.02, torch.bfloat16, "cuda")
    x = inputs.gaussian_matrix(7, 12, 1, k, 1.0, torch.bfloat16, "cuda")[0]
    codes, scales = tq.quantize(W)
    y_ref = tq.gemv(codes, scales, n, k, x)
    torch.cuda.synchronize()
    tq.tq_debug_set_flags(1)
    try:
        _static_gemv(tq, codes, scales, n, k, x)
        assert tq.tq_static_scratch_status(1, stream) == TQ_ERR_TIMEOUT
    finally:
        tq.tq_debug_set_flags(0)
    assert tq.tq_static_scratch_status(0, stream) == 0  # cleared
    y = _static_gemv(tq, codes, scales, n, k, x)
    assert tq.tq_static_scratch_status(0, stream) == 0
    assert _rel_l2(y.cpu().numpy(), y_ref.cpu().numpy()) <= REL_L2_TOL


def test_static_scratch_rejects_oversized_problems(cuda_lib):
    tq = cuda_lib
    # the pre-rotated activation alone (2 bytes per column) exceeds the fixed
    # scratch, whichever kernel would run the product
    n, k = 16, 1 << 22
    assert tq.tq_gemm_workspace_bytes(1, n, k) > (4 << 20)
    assert 2 * k > (4 << 20)
    st = tq.tq_gemv_static_scratch(1 << 20, 1 << 20, n, k, 1 << 20, tq.TQ_BF16, 1 << 20, tq.TQ_F32,
                                   torch.cuda.current_stream().cuda_stream)
    assert st == 2  # TQ_ERR_SHAPE, returned before anything is launched

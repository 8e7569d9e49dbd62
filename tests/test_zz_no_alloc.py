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

from dequant_gemv_tq4_b200 import inputs

pytestmark = pytest.mark.gpu

REL_L2_TOL = 1e-3


def _rel_l2(a, b):
    a = a.astype(np.float64)
    b = b.astype(np.float64)
    return np.linalg.norm(a - b) / np.linalg.norm(b)


def test_static_scratch_gemv_matches_workspace_gemv(cuda_lib):
    tq = cuda_lib
    stream = torch.cuda.current_stream().cuda_stream
    # two calls in a row on different problems: the second must not depend on
    # what the first left in the shared scratch
    for seed, (n, k) in enumerate(((4096, 4096), (1000, 1056))):
        W = inputs.gaussian_matrix(seed, 11, n, k, 0.02, torch.bfloat16, "cuda")
        x = inputs.gaussian_matrix(seed, 12, 1, k, 1.0, torch.bfloat16, "cuda")[0]
        codes, scales = tq.quantize(W)
        y_ref = tq.gemv(codes, scales, n, k, x)  # the entry point with a caller workspace
        y = torch.full((n,), float("nan"), dtype=torch.float32, device="cuda")
        st = tq.tq_gemv_static_scratch(codes.data_ptr(), scales.data_ptr(), n, k, x.data_ptr(), tq.TQ_BF16,
                                       y.data_ptr(), tq.TQ_F32, stream)
        assert st == 0, tq.status_string(st)
        torch.cuda.synchronize()
        assert _rel_l2(y.cpu().numpy(), y_ref.cpu().numpy()) <= REL_L2_TOL


def test_static_scratch_rejects_oversized_problems(cuda_lib):
    tq = cuda_lib
    n, k = 1 << 20, 4096  # partial sums alone exceed the fixed scratch
    assert tq.tq_gemm_workspace_bytes(1, n, k) > (4 << 20)
    st = tq.tq_gemv_static_scratch(1 << 20, 1 << 20, n, k, 1 << 20, tq.TQ_BF16, 1 << 20, tq.TQ_F32,
                                   torch.cuda.current_stream().cuda_stream)
    assert st == 2  # TQ_ERR_SHAPE, returned before anything is launched

"""TQ4_1S weight codec and fused dequant-GEMV for NVIDIA B200 (sm_100a).

Thin Python binding over the C ABI in ``include/tq.h`` (``libtq.so``, built
in-tree by ``dequant_gemv_tq4_b200/build.py``).  Every step of the path runs in
the library's CUDA kernels; this module only marshals arguments.  PyTorch is
used for device memory and streams.  There is no CPU fallback: if the
library cannot be loaded, every call raises.

Two layers:
  * ``tq_*`` functions with the C names and raw integer pointers (what the
    ABI tests call);
  * tensor helpers (``quantize``, ``dequantize``, ``prerotate``, ``gemm``,
    ``gemv``, ``gemm_xrot``) that allocate outputs with torch and pass
    ``data_ptr()`` and the current CUDA stream.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtq.so")

TQ_F32, TQ_BF16, TQ_F16 = 0, 1, 2
_DTYPE_CODE = {torch.float32: TQ_F32, torch.bfloat16: TQ_BF16, torch.float16: TQ_F16}
STATUS_NAMES = {0: "TQ_OK", 1: "TQ_ERR_INVALID_ARG", 2: "TQ_ERR_SHAPE", 3: "TQ_ERR_ALIGNMENT",
                4: "TQ_ERR_DTYPE", 5: "TQ_ERR_WORKSPACE", 6: "TQ_ERR_CUDA", 7: "TQ_ERR_UNSUPPORTED",
                8: "TQ_ERR_TIMEOUT"}
TQ_MAX_BATCH = 8


class GemmDesc(ctypes.Structure):
    """Mirror of ``tq_gemm_desc`` in include/tq.h."""
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("n", ctypes.c_int64),
                ("k", ctypes.c_int64), ("X", ctypes.c_void_p), ("ldx", ctypes.c_int64), ("Y", ctypes.c_void_p),
                ("ldy", ctypes.c_int64)]


class DequantDesc(ctypes.Structure):
    """Mirror of ``tq_dequant_desc`` in include/tq.h."""
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("n", ctypes.c_int64),
                ("k", ctypes.c_int64), ("w_out", ctypes.c_void_p), ("ldo", ctypes.c_int64)]


class Nvfp4GemmDesc(ctypes.Structure):
    """Mirror of ``tq_nvfp4_gemm_desc`` in include/tq.h."""
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("tensor_scale", ctypes.c_void_p),
                ("n", ctypes.c_int64), ("k", ctypes.c_int64), ("X", ctypes.c_void_p), ("ldx", ctypes.c_int64),
                ("Y", ctypes.c_void_p), ("ldy", ctypes.c_int64)]


TQ_NVFP4_TENSOR_BYTES = 16

_lock = threading.Lock()
_lib = None


class TQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)}")


def load_library() -> ctypes.CDLL:
    """Load libtq.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libtq.so not built ({LIB_PATH}); run dequant_gemv_tq4_b200/build.py")
        lib = ctypes.CDLL(LIB_PATH)
        P, I64, SZ, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_size_t, ctypes.c_int
        sig = {
            "tq_status_string": ([I], ctypes.c_char_p),
            "tq_codes_bytes": ([I64, I64], SZ),
            "tq_scales_bytes": ([I64, I64], SZ),
            "tq_xrot_bytes": ([I64, I64], SZ),
            "tq_gemm_workspace_bytes": ([I64, I64, I64], SZ),
            "tq_quantize": ([P, I, I64, I64, I64, P, P, P], I),
            "tq_dequantize": ([P, P, I64, I64, P, I, I64, P], I),
            "tq_dequantize_batch": ([ctypes.POINTER(DequantDesc), I, I, P], I),
            "tq_prerotate": ([P, I, I64, I64, I64, P, P], I),
            "tq_gemm": ([P, P, I64, I64, P, I, I64, I64, P, I, I64, P, SZ, P], I),
            "tq_gemv": ([P, P, I64, I64, P, I, P, I, P, SZ, P], I),
            "tq_gemm_xrot": ([P, P, I64, I64, P, I64, P, I, I64, P, SZ, P], I),
            "tq_gemm_batch_workspace_bytes": ([ctypes.POINTER(GemmDesc), I, I64], SZ),
            "tq_gemm_batch": ([ctypes.POINTER(GemmDesc), I, I64, I, I, P, SZ, P], I),
            "tq_workspace_status": ([P, I, P], I),
            "tq_debug_set_flags": ([ctypes.c_uint32], None),
            "tq_gemv_static_scratch": ([P, P, I64, I64, P, I, P, I, P], I),
            "tq_static_scratch_status": ([I, P], I),
            "tq_gemm_prefill_workspace_bytes": ([I64, I64], SZ),
            "tq_gemm_prefill": ([P, P, I64, I64, P, I, I64, I64, P, I, I64, P, SZ, P], I),
            "tq_prefill_xrot_bytes": ([I64, I64], SZ),
            "tq_prerotate_plain": ([P, I, I64, I64, I64, P, P], I),
            "tq_gemm_prefill_xrot": ([P, P, I64, I64, P, I64, P, I, I64, P, SZ, P], I),
            "tq_nvfp4_scales_bytes": ([I64, I64], SZ),
            "tq_nvfp4_quantize": ([P, I, I64, I64, I64, P, P, P, P], I),
            "tq_nvfp4_dequantize": ([P, P, P, I64, I64, P, I, I64, P], I),
            "tq_nvfp4_gemm": ([P, P, P, I64, I64, P, I, I64, I64, P, I, I64, P, SZ, P], I),
            "tq_nvfp4_gemm_batch_workspace_bytes": ([ctypes.POINTER(Nvfp4GemmDesc), I, I64], SZ),
            "tq_nvfp4_gemm_batch": ([ctypes.POINTER(Nvfp4GemmDesc), I, I64, I, I, P, SZ, P], I),
        }
        for name, (args, res) in sig.items():
            fn = getattr(lib, name)
            fn.argtypes = args
            fn.restype = res
        _lib = lib
        return lib


def _check(status: int, where: str) -> None:
    if status != 0:
        raise TQError(status, where)


# ---------------------------------------------------------------------------
# raw C-ABI layer (integer pointers)
# ---------------------------------------------------------------------------
def status_string(status: int) -> str:
    return load_library().tq_status_string(int(status)).decode()


def tq_codes_bytes(n: int, k: int) -> int:
    return int(load_library().tq_codes_bytes(n, k))


def tq_scales_bytes(n: int, k: int) -> int:
    return int(load_library().tq_scales_bytes(n, k))


def tq_xrot_bytes(m: int, k: int) -> int:
    return int(load_library().tq_xrot_bytes(m, k))


def tq_gemm_workspace_bytes(m: int, n: int, k: int) -> int:
    return int(load_library().tq_gemm_workspace_bytes(m, n, k))


def tq_quantize(w, wt, n, k, ldw, codes, scales, stream) -> int:
    return load_library().tq_quantize(w, wt, n, k, ldw, codes, scales, stream)


def tq_dequantize(codes, scales, n, k, w_out, ot, ldo, stream) -> int:
    return load_library().tq_dequantize(codes, scales, n, k, w_out, ot, ldo, stream)


def tq_dequantize_batch(descs, count, ot, stream) -> int:
    return load_library().tq_dequantize_batch(descs, count, ot, stream)


def tq_prerotate(X, xt, m, k, ldx, xrot, stream) -> int:
    return load_library().tq_prerotate(X, xt, m, k, ldx, xrot, stream)


def tq_gemm(codes, scales, n, k, X, xt, m, ldx, Y, yt, ldy, workspace, ws_bytes, stream) -> int:
    return load_library().tq_gemm(codes, scales, n, k, X, xt, m, ldx, Y, yt, ldy, workspace, ws_bytes, stream)


def tq_gemv(codes, scales, n, k, x, xt, y, yt, workspace, ws_bytes, stream) -> int:
    return load_library().tq_gemv(codes, scales, n, k, x, xt, y, yt, workspace, ws_bytes, stream)


def tq_gemm_xrot(codes, scales, n, k, xrot, m, Y, yt, ldy, workspace, ws_bytes, stream) -> int:
    return load_library().tq_gemm_xrot(codes, scales, n, k, xrot, m, Y, yt, ldy, workspace, ws_bytes, stream)


def tq_gemm_batch_workspace_bytes(descs, count, m) -> int:
    return int(load_library().tq_gemm_batch_workspace_bytes(descs, count, m))


def tq_gemm_batch(descs, count, m, xt, yt, workspace, ws_bytes, stream) -> int:
    return load_library().tq_gemm_batch(descs, count, m, xt, yt, workspace, ws_bytes, stream)


def tq_workspace_status(workspace, clear, stream) -> int:
    return load_library().tq_workspace_status(workspace, clear, stream)


def tq_debug_set_flags(flags: int) -> None:
    load_library().tq_debug_set_flags(flags)


def tq_gemv_static_scratch(codes, scales, n, k, x, xt, y, yt, stream) -> int:
    """GEMV without a workspace argument, for callers that cannot allocate
    device memory: the scratch is a fixed array inside the library (see
    include/tq.h).  Calls that overlap on the GPU must not share it."""
    return load_library().tq_gemv_static_scratch(codes, scales, n, k, x, xt, y, yt, stream)


def tq_static_scratch_status(clear, stream) -> int:
    """Timeout flag of the last tq_gemv_static_scratch call (synchronises)."""
    return load_library().tq_static_scratch_status(clear, stream)


def tq_gemm_prefill_workspace_bytes(m: int, k: int) -> int:
    return int(load_library().tq_gemm_prefill_workspace_bytes(m, k))


def tq_prefill_xrot_bytes(m: int, k: int) -> int:
    return int(load_library().tq_prefill_xrot_bytes(m, k))


def tq_prerotate_plain(X, xt, m, k, ldx, xrot, stream) -> int:
    return load_library().tq_prerotate_plain(X, xt, m, k, ldx, xrot, stream)


def tq_gemm_prefill_xrot(codes, scales, n, k, xrot, m, Y, yt, ldy, workspace, ws_bytes, stream) -> int:
    return load_library().tq_gemm_prefill_xrot(codes, scales, n, k, xrot, m, Y, yt, ldy, workspace, ws_bytes, stream)


def tq_gemm_prefill(codes, scales, n, k, X, xt, m, ldx, Y, yt, ldy, workspace, ws_bytes, stream) -> int:
    return load_library().tq_gemm_prefill(codes, scales, n, k, X, xt, m, ldx, Y, yt, ldy, workspace, ws_bytes,
                                          stream)


def tq_nvfp4_scales_bytes(n: int, k: int) -> int:
    return int(load_library().tq_nvfp4_scales_bytes(n, k))


def tq_nvfp4_quantize(w, wt, n, k, ldw, codes, scales, tensor_scale, stream) -> int:
    return load_library().tq_nvfp4_quantize(w, wt, n, k, ldw, codes, scales, tensor_scale, stream)


def tq_nvfp4_dequantize(codes, scales, tensor_scale, n, k, w_out, ot, ldo, stream) -> int:
    return load_library().tq_nvfp4_dequantize(codes, scales, tensor_scale, n, k, w_out, ot, ldo, stream)


def tq_nvfp4_gemm(codes, scales, tensor_scale, n, k, X, xt, m, ldx, Y, yt, ldy, workspace, ws_bytes, stream) -> int:
    return load_library().tq_nvfp4_gemm(codes, scales, tensor_scale, n, k, X, xt, m, ldx, Y, yt, ldy, workspace,
                                        ws_bytes, stream)


def tq_nvfp4_gemm_batch_workspace_bytes(descs, count, m) -> int:
    return int(load_library().tq_nvfp4_gemm_batch_workspace_bytes(descs, count, m))


def tq_nvfp4_gemm_batch(descs, count, m, xt, yt, workspace, ws_bytes, stream) -> int:
    return load_library().tq_nvfp4_gemm_batch(descs, count, m, xt, yt, workspace, ws_bytes, stream)


# ---------------------------------------------------------------------------
# tensor helpers
# ---------------------------------------------------------------------------
def _stream(stream=None) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return int(s.cuda_stream)


def _dt(t: torch.dtype) -> int:
    if t not in _DTYPE_CODE:
        raise TypeError(f"unsupported dtype {t}")
    return _DTYPE_CODE[t]


def superblocks(k: int) -> int:
    return (k // 32 + 3) // 4


def _ld(t: torch.Tensor) -> int:
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError("expected a 2-D tensor with unit column stride")
    return t.stride(0)


def workspace(m: int, n: int, k: int, device=None) -> torch.Tensor:
    """A workspace tensor for gemm/gemv/gemm_xrot of these sizes (zero-filled)."""
    nbytes = tq_gemm_workspace_bytes(m, n, k)
    if nbytes == 0:
        raise ValueError("invalid sizes for workspace query")
    return torch.zeros(nbytes, dtype=torch.uint8, device=device or torch.cuda.current_device())


def tiles(n: int) -> int:
    return (n + 15) // 16


def quantize(w: torch.Tensor, codes: torch.Tensor | None = None, scales: torch.Tensor | None = None,
             stream=None):
    """Encode W (n x k, fp32/bf16/fp16, on the GPU).  Returns the packed planes
    (codes uint8 [T*NSB*1024], scales int16 [T*NSB*128] holding fp16 bit
    patterns), T = ceil(n/16), in the tile-major layout of include/tq.h."""
    n, k = w.shape
    if codes is None:
        codes = torch.empty(tq_codes_bytes(n, k), dtype=torch.uint8, device=w.device)
    if scales is None:
        scales = torch.empty(tq_scales_bytes(n, k) // 2, dtype=torch.int16, device=w.device)
    _check(tq_quantize(w.data_ptr(), _dt(w.dtype), n, k, _ld(w), codes.data_ptr(), scales.data_ptr(),
                       _stream(stream)), "tq_quantize")
    return codes, scales


def dequantize(codes: torch.Tensor, scales: torch.Tensor, n: int, k: int, dtype=torch.bfloat16,
               out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty((n, k), dtype=dtype, device=codes.device)
    _check(tq_dequantize(codes.data_ptr(), scales.data_ptr(), n, k, out.data_ptr(), _dt(out.dtype), _ld(out),
                         _stream(stream)), "tq_dequantize")
    return out


def dequant_descs(items):
    """items: sequence of (codes, scales, n, k, out [n, k]) -> ctypes array."""
    arr = (DequantDesc * len(items))()
    for i, (codes, scales, n, k, out) in enumerate(items):
        arr[i] = DequantDesc(codes.data_ptr(), scales.data_ptr(), n, k, out.data_ptr(), _ld(out))
    return arr


def dequantize_batch(items, stream=None, descs=None):
    """Dequantise every (codes, scales, n, k, out) in one launch (outputs of one dtype)."""
    dts = {it[4].dtype for it in items}
    if len(dts) != 1:
        raise ValueError("dequantize_batch: every output needs the same dtype")
    if descs is None:
        descs = dequant_descs(items)
    _check(tq_dequantize_batch(descs, len(items), _dt(dts.pop()), _stream(stream)), "tq_dequantize_batch")


def prerotate(X: torch.Tensor, xrot: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    X2 = X.view(1, -1) if X.dim() == 1 else X
    m, k = X2.shape
    if xrot is None:
        xrot = torch.empty(tq_xrot_bytes(m, k) // 2, dtype=torch.int16, device=X.device)
    _check(tq_prerotate(X2.data_ptr(), _dt(X2.dtype), m, k, _ld(X2), xrot.data_ptr(), _stream(stream)),
           "tq_prerotate")
    return xrot


def gemm(codes, scales, n: int, k: int, X: torch.Tensor, dtype=torch.float32, out=None, ws=None,
         stream=None) -> torch.Tensor:
    """Y[m, n] = X[m, k] @ w~[n, k]^T (w~ = the dequantised weights), fused."""
    X2 = X.view(1, -1) if X.dim() == 1 else X
    m = X2.shape[0]
    if out is None:
        out = torch.empty((m, n), dtype=dtype, device=X.device)
    if ws is None:
        ws = workspace(m, n, k, X.device)
    _check(tq_gemm(codes.data_ptr(), scales.data_ptr(), n, k, X2.data_ptr(), _dt(X2.dtype), m, _ld(X2),
                   out.data_ptr(), _dt(out.dtype), _ld(out), ws.data_ptr(), ws.numel(), _stream(stream)),
           "tq_gemm")
    return out


def prefill_workspace(m: int, k: int, device=None) -> torch.Tensor:
    nbytes = tq_gemm_prefill_workspace_bytes(m, k)
    if nbytes == 0:
        raise ValueError("invalid sizes for workspace query")
    return torch.zeros(nbytes, dtype=torch.uint8, device=device or torch.cuda.current_device())


def gemm_prefill(codes, scales, n: int, k: int, X: torch.Tensor, dtype=torch.float32, out=None, ws=None,
                 stream=None) -> torch.Tensor:
    """Y[m, n] = X[m, k] @ w~[n, k]^T on the tensor-core prefill path (any m)."""
    X2 = X.view(1, -1) if X.dim() == 1 else X
    m = X2.shape[0]
    if out is None:
        out = torch.empty((m, n), dtype=dtype, device=X.device)
    if ws is None:
        ws = prefill_workspace(m, k, X.device)
    _check(tq_gemm_prefill(codes.data_ptr(), scales.data_ptr(), n, k, X2.data_ptr(), _dt(X2.dtype), m, _ld(X2),
                           out.data_ptr(), _dt(out.dtype), _ld(out), ws.data_ptr(), ws.numel(), _stream(stream)),
           "tq_gemm_prefill")
    return out


def prerotate_plain(X: torch.Tensor, out=None, stream=None) -> torch.Tensor:
    """Plain row-major fp16 pre-rotation of X (m x k) for the prefill product."""
    X2 = X.view(1, -1) if X.dim() == 1 else X
    m, k = X2.shape
    if out is None:
        out = torch.empty((m, k), dtype=torch.float16, device=X.device)
    _check(tq_prerotate_plain(X2.data_ptr(), _dt(X2.dtype), m, k, _ld(X2), out.data_ptr(), _stream(stream)),
           "tq_prerotate_plain")
    return out


def gemm_prefill_xrot(codes, scales, n: int, k: int, xrot: torch.Tensor, dtype=torch.float32, out=None, ws=None,
                      stream=None) -> torch.Tensor:
    """The tensor-core product over an activation from ``prerotate_plain``."""
    m = xrot.shape[0]
    if out is None:
        out = torch.empty((m, n), dtype=dtype, device=xrot.device)
    if ws is None:
        ws = torch.zeros(256, dtype=torch.uint8, device=xrot.device)
    _check(tq_gemm_prefill_xrot(codes.data_ptr(), scales.data_ptr(), n, k, xrot.data_ptr(), m, out.data_ptr(),
                                _dt(out.dtype), _ld(out), ws.data_ptr(), ws.numel(), _stream(stream)),
           "tq_gemm_prefill_xrot")
    return out


def gemv(codes, scales, n: int, k: int, x: torch.Tensor, dtype=torch.float32, out=None, ws=None,
         stream=None) -> torch.Tensor:
    """y[n] = w~[n, k] @ x[k], fused (m = 1)."""
    if out is None:
        out = torch.empty((n,), dtype=dtype, device=x.device)
    if ws is None:
        ws = workspace(1, n, k, x.device)
    _check(tq_gemv(codes.data_ptr(), scales.data_ptr(), n, k, x.data_ptr(), _dt(x.dtype), out.data_ptr(),
                   _dt(out.dtype), ws.data_ptr(), ws.numel(), _stream(stream)), "tq_gemv")
    return out


def gemm_xrot(codes, scales, n: int, k: int, xrot: torch.Tensor, m: int, dtype=torch.float32, out=None,
              ws=None, stream=None) -> torch.Tensor:
    """The fused product with an activation pre-rotated by ``prerotate`` (m <= 32)."""
    if out is None:
        out = torch.empty((m, n), dtype=dtype, device=xrot.device)
    if ws is None:
        ws = workspace(m, n, k, xrot.device)
    _check(tq_gemm_xrot(codes.data_ptr(), scales.data_ptr(), n, k, xrot.data_ptr(), m, out.data_ptr(),
                        _dt(out.dtype), _ld(out), ws.data_ptr(), ws.numel(), _stream(stream)), "tq_gemm_xrot")
    return out


def batch_descs(items):
    """items: sequence of (codes, scales, n, k, X [m, k], Y [m, n]) -> ctypes array."""
    arr = (GemmDesc * len(items))()
    for i, (codes, scales, n, k, X, Y) in enumerate(items):
        X2 = X.view(1, -1) if X.dim() == 1 else X
        Y2 = Y.view(1, -1) if Y.dim() == 1 else Y
        arr[i] = GemmDesc(codes.data_ptr(), scales.data_ptr(), n, k, X2.data_ptr(), _ld(X2), Y2.data_ptr(), _ld(Y2))
    return arr


def batch_workspace(items, m: int, device=None) -> torch.Tensor:
    descs = batch_descs(items)
    nbytes = tq_gemm_batch_workspace_bytes(descs, len(items), m)
    if nbytes == 0:
        raise ValueError("invalid batch for workspace query")
    return torch.zeros(nbytes, dtype=torch.uint8, device=device or torch.cuda.current_device())


def gemm_batch(items, m: int = 1, ws=None, stream=None, descs=None):
    """Fused products for several matrices in two launches (one pre-rotation
    per distinct input, one product launch).  items as in ``batch_descs``;
    the outputs Y are written in place.  All X share one dtype, all Y too."""
    if descs is None:
        descs = batch_descs(items)
    X0, Y0 = items[0][4], items[0][5]
    if ws is None:
        ws = batch_workspace(items, m, X0.device)
    _check(tq_gemm_batch(descs, len(items), m, _dt(X0.dtype), _dt(Y0.dtype), ws.data_ptr(), ws.numel(),
                         _stream(stream)), "tq_gemm_batch")
    return [it[5] for it in items]


def workspace_status(ws: torch.Tensor, clear: bool = True, stream=None) -> int:
    """0 (TQ_OK) or 8 (TQ_ERR_TIMEOUT) for the last product that used ``ws``."""
    return tq_workspace_status(ws.data_ptr(), 1 if clear else 0, _stream(stream))


# ---------------------------------------------------------------------------
# NVFP4 comparison codec (tensor helpers)
# ---------------------------------------------------------------------------
def nvfp4_quantize(w: torch.Tensor, stream=None):
    """Encode W (n x k) as NVFP4.  Returns (codes uint8 [tq_codes_bytes],
    scales uint8 [tq_nvfp4_scales_bytes] of E4M3 bytes, tensor block float32[4]
    holding g at [0] and amax|W| at [1])."""
    n, k = w.shape
    codes = torch.empty(tq_codes_bytes(n, k), dtype=torch.uint8, device=w.device)
    scales = torch.empty(tq_nvfp4_scales_bytes(n, k), dtype=torch.uint8, device=w.device)
    tensor = torch.empty(TQ_NVFP4_TENSOR_BYTES // 4, dtype=torch.float32, device=w.device)
    _check(tq_nvfp4_quantize(w.data_ptr(), _dt(w.dtype), n, k, _ld(w), codes.data_ptr(), scales.data_ptr(),
                             tensor.data_ptr(), _stream(stream)), "tq_nvfp4_quantize")
    return codes, scales, tensor


def nvfp4_dequantize(codes, scales, tensor, n: int, k: int, dtype=torch.bfloat16, out=None,
                     stream=None) -> torch.Tensor:
    if out is None:
        out = torch.empty((n, k), dtype=dtype, device=codes.device)
    _check(tq_nvfp4_dequantize(codes.data_ptr(), scales.data_ptr(), tensor.data_ptr(), n, k, out.data_ptr(),
                               _dt(out.dtype), _ld(out), _stream(stream)), "tq_nvfp4_dequantize")
    return out


def nvfp4_gemm(codes, scales, tensor, n: int, k: int, X: torch.Tensor, dtype=torch.float32, out=None, ws=None,
               stream=None) -> torch.Tensor:
    """Y[m, n] = X[m, k] @ w~[n, k]^T for NVFP4 weights (m <= 32), fused."""
    X2 = X.view(1, -1) if X.dim() == 1 else X
    m = X2.shape[0]
    if out is None:
        out = torch.empty((m, n), dtype=dtype, device=X.device)
    if ws is None:
        ws = workspace(m, n, k, X.device)
    _check(tq_nvfp4_gemm(codes.data_ptr(), scales.data_ptr(), tensor.data_ptr(), n, k, X2.data_ptr(),
                         _dt(X2.dtype), m, _ld(X2), out.data_ptr(), _dt(out.dtype), _ld(out), ws.data_ptr(),
                         ws.numel(), _stream(stream)), "tq_nvfp4_gemm")
    return out


def nvfp4_batch_descs(items):
    """items: sequence of (codes, scales, tensor, n, k, X [m, k], Y [m, n])."""
    arr = (Nvfp4GemmDesc * len(items))()
    for i, (codes, scales, tensor, n, k, X, Y) in enumerate(items):
        X2 = X.view(1, -1) if X.dim() == 1 else X
        Y2 = Y.view(1, -1) if Y.dim() == 1 else Y
        arr[i] = Nvfp4GemmDesc(codes.data_ptr(), scales.data_ptr(), tensor.data_ptr(), n, k, X2.data_ptr(),
                               _ld(X2), Y2.data_ptr(), _ld(Y2))
    return arr


def nvfp4_batch_workspace(items, m: int, device=None) -> torch.Tensor:
    descs = nvfp4_batch_descs(items)
    nbytes = tq_nvfp4_gemm_batch_workspace_bytes(descs, len(items), m)
    if nbytes == 0:
        raise ValueError("invalid batch for workspace query")
    return torch.zeros(nbytes, dtype=torch.uint8, device=device or torch.cuda.current_device())


def nvfp4_gemm_batch(items, m: int = 1, ws=None, stream=None, descs=None):
    """NVFP4 products for several matrices in two launches; outputs in place."""
    if descs is None:
        descs = nvfp4_batch_descs(items)
    X0, Y0 = items[0][5], items[0][6]
    if ws is None:
        ws = nvfp4_batch_workspace(items, m, X0.device)
    _check(tq_nvfp4_gemm_batch(descs, len(items), m, _dt(X0.dtype), _dt(Y0.dtype), ws.data_ptr(), ws.numel(),
                               _stream(stream)), "tq_nvfp4_gemm_batch")
    return [it[6] for it in items]

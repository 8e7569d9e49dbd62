"""CPU oracle for the TQ4_1S codec and its dequant-GEMV (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package.  The product library never loads it, and it
imports nothing from the product package: the two share no code, table or
constant generator.  Inputs come from the caller (the seeded generators live
in their own module).

The arithmetic lives in ``tq_oracle.c`` (plain single-threaded C, fp32 where
the codec fixes fp32, fp64 elsewhere); this module compiles it with gcc and
marshals numpy arrays through ctypes.  Every function cites, in the C source,
the passage of the TQ4_1S page (title "企业官网建设流程全解析",
hotelren.com/news/5458160, paragraph 格式原理 and section 解码速度) it follows.

Parity status: every function here is pinned by ``tests/test_oracle_*.py``
against closed forms, library routines, brute force or values the pages print.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tq_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

GCC_FLAGS = ["-O2", "-std=c99", "-D_GNU_SOURCE", "-ffp-contract=off", "-fno-fast-math",
             "-fPIC", "-shared", "-Wall", "-Wextra"]


def build(force: bool = False) -> str:
    """Compile ``tq_oracle.c`` into ``liboracle.so`` next to it (gcc)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".{os.getpid()}.tmp"
        subprocess.run(["gcc", *GCC_FLAGS, "-o", tmp, _SRC, "-lm"], check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            I64 = ctypes.c_int64
            lib.tqo_lloyd.argtypes = [ctypes.c_int, ctypes.c_int, P, P, P]
            lib.tqo_lloyd.restype = ctypes.c_int
            lib.tqo_codebook.argtypes = [P, P, P]
            lib.tqo_codebook.restype = ctypes.c_int
            lib.tqo_sign_hash.argtypes = [ctypes.c_uint32]
            lib.tqo_sign_hash.restype = ctypes.c_uint32
            lib.tqo_sign.argtypes = [ctypes.c_uint32]
            lib.tqo_sign.restype = ctypes.c_int
            lib.tqo_fwht32_f32.argtypes = [P]
            lib.tqo_fwht32_f64.argtypes = [P]
            lib.tqo_f32_to_f16.argtypes = [ctypes.c_float]
            lib.tqo_f32_to_f16.restype = ctypes.c_uint16
            lib.tqo_f16_to_f32.argtypes = [ctypes.c_uint16]
            lib.tqo_f16_to_f32.restype = ctypes.c_float
            lib.tqo_quantize_block.argtypes = [P, ctypes.c_uint32, P, P, P]
            lib.tqo_superblocks.argtypes = [I64]
            lib.tqo_superblocks.restype = I64
            lib.tqo_tiles.argtypes = [I64]
            lib.tqo_tiles.restype = I64
            lib.tqo_quantize.argtypes = [P, I64, I64, I64, P, P]
            lib.tqo_quantize.restype = ctypes.c_int
            lib.tqo_unpack.argtypes = [P, P, I64, I64, P, P]
            lib.tqo_dequantize.argtypes = [P, P, I64, I64, P, I64]
            lib.tqo_gemm.argtypes = [P, P, I64, I64, P, I64, I64, P, I64]
            lib.tqo_e4m3_to_f32.argtypes = [ctypes.c_uint8]
            lib.tqo_e4m3_to_f32.restype = ctypes.c_float
            lib.tqo_e4m3_from_f32.argtypes = [ctypes.c_float]
            lib.tqo_e4m3_from_f32.restype = ctypes.c_uint8
            lib.tqo_e2m1_to_f32.argtypes = [ctypes.c_uint8]
            lib.tqo_e2m1_to_f32.restype = ctypes.c_float
            lib.tqo_e2m1_from_f32.argtypes = [ctypes.c_float]
            lib.tqo_e2m1_from_f32.restype = ctypes.c_uint8
            lib.tqo_nvfp4_quantize.argtypes = [P, I64, I64, I64, P, P, P]
            lib.tqo_nvfp4_quantize.restype = ctypes.c_int
            lib.tqo_nvfp4_dequantize.argtypes = [P, P, ctypes.c_float, I64, I64, P, I64]
            lib.tqo_nvfp4_gemm.argtypes = [P, P, ctypes.c_float, I64, I64, P, I64, I64, P, I64]
            _lib = lib
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


# --------------------------------------------------------------------------
# codebook
# --------------------------------------------------------------------------
def lloyd(levels: int, max_iter: int = 1_000_000):
    """Lloyd-Max quantiser of N(0,1): (centroids fp64 ascending, mse, iterations)."""
    lib = _load()
    c = np.zeros(levels, np.float64)
    mse = ctypes.c_double()
    it = ctypes.c_int()
    rc = lib.tqo_lloyd(levels, max_iter, _ptr(c), ctypes.addressof(mse), ctypes.addressof(it))
    if rc == 2:
        raise ValueError("levels out of range")
    return c, mse.value, it.value


def codebook():
    """(M32 float32[8] magnitudes, B32 float32[7] thresholds, M64 float64[8])."""
    lib = _load()
    M32 = np.zeros(8, np.float32)
    B32 = np.zeros(7, np.float32)
    M64 = np.zeros(8, np.float64)
    lib.tqo_codebook(_ptr(M32), _ptr(B32), _ptr(M64))
    return M32, B32, M64


# --------------------------------------------------------------------------
# elementwise helpers
# --------------------------------------------------------------------------
def sign_hash(k) -> np.ndarray:
    lib = _load()
    k = np.asarray(k, dtype=np.uint64).ravel()
    return np.array([lib.tqo_sign_hash(int(v)) for v in k], dtype=np.uint32)


def sign(k) -> np.ndarray:
    """+1/-1 sign of global column index k (int8 array)."""
    lib = _load()
    k = np.asarray(k, dtype=np.uint64).ravel()
    return np.array([lib.tqo_sign(int(v)) for v in k], dtype=np.int8)


def fwht32(v: np.ndarray) -> np.ndarray:
    """Fast WHT of each row of a (..., 32) array, in the array's precision (f32/f64)."""
    lib = _load()
    a = np.array(v, copy=True, order="C")
    if a.shape[-1] != 32 or a.dtype not in (np.float32, np.float64):
        raise ValueError("need (..., 32) float32 or float64")
    fn = lib.tqo_fwht32_f32 if a.dtype == np.float32 else lib.tqo_fwht32_f64
    flat = a.reshape(-1, 32)
    for i in range(flat.shape[0]):
        fn(flat[i].ctypes.data)
    return a


def f32_to_f16_bits(x) -> np.ndarray:
    lib = _load()
    x = np.asarray(x, dtype=np.float32).ravel()
    return np.array([lib.tqo_f32_to_f16(float(v)) for v in x], dtype=np.uint16)


def f16_bits_to_f32(h) -> np.ndarray:
    lib = _load()
    h = np.asarray(h, dtype=np.uint16).ravel()
    return np.array([lib.tqo_f16_to_f32(int(v)) for v in h], dtype=np.float32)


# --------------------------------------------------------------------------
# codec
# --------------------------------------------------------------------------
def superblocks(k: int) -> int:
    return int(_load().tqo_superblocks(int(k)))


def tiles(n: int) -> int:
    return int(_load().tqo_tiles(int(n)))


def codes_bytes(n: int, k: int) -> int:
    return tiles(n) * superblocks(k) * 1024


def scales_count(n: int, k: int) -> int:
    return tiles(n) * superblocks(k) * 128


def row_view(codes: np.ndarray, scales: np.ndarray, n: int, k: int):
    """Row-major views of the tiled planes: (codes [n, NSB*64], scales [n, NSB*8]).
    Pure re-indexing of the stored bytes (no arithmetic)."""
    T, nsb = tiles(n), superblocks(k)
    c = np.asarray(codes).reshape(T, nsb, 16, 64).transpose(0, 2, 1, 3).reshape(T * 16, nsb * 64)[:n]
    s = np.asarray(scales).reshape(T, nsb, 16, 8).transpose(0, 2, 1, 3).reshape(T * 16, nsb * 8)[:n]
    return c, s


def quantize_block(w32: np.ndarray, k0: int):
    """One block: (logical codes uint8[32], scale bits uint16[2])."""
    lib = _load()
    w = np.ascontiguousarray(w32, dtype=np.float32)
    assert w.shape == (32,)
    _, B32, _ = codebook()
    code = np.zeros(32, np.uint8)
    d = np.zeros(2, np.uint16)
    lib.tqo_quantize_block(_ptr(w), int(k0), _ptr(B32), _ptr(code), _ptr(d))
    return code, d


def quantize(W: np.ndarray):
    """W: float32 [n, k] (k % 32 == 0).  Returns the tiled planes
    (codes uint8 [T*NSB*1024], scales uint16 [T*NSB*128]), T = ceil(n/16)."""
    lib = _load()
    W = np.ascontiguousarray(W, dtype=np.float32)
    n, k = W.shape
    if k % 32 != 0:
        raise ValueError("k must be a multiple of 32")
    codes = np.zeros(codes_bytes(n, k), np.uint8)
    scales = np.zeros(scales_count(n, k), np.uint16)
    if lib.tqo_quantize(_ptr(W), n, k, k, _ptr(codes), _ptr(scales)) != 0:
        raise ValueError("k must be a multiple of 32")
    return codes, scales


def unpack(codes: np.ndarray, scales: np.ndarray, n: int, k: int):
    """Logical view: (codes uint8 [n, k], scale bits uint16 [n, k/32, 2])."""
    lib = _load()
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    code = np.zeros((n, k), np.uint8)
    d = np.zeros((n, k // 32, 2), np.uint16)
    lib.tqo_unpack(_ptr(codes), _ptr(scales), n, k, _ptr(code), _ptr(d))
    return code, d


def dequantize(codes: np.ndarray, scales: np.ndarray, n: int, k: int) -> np.ndarray:
    """fp64 [n, k] reconstruction."""
    lib = _load()
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    W = np.zeros((n, k), np.float64)
    lib.tqo_dequantize(_ptr(codes), _ptr(scales), n, k, _ptr(W), k)
    return W


def gemm(codes: np.ndarray, scales: np.ndarray, n: int, k: int, X: np.ndarray) -> np.ndarray:
    """fp64 Y[m, n] = sum_k w~[n, k] * X[m, k]  (X any float dtype, converted to fp64)."""
    lib = _load()
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    X = np.ascontiguousarray(np.atleast_2d(X), dtype=np.float64)
    m = X.shape[0]
    Y = np.zeros((m, n), np.float64)
    lib.tqo_gemm(_ptr(codes), _ptr(scales), n, k, _ptr(X), m, k, _ptr(Y), n)
    return Y


# --------------------------------------------------------------------------
# NVFP4 comparison codec
# --------------------------------------------------------------------------
def e4m3_to_f32(c) -> np.ndarray:
    lib = _load()
    return np.array([lib.tqo_e4m3_to_f32(int(v)) for v in np.asarray(c, np.uint8).ravel()], np.float32)


def e4m3_from_f32(x) -> np.ndarray:
    lib = _load()
    return np.array([lib.tqo_e4m3_from_f32(float(v)) for v in np.asarray(x, np.float32).ravel()], np.uint8)


def e2m1_to_f32(c) -> np.ndarray:
    lib = _load()
    return np.array([lib.tqo_e2m1_to_f32(int(v)) for v in np.asarray(c, np.uint8).ravel()], np.float32)


def e2m1_from_f32(x) -> np.ndarray:
    lib = _load()
    return np.array([lib.tqo_e2m1_from_f32(float(v)) for v in np.asarray(x, np.float32).ravel()], np.uint8)


def nvfp4_scales_bytes(n: int, k: int) -> int:
    return tiles(n) * superblocks(k) * 128


def nvfp4_quantize(W: np.ndarray):
    """W float32 [n, k] (k % 32 == 0) -> (codes uint8 [T*NSB*1024], scales uint8 [T*NSB*128], g float)."""
    lib = _load()
    W = np.ascontiguousarray(W, dtype=np.float32)
    n, k = W.shape
    if k % 32 != 0:
        raise ValueError("k must be a multiple of 32")
    codes = np.zeros(codes_bytes(n, k), np.uint8)
    scales = np.zeros(nvfp4_scales_bytes(n, k), np.uint8)
    g = np.zeros(1, np.float32)
    lib.tqo_nvfp4_quantize(_ptr(W), n, k, k, _ptr(codes), _ptr(scales), _ptr(g))
    return codes, scales, float(g[0])


def nvfp4_dequantize(codes, scales, g: float, n: int, k: int) -> np.ndarray:
    lib = _load()
    codes = np.ascontiguousarray(codes, np.uint8)
    scales = np.ascontiguousarray(scales, np.uint8)
    W = np.zeros((n, k), np.float64)
    lib.tqo_nvfp4_dequantize(_ptr(codes), _ptr(scales), float(g), n, k, _ptr(W), k)
    return W


def nvfp4_gemm(codes, scales, g: float, n: int, k: int, X: np.ndarray) -> np.ndarray:
    lib = _load()
    codes = np.ascontiguousarray(codes, np.uint8)
    scales = np.ascontiguousarray(scales, np.uint8)
    X = np.ascontiguousarray(np.atleast_2d(X), dtype=np.float64)
    m = X.shape[0]
    Y = np.zeros((m, n), np.float64)
    lib.tqo_nvfp4_gemm(_ptr(codes), _ptr(scales), float(g), n, k, _ptr(X), m, k, _ptr(Y), n)
    return Y

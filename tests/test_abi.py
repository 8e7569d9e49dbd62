"""C-ABI library checks that need no GPU: it loads, it exports every entry
point that include/tq.h declares, size queries, and argument validation that
returns before anything touches a device (every call below fails a host check
or is an empty problem, so no pointer is ever dereferenced)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tq.h")

OK, INVALID, SHAPE, ALIGN, DTYPE, WORKSPACE, CUDA, UNSUP, TIMEOUT = range(9)
FAKE = 1 << 20  # never dereferenced: every call using it fails validation first


@pytest.fixture(scope="module")
def lib():
    from dequant_gemv_tq4_b200 import build as b

    b.build()
    import dequant_gemv_tq4_b200 as tq

    return tq.load_library()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"TQ_API\s+[\w\s\*]*?\b(tq_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_symbols()
    for required in ("tq_quantize", "tq_dequantize", "tq_gemv", "tq_gemm", "tq_prerotate", "tq_gemm_xrot",
                     "tq_codes_bytes", "tq_scales_bytes", "tq_xrot_bytes", "tq_gemm_workspace_bytes",
                     "tq_status_string", "tq_gemm_batch", "tq_gemm_batch_workspace_bytes", "tq_workspace_status",
                     "tq_debug_set_flags"):
        assert required in names


def test_library_exports_every_declared_symbol(lib):
    from dequant_gemv_tq4_b200 import LIB_PATH

    out = subprocess.run(["nm", "-D", "--defined-only", LIB_PATH], capture_output=True, text=True, check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    for name in declared_symbols():
        assert name in exported, name
        assert getattr(lib, name) is not None
    # nothing but the declared C names is exported from the tq_ namespace
    assert {e for e in exported if e.startswith("tq_")} == set(declared_symbols())


def test_status_strings(lib):
    for code in range(9):
        s = lib.tq_status_string(code).decode()
        assert s.startswith("TQ_")
    assert lib.tq_status_string(99).decode() == "unknown tq_status"


def test_size_queries(lib):
    assert lib.tq_codes_bytes(3, 128) == 1024      # rows padded to a 16-row tile
    assert lib.tq_scales_bytes(3, 128) == 256
    assert lib.tq_codes_bytes(17, 160) == 2 * 2 * 1024  # two tiles, ragged last superblock padded
    assert lib.tq_scales_bytes(17, 160) == 2 * 2 * 256
    assert lib.tq_codes_bytes(14336, 4096) + lib.tq_scales_bytes(14336, 4096) == 14336 * 4096 * 5 // 8
    assert lib.tq_xrot_bytes(1, 4096) == 4096 * 2
    assert lib.tq_xrot_bytes(3, 96) == 3 * 128 * 2
    for bad in ((3, 100), (3, 0), (-1, 64), (3, -32)):
        assert lib.tq_codes_bytes(*bad) == 0
        assert lib.tq_scales_bytes(*bad) == 0


def test_quantize_argument_errors(lib):
    q = lib.tq_quantize
    assert q(FAKE, 0, 4, 48, 48, FAKE, FAKE, None) == SHAPE
    assert q(FAKE, 0, 4, 0, 8, FAKE, FAKE, None) == SHAPE
    assert q(FAKE, 0, -1, 64, 64, FAKE, FAKE, None) == INVALID
    assert q(FAKE, 9, 4, 64, 64, FAKE, FAKE, None) == DTYPE
    assert q(None, 0, 4, 64, 64, FAKE, FAKE, None) == INVALID
    assert q(FAKE, 0, 4, 64, 32, FAKE, FAKE, None) == INVALID        # ldw < k
    assert q(FAKE + 4, 0, 4, 64, 64, FAKE, FAKE, None) == ALIGN      # w not 16-byte aligned
    assert q(FAKE, 1, 4, 64, 68, FAKE, FAKE, None) == ALIGN          # ldw % 8 != 0
    assert q(FAKE, 0, 4, 64, 64, None, FAKE, None) == INVALID
    assert q(FAKE, 0, 4, 64, 64, FAKE, FAKE + 2, None) == ALIGN
    assert q(FAKE, 0, 0, 64, 64, FAKE, FAKE, None) == OK             # empty: nothing launched
    assert q(FAKE, 0, 1, 1 << 27, 1 << 27, FAKE, FAKE, None) == SHAPE


def test_dequantize_and_prerotate_argument_errors(lib):
    d = lib.tq_dequantize
    assert d(FAKE, FAKE, 4, 40, FAKE, 0, 40, None) == SHAPE
    assert d(FAKE, FAKE, 4, 64, FAKE, 5, 64, None) == DTYPE
    assert d(None, FAKE, 4, 64, FAKE, 0, 64, None) == INVALID
    assert d(FAKE, FAKE, 4, 64, None, 0, 64, None) == INVALID
    assert d(FAKE, FAKE, 4, 64, FAKE + 8, 0, 64, None) == ALIGN
    assert d(FAKE, FAKE, 0, 64, FAKE, 0, 64, None) == OK
    from dequant_gemv_tq4_b200 import DequantDesc
    b = lib.tq_dequantize_batch

    def descs(*rows):
        arr = (DequantDesc * len(rows))()
        for i, r in enumerate(rows):
            arr[i] = DequantDesc(*r)
        return arr

    good = (FAKE, FAKE, 4, 64, FAKE, 64)
    assert b(None, 1, 0, None) == INVALID
    assert b(descs(good), 0, 0, None) == SHAPE
    assert b(descs(*[good] * 9), 9, 0, None) == SHAPE
    assert b(descs(good), 1, 5, None) == DTYPE
    assert b(descs(good, (FAKE, FAKE, 4, 40, FAKE, 64)), 2, 0, None) == SHAPE
    assert b(descs(good, (None, FAKE, 4, 64, FAKE, 64)), 2, 0, None) == INVALID
    assert b(descs(good, (FAKE, FAKE, 4, 64, FAKE + 8, 64)), 2, 0, None) == ALIGN
    assert b(descs(good, (FAKE, FAKE, 4, 64, FAKE, 60)), 2, 0, None) == INVALID  # ldo < k
    assert b(descs((FAKE, FAKE, 0, 64, FAKE, 64), (None, None, 0, 96, None, 0)), 2, 0, None) == OK  # no rows
    p = lib.tq_prerotate
    assert p(FAKE, 0, 1, 33, 40, FAKE, None) == SHAPE
    assert p(FAKE, 3, 1, 64, 64, FAKE, None) == DTYPE
    assert p(FAKE, 0, 1, 64, 64, None, None) == INVALID
    assert p(FAKE, 0, 1, 64, 64, FAKE + 4, None) == ALIGN
    assert p(FAKE, 0, 0, 64, 64, FAKE, None) == OK


def test_gemm_argument_errors(lib):
    g = lib.tq_gemm
    assert g(FAKE, FAKE, 8, 50, FAKE, 1, 1, 64, FAKE, 0, 8, FAKE, 1 << 20, None) == SHAPE
    assert g(FAKE, FAKE, 8, 64, FAKE, 1, -1, 64, FAKE, 0, 8, FAKE, 1 << 20, None) == INVALID
    assert g(FAKE, FAKE, 8, 64, FAKE, 1, 1, 64, FAKE, 7, 8, FAKE, 1 << 20, None) == DTYPE
    assert g(None, FAKE, 8, 64, FAKE, 1, 1, 64, FAKE, 0, 8, FAKE, 1 << 20, None) == INVALID
    assert g(FAKE, FAKE, 8, 64, FAKE, 1, 1, 64, None, 0, 8, FAKE, 1 << 20, None) == INVALID
    assert g(FAKE, FAKE, 8, 64, FAKE, 1, 1, 64, FAKE, 0, 4, FAKE, 1 << 20, None) == INVALID  # ldy < n
    assert g(FAKE, FAKE, 8, 64, FAKE, 1, 1, 64, FAKE + 2, 0, 8, FAKE, 1 << 20, None) == ALIGN
    assert g(FAKE, FAKE, 8, 64, FAKE, 6, 1, 64, FAKE, 0, 8, FAKE, 1 << 20, None) == DTYPE
    assert g(FAKE, FAKE, 8, 64, FAKE + 8, 1, 1, 64, FAKE, 0, 8, FAKE, 1 << 20, None) == ALIGN
    assert g(FAKE, FAKE, 8, 64, FAKE, 1, 0, 64, FAKE, 0, 8, FAKE, 1 << 20, None) == OK
    assert g(FAKE, FAKE, 0, 64, FAKE, 1, 4, 64, FAKE, 0, 8, FAKE, 1 << 20, None) == OK
    v = lib.tq_gemv
    assert v(FAKE, FAKE, 8, 65, FAKE, 1, FAKE, 0, FAKE, 1 << 20, None) == SHAPE
    assert v(FAKE, None, 8, 64, FAKE, 1, FAKE, 0, FAKE, 1 << 20, None) == INVALID
    x = lib.tq_gemm_xrot
    assert x(FAKE, FAKE, 8, 64, FAKE, 33, FAKE, 0, 8, FAKE, 1 << 20, None) == SHAPE
    assert x(FAKE, FAKE, 8, 64, None, 2, FAKE, 0, 8, FAKE, 1 << 20, None) == INVALID
    assert x(FAKE, FAKE, 8, 64, FAKE + 2, 2, FAKE, 0, 8, FAKE, 1 << 20, None) == ALIGN


def test_batch_argument_errors(lib):
    import dequant_gemv_tq4_b200 as tq

    def descs(*specs):
        arr = (tq.GemmDesc * max(1, len(specs)))()
        for i, (codes, scales, n, k, X, ldx, Y, ldy) in enumerate(specs):
            arr[i] = tq.GemmDesc(codes, scales, n, k, X, ldx, Y, ldy)
        return arr

    good = (FAKE, FAKE, 64, 128, FAKE, 128, FAKE, 64)
    b = lib.tq_gemm_batch
    assert b(None, 1, 1, 1, 0, FAKE, 1 << 20, None) == INVALID
    assert b(descs(good), 0, 1, 1, 0, FAKE, 1 << 20, None) == SHAPE
    assert b(descs(*[good] * 9), 9, 1, 1, 0, FAKE, 1 << 20, None) == SHAPE
    assert b(descs(good), 1, 33, 1, 0, FAKE, 1 << 20, None) == SHAPE
    assert b(descs(good), 1, -1, 1, 0, FAKE, 1 << 20, None) == INVALID
    assert b(descs(good), 1, 1, 5, 0, FAKE, 1 << 20, None) == DTYPE
    assert b(descs(good, (FAKE, FAKE, 64, 100, FAKE, 128, FAKE, 64)), 2, 1, 1, 0, FAKE, 1 << 20, None) == SHAPE
    assert b(descs(good, (FAKE, FAKE, 0, 128, FAKE, 128, FAKE, 64)), 2, 1, 1, 0, FAKE, 1 << 20, None) == SHAPE
    assert b(descs((None, FAKE, 64, 128, FAKE, 128, FAKE, 64)), 1, 1, 1, 0, FAKE, 1 << 20, None) == INVALID
    assert b(descs((FAKE, FAKE, 64, 128, FAKE + 4, 128, FAKE, 64)), 1, 1, 1, 0, FAKE, 1 << 20, None) == ALIGN
    assert b(descs(good), 1, 0, 1, 0, FAKE, 1 << 20, None) == OK  # m = 0: nothing launched
    assert lib.tq_gemm_batch_workspace_bytes(None, 1, 1) == 0
    assert lib.tq_gemm_batch_workspace_bytes(descs(good), 1, 33) == 0
    assert lib.tq_workspace_status(None, 0, None) == INVALID


def test_binding_has_no_cpu_fallback(monkeypatch, tmp_path):
    import dequant_gemv_tq4_b200 as tq

    monkeypatch.setattr(tq, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(tq, "_lib", None)
    with pytest.raises(RuntimeError, match="not built"):
        tq.load_library()

"""Build libtq.so (the C-ABI library) in-tree with nvcc for sm_100a."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libtq.so")
SOURCES = ["tq_codec.cu", "tq_gemv.cu", "tq_tcgemv.cu", "tq_nvfp4.cu", "tq_prefill.cu", "tq_capi.cu"]
HEADERS = ["tq_device.cuh", "tq_internal.h", "tq_codebook.h", os.path.join("..", "..", "include", "tq.h")]

NVCC_FLAGS = [
    "-O3", "-std=c++17", "-lineinfo",
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
    "-shared", "-cudart", "static",
]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, s) for s in SOURCES + HEADERS] + [__file__]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose_ptxas: bool = False, out: str | None = None, defines=()) -> str:
    target = out or LIB
    if not force and out is None and not stale():
        return LIB
    tmp = target + f".{os.getpid()}.tmp"
    cmd = [nvcc(), *NVCC_FLAGS, *(["-Xptxas", "-v"] if verbose_ptxas else []), *[f"-D{d}" for d in defines],
           "-o", tmp, *[os.path.join(CSRC, s) for s in SOURCES]]
    subprocess.run(cmd, check=True, cwd=CSRC)
    os.replace(tmp, target)
    return target


if __name__ == "__main__":
    print(build(force=True, verbose_ptxas="-v" in sys.argv))

"""Build step: compile the CUDA sources into the in-tree shared library
``rotation_quantized_bit_b200/libconvrot_b200.so`` for sm_100a with nvcc.

Run ``python -m rotation_quantized_bit_b200.build`` (or ``build(force=True)``).
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libconvrot_b200.so")
SOURCES = ["api.cu", "rotate_quant.cu", "gemm.cu", "small_m.cu", "int8.cu", "noalloc.cu", "peak.cu"]
HEADERS = ["ptx.cuh", "kernels.cuh"]


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found: the CUDA 12.9 toolkit is needed to build libconvrot_b200.so")


def nvcc_flags(verbose_ptxas: bool = False) -> list[str]:
    flags = [
        "-gencode", "arch=compute_100a,code=sm_100a",
        "-O3", "-lineinfo", "-std=c++17", "-rdc=true",
        "-shared", "-Xcompiler", "-fPIC,-O2",
        "-I", os.path.join(ROOT, "include"),
    ]
    if verbose_ptxas:
        flags += ["-Xptxas", "-v"]
    return flags


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.join(ROOT, "include", "convrot.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose_ptxas: bool = False) -> str:
    """Compile libconvrot_b200.so if it is missing or older than its sources."""
    if not force and not _stale():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [nvcc_path(), *nvcc_flags(verbose_ptxas), "-o", tmp, *[os.path.join(CSRC, f) for f in SOURCES]]
    subprocess.check_call(cmd, cwd=CSRC)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose_ptxas="-v" in sys.argv))

"""Build libblasst.so (sm_100a) in-tree with nvcc.

    python -m block_sparse_flashattention_tcgen05_b200.build [--verbose-ptxas]
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libblasst.so")
SOURCES = ["blasst_api.cu", "decode.cu", "decode_wide.cu", "prefill.cu", "mla.cu", "decode_noalloc.cu", "backward.cu"]
HEADERS = ["ptx.cuh", "internal.h"]
INCLUDE = os.path.join(os.path.dirname(HERE), "include")


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.join(INCLUDE, h) for h in ("blasst.h", "blasst_measure.h")]
    return any(os.path.getmtime(f) > t for f in deps)


def build(force: bool = False, ptxas_verbose: bool = False) -> str:
    if not force and not _stale():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [
        _nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
        "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
        "-I", INCLUDE, "-o", tmp,
    ] + [os.path.join(CSRC, f) for f in SOURCES]
    if ptxas_verbose:
        cmd += ["-Xptxas", "-v"]
    subprocess.check_call(cmd)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force=True, ptxas_verbose="--verbose-ptxas" in sys.argv)
    print(LIB)

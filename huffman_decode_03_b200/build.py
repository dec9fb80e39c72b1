"""Builds the in-tree shared library ``libdf11_b200.so`` with nvcc (sm_100a).

The library holds the host format builder (C++) and the CUDA kernels; the
CUDA runtime is linked statically so the library loads on machines without a
GPU (host-only entry points work there) and carries no runtime-version clash
with other CUDA users in the process.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB_NAME = "libdf11_b200.so"
LIB_PATH = os.path.join(HERE, LIB_NAME)
SOURCES = [os.path.join(CSRC, "df11_decode.cu"), os.path.join(CSRC, "df11_gemm.cu"),
           os.path.join(CSRC, "df11_encode.cu"), os.path.join(CSRC, "df11_format.cpp"),
           os.path.join(CSRC, "df11_rans.cu"), os.path.join(CSRC, "df11_rans_format.cpp")]
HEADERS = [os.path.join(INCLUDE, "df11.h"), os.path.join(CSRC, "df11_block.cuh")]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.sep not in cand or os.path.exists(cand)):
            return cand
    return "nvcc"


def _stale() -> bool:
    if not os.path.exists(LIB_PATH):
        return True
    t = os.path.getmtime(LIB_PATH)
    deps = SOURCES + HEADERS
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False, extra=()) -> str:
    if not force and not _stale():
        return LIB_PATH
    tmp = LIB_PATH + f".tmp{os.getpid()}"
    cmd = [
        nvcc(), "-O3", "-std=c++17", *ARCH, "-lineinfo", "-shared",
        "-Xcompiler", "-fPIC,-pthread,-O3", "-cudart", "static",
        "-I", INCLUDE, *SOURCES, "-o", tmp, *extra,
    ]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB_PATH)
    return LIB_PATH


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose=True,
          extra=["-Xptxas", "-v"] if "--ptxas" in sys.argv else [])

"""Build libpagedattn.so in-tree with nvcc for sm_100a.

    python -m paged_kv_cache_435_b200.build [--verbose-ptxas]

The library is a plain shared object with a C ABI (include/pa.h); the CUDA
runtime is linked statically so the file loads on hosts without a GPU too.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libpagedattn.so")
SOURCES = ["pa_api.cu", "pa_decode.cu", "pa_multi_query.cu", "pa_multi_query_tc.cu",
           "pa_multi_row.cu", "pa_cache_ops.cu",
           "pa_swap.cu", "pa_static_ws.cu", "pa_block_manager.cpp"]
HEADERS = ["pa_common.cuh", "pa_decode.cuh", "pa_multi_query.cuh",
           "pa_multi_row.cuh", "pa_cascade.cuh", "pa_split.cuh", "pa_cache_ops.cuh", "pa_swap.cuh"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC,-O2",
    "-cudart", "static",
]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _inputs():
    return ([os.path.join(CSRC, s) for s in SOURCES + HEADERS] +
            [os.path.join(INCLUDE, "pa.h"), os.path.abspath(__file__)])


def is_stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(p) > t for p in _inputs())


def build(force: bool = False, ptxas_verbose: bool = False) -> str:
    if not force and not is_stale():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [_nvcc(), *NVCC_FLAGS, "-shared", "-I", INCLUDE, "-I", CSRC,
           *(os.path.join(CSRC, s) for s in SOURCES), "-o", tmp]
    if ptxas_verbose:
        cmd[1:1] = ["-Xptxas", "-v"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True, ptxas_verbose="--verbose-ptxas" in sys.argv))

"""Build libpagedattn.so in-tree with nvcc for sm_100a.

    python -m paged_kv_cache_435_b200.build [--verbose-ptxas]

The library is a plain shared object with a C ABI (include/pa.h); the CUDA
runtime is linked statically so the file loads on hosts without a GPU too.
Sources compile in parallel into _build/ and are linked once.

A second library, libpagedattn_waittest.so, is the same sources built with
PA_TEST_UNSIGNALLED_FIRST_WAIT: its decode kernel's first chunk wait polls a
barrier nothing arrives on, so the tests can watch a bounded wait run out.
It is test infrastructure; nothing but the tests loads it.
"""
from __future__ import annotations

import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libpagedattn.so")
WAITTEST_LIB = os.path.join(PKG, "libpagedattn_waittest.so")
BUILD_DIR = os.path.join(ROOT, "_build")
VARIANTS = {LIB: [], WAITTEST_LIB: ["-DPA_TEST_UNSIGNALLED_FIRST_WAIT"]}
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


def is_stale(lib: str = LIB) -> bool:
    if not os.path.exists(lib):
        return True
    t = os.path.getmtime(lib)
    return any(os.path.getmtime(p) > t for p in _inputs())


def _build_one(lib: str, defines, ptxas_verbose: bool, pool) -> None:
    tag = os.path.splitext(os.path.basename(lib))[0]
    objdir = os.path.join(BUILD_DIR, tag)
    os.makedirs(objdir, exist_ok=True)
    extra = ["-Xptxas", "-v"] if ptxas_verbose else []

    def compile_one(src):
        obj = os.path.join(objdir, os.path.splitext(src)[0] + ".o")
        subprocess.run([_nvcc(), *NVCC_FLAGS, *extra, *defines, "-c", "-I", INCLUDE,
                        "-I", CSRC, os.path.join(CSRC, src), "-o", obj], check=True)
        return obj

    objs = list(pool.map(compile_one, SOURCES))
    tmp = lib + f".tmp{os.getpid()}"
    subprocess.run([_nvcc(), *NVCC_FLAGS, "-shared", *objs, "-o", tmp], check=True)
    os.replace(tmp, lib)


def build(force: bool = False, ptxas_verbose: bool = False) -> str:
    """Build the product library and the wait-test library when stale;
    returns the product library's path."""
    todo = [lib for lib in VARIANTS if force or is_stale(lib)]
    if todo:
        with ThreadPoolExecutor(max_workers=max(1, min(16, os.cpu_count() or 1))) as pool:
            for lib in todo:
                _build_one(lib, VARIANTS[lib], ptxas_verbose and lib == LIB, pool)
    return LIB


if __name__ == "__main__":
    print(build(force=True, ptxas_verbose="--verbose-ptxas" in sys.argv))

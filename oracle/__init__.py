"""fp64 CPU oracle for paged decode attention, reshape_and_cache and copy_blocks.

TEST INFRASTRUCTURE ONLY.  The tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline / reference arm are the only callers.  The product
library (``paged_kv_cache_435_b200``) never imports this package and shares no
code with it; the one thing both sides use is the seeded input module
``paged_kv_cache_435_b200.inputs``, which holds no attention arithmetic.

The arithmetic lives in ``pa_oracle.c`` (plain C, double precision).  This file
only compiles it with gcc and marshals numpy / torch CPU arrays into it.

Pages the oracle follows (by title and section):
  * "vLLM: Anatomy and Mechanisms of High-Throughput LLM Inference":
    "Block-Level Management" (logical -> physical blocks via a block table,
    on-demand allocation, 16-token default block), "Memory Sharing via
    Copy-on-Write (CoW)" (copy only the diverging block), "Prefill vs. Decode
    Operations" (decode = one new token per sequence).
  * "Inside vLLM: Anatomy of a High-Throughput LLM Inference System":
    "LLM Engine constructor" (per-block bytes
    2 * block_size * num_kv_heads * head_size * dtype_bytes; allocate, reshape
    and bind KV cache tensors).
  * "vLLM Internals": "The Block Manager" (per-request block tables).

Readings where the pages are silent: query head h reads kv head
h // (num_heads // num_kv_heads); z = scale * q.k; context length 0 gives a zero
output; a negative slot is padding.  Every oracle function is pinned by
``tests/test_oracle.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libpa_oracle.so")
_lock = threading.Lock()
_lib = None

OK, ERR_ARG, ERR_RANGE, ERR_NOMEM = 0, -1, -2, -3


def build(force: bool = False) -> str:
    """Compile ``pa_oracle.c`` into ``libpa_oracle.so`` (plain gcc, -O2)."""
    stale = (not os.path.exists(_LIB_PATH)) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC",
               "-shared", "-pthread", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            # A test may point the binding at a deliberately mutated build of
            # pa_oracle.c to check that the pins catch the planted mistake.
            lib = ctypes.CDLL(os.environ.get("PA_ORACLE_LIB") or build())
            p, i32, i64, dbl = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64,
                                ctypes.c_double)
            lib.oracle_reshape_and_cache.argtypes = [
                p, p, i64, i64, p, p, p, i32, i32, i32, i32, i32]
            lib.oracle_reshape_and_cache.restype = i32
            lib.oracle_copy_blocks.argtypes = [
                p, p, i32, p, i32, i32, i32, i32, i32]
            lib.oracle_copy_blocks.restype = i32
            lib.oracle_paged_decode_attention.argtypes = [
                p, p, p, p, p, i32, p, i32, i32, i32, i32, i32, i32, dbl, i32]
            lib.oracle_paged_decode_attention.restype = i32
            lib.oracle_paged_multi_query_attention.argtypes = [
                p, p, p, p, p, i32, p, p, i32, i32, i32, i32, i32, i32, dbl,
                i32]
            lib.oracle_paged_multi_query_attention.restype = i32
            lib.oracle_swap_blocks.argtypes = [p, p, i32, p, i32, i64, i64, i64]
            lib.oracle_swap_blocks.restype = i32
            _lib = lib
    return _lib


def _bits16(a) -> np.ndarray:
    """A C-contiguous uint16 view of a bf16 torch tensor or a uint16 array."""
    if hasattr(a, "view") and hasattr(a, "dtype") and "bfloat16" in str(a.dtype):
        import torch
        a = a.contiguous().view(torch.int16).numpy().view(np.uint16)
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError(f"expected bf16 bits, got {a.dtype}")
    return a


def _arr(a, dtype) -> np.ndarray:
    if hasattr(a, "numpy"):
        a = a.cpu().numpy()
    a = np.ascontiguousarray(a, dtype=dtype)
    return a


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str) -> None:
    if rc != OK:
        raise ValueError(f"oracle {what} failed with status {rc}")


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def paged_decode_attention(q, k_cache, v_cache, block_tables, context_lens,
                           scale: float, num_kv_heads: int,
                           threads: int | None = None) -> np.ndarray:
    """fp64 decode attention through the block table.

    q: bf16 [B, Hq, D]; k_cache, v_cache: bf16 [NB, bs, Hkv, D];
    block_tables: int32 [B, MB]; context_lens: int32 [B].
    Returns float64 [B, Hq, D].
    """
    lib = _load()
    qb, kb, vb = _bits16(q), _bits16(k_cache), _bits16(v_cache)
    bt = _arr(block_tables, np.int32)
    cl = _arr(context_lens, np.int32)
    B, Hq, D = qb.shape
    NB, bs, Hkv, D2 = kb.shape
    if D2 != D or Hkv != num_kv_heads or vb.shape != kb.shape:
        raise ValueError("shape mismatch")
    if bt.ndim != 2 or bt.shape[0] != B or cl.shape != (B,):
        raise ValueError("block_tables / context_lens shape mismatch")
    out = np.zeros((B, Hq, D), dtype=np.float64)
    rc = lib.oracle_paged_decode_attention(
        _ptr(out), _ptr(qb), _ptr(kb), _ptr(vb), _ptr(bt), bt.shape[1],
        _ptr(cl), B, Hq, Hkv, D, bs, NB, float(scale),
        threads if threads is not None else default_threads())
    _check(rc, "paged_decode_attention")
    return out


def paged_multi_query_attention(q, k_cache, v_cache, block_tables,
                                context_lens, query_start_loc, scale: float,
                                num_kv_heads: int,
                                threads: int | None = None) -> np.ndarray:
    """fp64 causal attention of k new query tokens per sequence.

    q: bf16 [T, Hq, D] (T = query_start_loc[-1]); query_start_loc: int32
    [B+1]; the last k_s = qsl[s+1]-qsl[s] of sequence s's context_lens[s]
    tokens are its queries.  Returns float64 [T, Hq, D].
    """
    lib = _load()
    qb, kb, vb = _bits16(q), _bits16(k_cache), _bits16(v_cache)
    bt = _arr(block_tables, np.int32)
    cl = _arr(context_lens, np.int32)
    qsl = _arr(query_start_loc, np.int32)
    T, Hq, D = qb.shape
    NB, bs, Hkv, D2 = kb.shape
    B = cl.shape[0]
    if D2 != D or Hkv != num_kv_heads or vb.shape != kb.shape:
        raise ValueError("shape mismatch")
    if qsl.shape != (B + 1,) or int(qsl[-1]) != T or bt.shape[0] != B:
        raise ValueError("query_start_loc / block_tables shape mismatch")
    out = np.zeros((T, Hq, D), dtype=np.float64)
    rc = lib.oracle_paged_multi_query_attention(
        _ptr(out), _ptr(qb), _ptr(kb), _ptr(vb), _ptr(bt), bt.shape[1],
        _ptr(cl), _ptr(qsl), B, Hq, Hkv, D, bs, NB, float(scale),
        threads if threads is not None else default_threads())
    _check(rc, "paged_multi_query_attention")
    return out


def reshape_and_cache(key, value, k_cache_bits: np.ndarray,
                      v_cache_bits: np.ndarray, slot_mapping) -> None:
    """In-place scatter of new K/V rows into uint16 pool arrays.

    key, value: bf16 [T, Hkv, D] (C-contiguous); k/v_cache_bits: uint16
    [NB, bs, Hkv, D], modified in place; slot_mapping: int64 [T].
    """
    lib = _load()
    kb, vb = _bits16(key), _bits16(value)
    if not (k_cache_bits.flags.c_contiguous and v_cache_bits.flags.c_contiguous):
        raise ValueError("caches must be C-contiguous")
    sm = _arr(slot_mapping, np.int64)
    T, Hkv, D = kb.shape
    NB, bs, Hkv2, D2 = k_cache_bits.shape
    if (Hkv2, D2) != (Hkv, D):
        raise ValueError("shape mismatch")
    rc = lib.oracle_reshape_and_cache(
        _ptr(kb), _ptr(vb), Hkv * D, Hkv * D, _ptr(k_cache_bits),
        _ptr(v_cache_bits), _ptr(sm), T, NB, bs, Hkv, D)
    _check(rc, "reshape_and_cache")


def copy_blocks(k_caches_bits: list, v_caches_bits: list,
                block_mapping) -> None:
    """In-place copy-on-write block copies over every layer's uint16 pools."""
    lib = _load()
    L = len(k_caches_bits)
    if L == 0 or len(v_caches_bits) != L:
        raise ValueError("need matching, non-empty K and V layer lists")
    NB, bs, Hkv, D = k_caches_bits[0].shape
    for a in list(k_caches_bits) + list(v_caches_bits):
        if a.shape != (NB, bs, Hkv, D) or a.dtype != np.uint16 or \
                not a.flags.c_contiguous:
            raise ValueError("every layer pool must be uint16 [NB,bs,Hkv,D]")
    bm = _arr(block_mapping, np.int64).reshape(-1, 2)
    karr = (ctypes.c_void_p * L)(*[a.ctypes.data for a in k_caches_bits])
    varr = (ctypes.c_void_p * L)(*[a.ctypes.data for a in v_caches_bits])
    rc = lib.oracle_copy_blocks(ctypes.cast(karr, ctypes.c_void_p),
                                ctypes.cast(varr, ctypes.c_void_p), L,
                                _ptr(bm), bm.shape[0], NB, bs, Hkv, D)
    _check(rc, "copy_blocks")


def swap_blocks(src_caches: list, dst_caches: list, block_mapping) -> None:
    """In-place whole-block copies src_caches[c][src] -> dst_caches[c][dst]
    for each (src, dst) pair; each cache a C-contiguous array whose first
    dimension is the block index (pools may differ in block count)."""
    lib = _load()
    n = len(src_caches)
    if n == 0 or len(dst_caches) != n:
        raise ValueError("need matching, non-empty source and destination lists")
    block_bytes = src_caches[0][0].nbytes
    for a in list(src_caches) + list(dst_caches):
        if not a.flags.c_contiguous or a[0].nbytes != block_bytes:
            raise ValueError("every cache must be C-contiguous with equal blocks")
    bm = _arr(block_mapping, np.int64).reshape(-1, 2)
    sarr = (ctypes.c_void_p * n)(*[a.ctypes.data for a in src_caches])
    darr = (ctypes.c_void_p * n)(*[a.ctypes.data for a in dst_caches])
    rc = lib.oracle_swap_blocks(ctypes.cast(sarr, ctypes.c_void_p),
                                ctypes.cast(darr, ctypes.c_void_p), n, _ptr(bm),
                                bm.shape[0], block_bytes, src_caches[0].shape[0],
                                dst_caches[0].shape[0])
    _check(rc, "swap_blocks")

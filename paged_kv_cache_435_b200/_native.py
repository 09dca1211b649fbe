"""ctypes binding of libpagedattn.so (C ABI declared in include/pa.h).

Argument marshalling only: tensors are checked for device, dtype, shape and
contiguity, then their data pointers and the current CUDA stream go to the C
entry point of the same name.  All computation happens in the library's CUDA
kernels; there is no fallback of any kind.  A missing library raises.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Sequence

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libpagedattn.so")

PA_OK = 0
PA_ERR_INVALID_ARG = -1
PA_ERR_UNSUPPORTED = -2
PA_ERR_WORKSPACE = -3
PA_ERR_CUDA = -4
PA_ERR_NO_BLOCKS = -5

PA_DEVERR_BLOCK_ID = 0x1
PA_DEVERR_CONTEXT_LEN = 0x2
PA_DEVERR_SLOT = 0x4
PA_DEVERR_COPY_PAIR = 0x8
PA_DEVERR_TIMEOUT = 0x10
PA_DEVERR_INTERNAL = 0x20
PA_DEVERR_QUERY_LEN = 0x40
PA_DEVERR_PREFIX = 0x80

_lock = threading.Lock()
_lib = None


class PAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


def library_path() -> str:
    return LIB_PATH


def raw():
    """The loaded ctypes library with argument types declared."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is not built; run `python -m "
                "paged_kv_cache_435_b200.build` (needs nvcc)")
        lib = ctypes.CDLL(LIB_PATH)
        p, i32, i64, f32, sz = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64,
                                ctypes.c_float, ctypes.c_size_t)
        lib.pa_status_string.argtypes = [i32]
        lib.pa_status_string.restype = ctypes.c_char_p
        lib.pa_version.argtypes = []
        lib.pa_version.restype = i32
        lib.pa_launch_count.argtypes = []
        lib.pa_launch_count.restype = ctypes.c_uint64
        lib.pa_reshape_and_cache.argtypes = [
            p, p, i64, i64, p, p, p, i32, i32, i32, i32, i32, p, p]
        lib.pa_reshape_and_cache.restype = i32
        lib.pa_decode_partition_size.argtypes = [i32] * 7
        lib.pa_decode_partition_size.restype = i32
        lib.pa_decode_workspace_size.argtypes = [i32] * 7
        lib.pa_decode_workspace_size.restype = sz
        lib.pa_decode_attention.argtypes = [
            p, p, p, p, p, i32, p, i32, i32, i32, i32, i32, i32, i32, f32, i32,
            p, sz, p, p]
        lib.pa_decode_attention.restype = i32
        lib.pa_multi_query_attention.argtypes = [
            p, p, p, p, p, i32, p, i32, p, i32, i32, i32, i32, i32, i32, i32,
            f32, p, p]
        lib.pa_multi_query_attention.restype = i32
        lib.pa_shared_prefix_workspace_size.argtypes = [i32] * 7
        lib.pa_shared_prefix_workspace_size.restype = sz
        lib.pa_decode_attention_shared_prefix.argtypes = [
            p, p, p, p, p, i32, p, i32, p, p, i32, i32, i32, i32, i32, i32,
            i32, i32, f32, i32, p, sz, p, p]
        lib.pa_decode_attention_shared_prefix.restype = i32
        lib.pa_swap_blocks.argtypes = [p, p, i32, p, i32, i64, i64, i64, p, p]
        lib.pa_swap_blocks.restype = i32
        lib.pa_copy_blocks.argtypes = [p, p, i32, p, i32, i32, i32, i32, i32,
                                       p, p]
        lib.pa_copy_blocks.restype = i32
        lib.pa_decode_attention_static_ws.argtypes = [
            p, p, p, p, p, i32, p, i32, i32, i32, i32, i32, i32, i32, f32, i32,
            p, p]
        lib.pa_decode_attention_static_ws.restype = i32
        _lib = lib
        return lib


def status_string(status: int) -> str:
    return raw().pa_status_string(int(status)).decode()


def pa_launch_count() -> int:
    return int(raw().pa_launch_count())


def _check(status: int, where: str) -> int:
    if status != PA_OK:
        raise PAError(status, where)
    return status


def _cuda(t, name: str, dtype=None, ndim: Optional[int] = None):
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")
    return t


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def pa_reshape_and_cache(key, value, k_cache, v_cache, slot_mapping,
                         error_flags=None, stream=None) -> int:
    """Scatter key/value [T, Hkv, D] (token stride = stride(0)) into the
    bf16 pools [NB, bs, Hkv, D] at slot_mapping [T] (int64, <0 = skip)."""
    import torch
    bf = torch.bfloat16
    _cuda(key, "key", bf, 3); _cuda(value, "value", bf, 3)
    _cuda(k_cache, "k_cache", bf, 4); _cuda(v_cache, "v_cache", bf, 4)
    _cuda(slot_mapping, "slot_mapping", torch.int64, 1)
    NB, bs, Hkv, D = k_cache.shape
    if v_cache.shape != k_cache.shape or not (k_cache.is_contiguous() and
                                              v_cache.is_contiguous()):
        raise ValueError("k_cache/v_cache must be equal-shaped contiguous pools")
    T = key.shape[0]
    for name, t in (("key", key), ("value", value)):
        if tuple(t.shape) != (T, Hkv, D) or t.stride(2) != 1 or t.stride(1) != D:
            raise ValueError(f"{name} must be [T,{Hkv},{D}] with contiguous heads")
    if slot_mapping.shape[0] != T or not slot_mapping.is_contiguous():
        raise ValueError("slot_mapping must be a contiguous [T] tensor")
    rc = raw().pa_reshape_and_cache(
        _ptr(key), _ptr(value), key.stride(0), value.stride(0), _ptr(k_cache),
        _ptr(v_cache), _ptr(slot_mapping), T, NB, bs, Hkv, D,
        _ptr(error_flags), _stream(stream))
    return _check(rc, "pa_reshape_and_cache")


def pa_decode_partition_size(num_seqs, num_heads, num_kv_heads, head_size,
                             block_size, max_context_len,
                             partition_size=0) -> int:
    r = raw().pa_decode_partition_size(num_seqs, num_heads, num_kv_heads,
                                       head_size, block_size, max_context_len,
                                       partition_size)
    if r < 0:
        raise PAError(r, "pa_decode_partition_size")
    return r


def pa_decode_workspace_size(num_seqs, num_heads, num_kv_heads, head_size,
                             block_size, max_context_len,
                             partition_size=0) -> int:
    return int(raw().pa_decode_workspace_size(
        num_seqs, num_heads, num_kv_heads, head_size, block_size,
        max_context_len, partition_size))


def pa_decode_attention(out, q, k_cache, v_cache, block_tables, context_lens,
                        max_context_len: int, scale: float,
                        partition_size: int = 0, workspace=None,
                        error_flags=None, stream=None) -> int:
    """out fp32 [B,Hq,D] = paged decode attention of q bf16 [B,Hq,D] over the
    pools [NB,bs,Hkv,D] through block_tables int32 [B,MB] / context_lens [B]."""
    import torch
    bf = torch.bfloat16
    _cuda(out, "out", torch.float32, 3); _cuda(q, "q", bf, 3)
    _cuda(k_cache, "k_cache", bf, 4); _cuda(v_cache, "v_cache", bf, 4)
    _cuda(block_tables, "block_tables", torch.int32, 2)
    _cuda(context_lens, "context_lens", torch.int32, 1)
    for name, t in (("out", out), ("q", q), ("k_cache", k_cache),
                    ("v_cache", v_cache), ("block_tables", block_tables),
                    ("context_lens", context_lens)):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    B, Hq, D = q.shape
    NB, bs, Hkv, D2 = k_cache.shape
    if out.shape != q.shape or D2 != D or v_cache.shape != k_cache.shape:
        raise ValueError("shape mismatch between q, out and the pools")
    if block_tables.shape[0] != B or context_lens.shape[0] != B:
        raise ValueError("block_tables / context_lens must have B rows")
    ws_bytes = 0
    if workspace is not None:
        _cuda(workspace, "workspace")
        ws_bytes = workspace.numel() * workspace.element_size()
    rc = raw().pa_decode_attention(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
        block_tables.shape[1], _ptr(context_lens), int(max_context_len), B, Hq,
        Hkv, D, bs, NB, float(scale), int(partition_size), _ptr(workspace),
        ws_bytes, _ptr(error_flags), _stream(stream))
    return _check(rc, "pa_decode_attention")


def pa_multi_query_attention(out, q, k_cache, v_cache, block_tables,
                             context_lens, query_start_loc, max_context_len: int,
                             max_query_len: int, scale: float,
                             error_flags=None, stream=None) -> int:
    """out fp32 [T,Hq,D] = causal paged attention of the last k_s context
    tokens of each sequence (q bf16 [T,Hq,D], query_start_loc int32 [B+1])."""
    import torch
    bf = torch.bfloat16
    _cuda(out, "out", torch.float32, 3); _cuda(q, "q", bf, 3)
    _cuda(k_cache, "k_cache", bf, 4); _cuda(v_cache, "v_cache", bf, 4)
    _cuda(block_tables, "block_tables", torch.int32, 2)
    _cuda(context_lens, "context_lens", torch.int32, 1)
    _cuda(query_start_loc, "query_start_loc", torch.int32, 1)
    for name, t in (("out", out), ("q", q), ("k_cache", k_cache),
                    ("v_cache", v_cache), ("block_tables", block_tables),
                    ("context_lens", context_lens),
                    ("query_start_loc", query_start_loc)):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    T, Hq, D = q.shape
    NB, bs, Hkv, D2 = k_cache.shape
    B = context_lens.shape[0]
    if out.shape != q.shape or D2 != D or v_cache.shape != k_cache.shape:
        raise ValueError("shape mismatch between q, out and the pools")
    if block_tables.shape[0] != B or query_start_loc.shape[0] != B + 1:
        raise ValueError("block_tables / query_start_loc must match B")
    rc = raw().pa_multi_query_attention(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
        block_tables.shape[1], _ptr(context_lens), int(max_context_len),
        _ptr(query_start_loc), int(max_query_len), B, Hq, Hkv, D, bs, NB,
        float(scale), _ptr(error_flags), _stream(stream))
    return _check(rc, "pa_multi_query_attention")


def pa_shared_prefix_workspace_size(num_seqs, num_heads, num_kv_heads,
                                    head_size, block_size, max_context_len,
                                    partition_size=0) -> int:
    return int(raw().pa_shared_prefix_workspace_size(
        num_seqs, num_heads, num_kv_heads, head_size, block_size,
        max_context_len, partition_size))


def pa_decode_attention_shared_prefix(out, q, k_cache, v_cache, block_tables,
                                      context_lens, group_start, prefix_lens,
                                      max_context_len: int,
                                      max_group_size: int, scale: float,
                                      workspace, partition_size: int = 0,
                                      error_flags=None, stream=None) -> int:
    """pa_decode_attention for batches whose sequences share prompt blocks:
    sequences group_start[i] .. group_start[i+1]-1 (int32 [G+1]) share their
    first prefix_lens[i] tokens (int32 [G]); workspace of at least
    pa_shared_prefix_workspace_size(...) bytes."""
    import torch
    bf = torch.bfloat16
    _cuda(out, "out", torch.float32, 3); _cuda(q, "q", bf, 3)
    _cuda(k_cache, "k_cache", bf, 4); _cuda(v_cache, "v_cache", bf, 4)
    _cuda(block_tables, "block_tables", torch.int32, 2)
    _cuda(context_lens, "context_lens", torch.int32, 1)
    _cuda(group_start, "group_start", torch.int32, 1)
    _cuda(prefix_lens, "prefix_lens", torch.int32, 1)
    if workspace is not None:
        _cuda(workspace, "workspace")
    for name, t in (("out", out), ("q", q), ("k_cache", k_cache),
                    ("v_cache", v_cache), ("block_tables", block_tables),
                    ("context_lens", context_lens),
                    ("group_start", group_start), ("prefix_lens", prefix_lens)):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    B, Hq, D = q.shape
    NB, bs, Hkv, D2 = k_cache.shape
    G = prefix_lens.shape[0]
    if out.shape != q.shape or D2 != D or v_cache.shape != k_cache.shape:
        raise ValueError("shape mismatch between q, out and the pools")
    if block_tables.shape[0] != B or context_lens.shape[0] != B:
        raise ValueError("block_tables / context_lens must have B rows")
    if group_start.shape[0] != G + 1:
        raise ValueError("group_start must have one more entry than prefix_lens")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = raw().pa_decode_attention_shared_prefix(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
        block_tables.shape[1], _ptr(context_lens), int(max_context_len),
        _ptr(group_start), _ptr(prefix_lens), G, int(max_group_size), B, Hq,
        Hkv, D, bs, NB, float(scale), int(partition_size), _ptr(workspace),
        ws_bytes, _ptr(error_flags), _stream(stream))
    return _check(rc, "pa_decode_attention_shared_prefix")


def pa_swap_blocks(src_caches: Sequence, dst_caches: Sequence, block_mapping,
                   error_flags=None, stream=None) -> int:
    """Move whole blocks src_caches[c][src] -> dst_caches[c][dst] for each
    (src, dst) row of block_mapping (int64 [N,2]).  Each cache is a
    contiguous tensor whose first dimension is the block index, on the GPU or
    in pinned host memory (pin_memory()); block_mapping likewise."""
    import torch
    n = len(src_caches)
    if n == 0 or len(dst_caches) != n:
        raise ValueError("need matching, non-empty source and destination lists")
    block_bytes = src_caches[0][0].numel() * src_caches[0].element_size()
    for t in list(src_caches) + list(dst_caches):
        if not isinstance(t, torch.Tensor) or not t.is_contiguous():
            raise ValueError("caches must be contiguous tensors")
        if not (t.is_cuda or t.is_pinned()):
            raise ValueError("host caches must be pinned (pin_memory())")
        if t[0].numel() * t.element_size() != block_bytes:
            raise ValueError("every cache must have the same block size")
    if block_mapping.dtype != torch.int64 or block_mapping.dim() != 2 or \
            block_mapping.shape[1] != 2 or not block_mapping.is_contiguous():
        raise ValueError("block_mapping must be a contiguous int64 [N,2] tensor")
    if not (block_mapping.is_cuda or block_mapping.is_pinned()):
        raise ValueError("block_mapping must be on the GPU or pinned")
    sarr = (ctypes.c_void_p * n)(*[t.data_ptr() for t in src_caches])
    darr = (ctypes.c_void_p * n)(*[t.data_ptr() for t in dst_caches])
    rc = raw().pa_swap_blocks(ctypes.cast(sarr, ctypes.c_void_p),
                              ctypes.cast(darr, ctypes.c_void_p), n,
                              _ptr(block_mapping), block_mapping.shape[0],
                              block_bytes, src_caches[0].shape[0],
                              dst_caches[0].shape[0], _ptr(error_flags),
                              _stream(stream))
    return _check(rc, "pa_swap_blocks")


def pa_copy_blocks(k_caches: Sequence, v_caches: Sequence, block_mapping,
                   error_flags=None, stream=None) -> int:
    """Copy whole blocks src->dst (block_mapping int64 [N,2]) in every layer's
    K and V pool."""
    import torch
    if len(k_caches) == 0 or len(v_caches) != len(k_caches):
        raise ValueError("need matching, non-empty K and V layer lists")
    shape = k_caches[0].shape
    for t in list(k_caches) + list(v_caches):
        _cuda(t, "cache", torch.bfloat16, 4)
        if t.shape != shape or not t.is_contiguous():
            raise ValueError("every layer pool must be a contiguous [NB,bs,Hkv,D]")
    _cuda(block_mapping, "block_mapping", torch.int64, 2)
    if block_mapping.shape[1] != 2 or not block_mapping.is_contiguous():
        raise ValueError("block_mapping must be a contiguous [N,2] tensor")
    NB, bs, Hkv, D = shape
    n = len(k_caches)
    karr = (ctypes.c_void_p * n)(*[t.data_ptr() for t in k_caches])
    varr = (ctypes.c_void_p * n)(*[t.data_ptr() for t in v_caches])
    rc = raw().pa_copy_blocks(ctypes.cast(karr, ctypes.c_void_p),
                              ctypes.cast(varr, ctypes.c_void_p), n,
                              _ptr(block_mapping), block_mapping.shape[0], NB,
                              bs, Hkv, D, _ptr(error_flags), _stream(stream))
    return _check(rc, "pa_copy_blocks")


def pa_decode_attention_static_ws(out, q, k_cache, v_cache, block_tables,
                                  context_lens, max_context_len: int,
                                  scale: float, partition_size: int = 0,
                                  error_flags=None, stream=None) -> int:
    """pa_decode_attention with the library's built-in workspace, for callers
    that cannot allocate device memory (see include/pa.h)."""
    import torch
    f = raw().pa_decode_attention_static_ws
    bf = torch.bfloat16
    _cuda(out, "out", torch.float32, 3); _cuda(q, "q", bf, 3)
    _cuda(k_cache, "k_cache", bf, 4); _cuda(v_cache, "v_cache", bf, 4)
    _cuda(block_tables, "block_tables", torch.int32, 2)
    _cuda(context_lens, "context_lens", torch.int32, 1)
    for name, t in (("out", out), ("q", q), ("k_cache", k_cache),
                    ("v_cache", v_cache), ("block_tables", block_tables),
                    ("context_lens", context_lens)):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    B, Hq, D = q.shape
    NB, bs, Hkv, D2 = k_cache.shape
    if out.shape != q.shape or D2 != D or v_cache.shape != k_cache.shape:
        raise ValueError("shape mismatch between q, out and the pools")
    if block_tables.shape[0] != B or context_lens.shape[0] != B:
        raise ValueError("block_tables / context_lens must have B rows")
    # The built-in scratch is looked up on the current device: every buffer
    # must live there too.
    cur = torch.cuda.current_device()
    for name, t in (("out", out), ("q", q), ("k_cache", k_cache),
                    ("v_cache", v_cache), ("block_tables", block_tables),
                    ("context_lens", context_lens), ("error_flags", error_flags)):
        if t is not None and t.device.index != cur:
            raise ValueError(f"{name} is on cuda:{t.device.index}, the current "
                             f"device is cuda:{cur}")
    rc = f(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
           block_tables.shape[1], _ptr(context_lens), int(max_context_len), B,
           Hq, Hkv, D, bs, NB, float(scale), int(partition_size),
           _ptr(error_flags), _stream(stream))
    return _check(rc, "pa_decode_attention_static_ws")

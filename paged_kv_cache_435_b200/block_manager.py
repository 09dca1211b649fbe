"""ctypes wrapper of the library's host-side block manager (include/pa.h,
"Host-side block manager"): free block pool, per-sequence block tables,
reference-counted sharing with copy-on-write, prefix caching and CPU swap
bookkeeping.  Marshalling only; the logic is C++ in libpagedattn.so."""
from __future__ import annotations

import ctypes
from typing import Optional, Sequence

import numpy as np

from . import _native as nat


def _lib():
    lib = nat.raw()
    if not getattr(lib, "_bm_declared", False):
        p, i32, i64, u64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_uint64
        lib.pa_prefix_block_hash.argtypes = [u64, p, i32]
        lib.pa_prefix_block_hash.restype = u64
        lib.pa_prefix_hash_seed.argtypes = []
        lib.pa_prefix_hash_seed.restype = u64
        lib.pa_bm_create.argtypes = [i32, i32, i32, i32]
        lib.pa_bm_create.restype = p
        lib.pa_bm_destroy.argtypes = [p]
        lib.pa_bm_destroy.restype = None
        for name in ("pa_bm_num_free_blocks", "pa_bm_num_free_cpu_blocks"):
            getattr(lib, name).argtypes = [p]
            getattr(lib, name).restype = i32
        lib.pa_bm_add_sequence.argtypes = [p, p, i32, p, p]
        lib.pa_bm_add_sequence.restype = i32
        lib.pa_bm_fork.argtypes = [p, i32]
        lib.pa_bm_fork.restype = i32
        lib.pa_bm_append_slots.argtypes = [p, i32, i32, p, p, p, i32, p]
        lib.pa_bm_append_slots.restype = i32
        lib.pa_bm_free_sequence.argtypes = [p, i32]
        lib.pa_bm_free_sequence.restype = i32
        lib.pa_bm_seq_len.argtypes = [p, i32]
        lib.pa_bm_seq_len.restype = i32
        lib.pa_bm_block_table.argtypes = [p, i32, p, i32]
        lib.pa_bm_block_table.restype = i32
        lib.pa_bm_block_refcount.argtypes = [p, i32]
        lib.pa_bm_block_refcount.restype = i32
        lib.pa_bm_swap_out.argtypes = [p, i32, p, i32]
        lib.pa_bm_swap_out.restype = i32
        lib.pa_bm_swap_in.argtypes = [p, i32, p, i32]
        lib.pa_bm_swap_in.restype = i32
        lib.pa_bm_shared_prefix_groups.argtypes = [p, p, i32, i32, p, p, p]
        lib.pa_bm_shared_prefix_groups.restype = i32
        lib._bm_declared = True
    return lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def prefix_block_hash(parent: int, tokens: Sequence[int]) -> int:
    t = np.ascontiguousarray(tokens, dtype=np.int32)
    return int(_lib().pa_prefix_block_hash(parent, _ptr(t), t.size))


def prefix_hash_seed() -> int:
    return int(_lib().pa_prefix_hash_seed())


class BlockManager:
    def __init__(self, num_blocks: int, block_size: int,
                 num_cpu_blocks: int = 0, prefix_caching: bool = False):
        self.block_size = block_size
        self._m = _lib().pa_bm_create(num_blocks, num_cpu_blocks, block_size,
                                      int(prefix_caching))
        if not self._m:
            raise ValueError("pa_bm_create failed")

    def close(self):
        if self._m:
            _lib().pa_bm_destroy(self._m)
            self._m = None

    __del__ = close

    @staticmethod
    def _check(rc: int, where: str) -> int:
        if rc < 0:
            raise nat.PAError(rc, where)
        return rc

    @property
    def num_free_blocks(self) -> int:
        return _lib().pa_bm_num_free_blocks(self._m)

    @property
    def num_free_cpu_blocks(self) -> int:
        return _lib().pa_bm_num_free_cpu_blocks(self._m)

    def add_sequence(self, token_ids):
        """-> (seq_id, slot_mapping of the uncached tokens, cached token count)"""
        t = np.ascontiguousarray(token_ids, dtype=np.int32)
        slots = np.empty(max(t.size, 1), dtype=np.int64)
        cached = ctypes.c_int(0)
        sid = self._check(_lib().pa_bm_add_sequence(
            self._m, _ptr(t), t.size, _ptr(slots), ctypes.byref(cached)),
            "pa_bm_add_sequence")
        return sid, slots[:t.size - cached.value].copy(), cached.value

    def fork(self, parent: int) -> int:
        return self._check(_lib().pa_bm_fork(self._m, parent), "pa_bm_fork")

    def append_slots(self, seq_id: int, num_new_tokens: int, token_ids=None):
        """-> (slot_mapping [n], cow_pairs [c, 2])"""
        t = None if token_ids is None else np.ascontiguousarray(token_ids, dtype=np.int32)
        slots = np.empty(max(num_new_tokens, 1), dtype=np.int64)
        pairs = np.empty((1, 2), dtype=np.int64)
        ncow = ctypes.c_int(0)
        self._check(_lib().pa_bm_append_slots(
            self._m, seq_id, num_new_tokens, _ptr(t), _ptr(slots), _ptr(pairs),
            1, ctypes.byref(ncow)), "pa_bm_append_slots")
        return slots[:num_new_tokens].copy(), pairs[:ncow.value].copy()

    def free(self, seq_id: int) -> None:
        self._check(_lib().pa_bm_free_sequence(self._m, seq_id), "pa_bm_free_sequence")

    def seq_len(self, seq_id: int) -> int:
        return self._check(_lib().pa_bm_seq_len(self._m, seq_id), "pa_bm_seq_len")

    def block_table(self, seq_id: int) -> np.ndarray:
        n = self._check(_lib().pa_bm_block_table(self._m, seq_id, None, 0),
                        "pa_bm_block_table")
        out = np.empty(max(n, 1), dtype=np.int32)
        self._check(_lib().pa_bm_block_table(self._m, seq_id, _ptr(out), n),
                    "pa_bm_block_table")
        return out[:n].copy()

    def refcount(self, block: int) -> int:
        return self._check(_lib().pa_bm_block_refcount(self._m, block),
                           "pa_bm_block_refcount")

    def swap_out(self, seq_id: int) -> np.ndarray:
        cap = len(self.block_table(seq_id))
        pairs = np.empty((max(cap, 1), 2), dtype=np.int64)
        n = self._check(_lib().pa_bm_swap_out(self._m, seq_id, _ptr(pairs), cap),
                        "pa_bm_swap_out")
        return pairs[:n].copy()

    def swap_in(self, seq_id: int) -> np.ndarray:
        cap = len(self.block_table(seq_id))
        pairs = np.empty((max(cap, 1), 2), dtype=np.int64)
        n = self._check(_lib().pa_bm_swap_in(self._m, seq_id, _ptr(pairs), cap),
                        "pa_bm_swap_in")
        return pairs[:n].copy()

    def shared_prefix_groups(self, seq_ids, min_shared_blocks: int = 1):
        """(group_start int32 [G+1], prefix_lens int32 [G], max_group_size)
        for pa_decode_attention_shared_prefix on the batch `seq_ids` (in
        launch order): consecutive sequences sharing at least
        min_shared_blocks leading blocks are grouped."""
        ids = np.ascontiguousarray(seq_ids, dtype=np.int32)
        gs = np.zeros(ids.size + 1, dtype=np.int32)
        pl = np.zeros(max(ids.size, 1), dtype=np.int32)
        mg = ctypes.c_int(0)
        g = self._check(_lib().pa_bm_shared_prefix_groups(
            self._m, _ptr(ids), ids.size, int(min_shared_blocks), _ptr(gs),
            _ptr(pl), ctypes.byref(mg)), "pa_bm_shared_prefix_groups")
        return gs[:g + 1].copy(), pl[:g].copy(), int(mg.value)

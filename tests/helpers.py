"""Shared test plumbing: run a decode step through the C ABI on the GPU, run
the same step through the fp64 oracle on the host, compare."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import paged_kv_cache_435_b200 as pa

# Attention output (fp32) against the fp64 oracle on the same bf16 inputs.
TOL_MAX_ABS = 4e-3
TOL_REL_L2 = 1e-3


def bits(t: torch.Tensor) -> np.ndarray:
    """uint16 copy of a bf16 tensor's bits on the host."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16).copy()


def attn_errors(got: torch.Tensor, ref: np.ndarray):
    g = got.detach().double().cpu().numpy()
    assert g.shape == ref.shape, (g.shape, ref.shape)
    assert np.all(np.isfinite(g)), "non-finite GPU output"
    diff = g - ref
    max_abs = float(np.max(np.abs(diff))) if diff.size else 0.0
    denom = float(np.linalg.norm(ref))
    rel_l2 = float(np.linalg.norm(diff) / denom) if denom > 0 else float(np.linalg.norm(diff))
    return max_abs, rel_l2


def assert_attn_close(got, ref, what=""):
    max_abs, rel_l2 = attn_errors(got, ref)
    assert max_abs <= TOL_MAX_ABS and rel_l2 <= TOL_REL_L2, (
        f"{what}: max_abs={max_abs:.3e} rel_l2={rel_l2:.3e}")
    return max_abs, rel_l2


def gpu_step(case, partition_size: int = 0, error_flags=None,
             do_copy: bool = True, do_write: bool = True):
    """copy_blocks (when the case has CoW pairs) -> reshape_and_cache ->
    decode attention, all through the C ABI on the current stream.  Mutates
    case.k_cache / case.v_cache.  Returns the fp32 output."""
    w = case.workload
    B, Hq, D = case.q.shape
    if do_copy and case.copy_pairs.shape[0] > 0:
        pa.pa_copy_blocks([case.k_cache], [case.v_cache], case.copy_pairs,
                          error_flags=error_flags)
    if do_write:
        pa.pa_reshape_and_cache(case.new_key, case.new_value, case.k_cache,
                                case.v_cache, case.slot_mapping,
                                error_flags=error_flags)
    out = torch.empty(B, Hq, D, dtype=torch.float32, device=case.q.device)
    maxlen = case.max_context_len
    ws_bytes = pa.pa_decode_workspace_size(B, Hq, w.num_kv_heads, D,
                                           w.block_size, maxlen, partition_size)
    ws = (torch.empty(ws_bytes, dtype=torch.uint8, device=case.q.device)
          if ws_bytes else None)
    pa.pa_decode_attention(out, case.q, case.k_cache, case.v_cache,
                           case.block_tables, case.context_lens, maxlen,
                           case.scale, partition_size=partition_size,
                           workspace=ws, error_flags=error_flags)
    return out


def oracle_pools_after_step(case, k_bits, v_bits, do_copy=True, do_write=True):
    """Apply the step's cache writes to host pool bits with the oracle."""
    if do_copy and case.copy_pairs.shape[0] > 0:
        oracle.copy_blocks([k_bits], [v_bits], case.copy_pairs.cpu().numpy())
    if do_write:
        oracle.reshape_and_cache(case.new_key.cpu(), case.new_value.cpu(),
                                 k_bits, v_bits, case.slot_mapping.cpu().numpy())


def oracle_attention(case, k_bits, v_bits, seqs=None):
    q = case.q.cpu()
    tables = case.tables_np
    lens = case.lens_np.astype(np.int32)
    if seqs is not None:
        seqs = np.asarray(seqs)
        q = q[torch.from_numpy(seqs)]
        tables = tables[seqs]
        lens = lens[seqs]
    return oracle.paged_decode_attention(q, k_bits, v_bits, tables, lens,
                                         case.scale,
                                         case.workload.num_kv_heads)


# Bit patterns a never-written bf16 slot may hold: NaN, +inf, -inf, -NaN.
_POISON = np.array([0x7FC0, 0x7F80, 0xFF80, 0xFFC1], dtype=np.uint16)


def poison_unwritten_slots(case, extra_live=()):
    """Fill every K and V slot that no sequence's context covers (the rows
    past the last token of each last block, blocks no table reaches) with
    NaN and infinities.  A kernel must never let such a slot reach an
    output: the attention of a sequence depends on its first L tokens only.
    `extra_live`: further (sequence, length) pairs whose tokens stay as they
    are.  Returns the number of poisoned slots."""
    bs = case.workload.block_size
    NB = case.k_cache.shape[0]
    live = np.zeros(NB * bs, dtype=bool)
    pairs = list(zip(range(len(case.lens_np)), case.lens_np)) + list(extra_live)
    for s, L in pairs:
        L = int(L)
        if L <= 0:
            continue
        t = np.arange(L)
        ids = case.tables_np[s, t // bs].astype(np.int64)
        live[ids * bs + t % bs] = True
    dead = np.nonzero(~live)[0]
    pattern = torch.from_numpy(_POISON[dead % 4].view(np.int16).copy())
    idx = torch.from_numpy(dead)
    for pool in (case.k_cache, case.v_cache):
        flat = pool.view(NB * bs, -1).view(torch.int16)
        flat[idx.to(pool.device)] = pattern.to(pool.device)[:, None]
    return int(dead.size)

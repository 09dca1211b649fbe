"""pa_decode_attention_static_ws: the decode entry point for callers that
cannot allocate device memory (plugin hooks handed only inputs and outputs,
processes whose device memory another allocator reserved, C callers without a
device allocator).  Its split-KV scratch is an array built into the library,
shared by every call and never cleared, so the tests alternate two different
requests: a read of scratch left by the previous call would change the
second one's output.  Each output must equal pa_decode_attention's with a
caller-allocated workspace bit for bit (same kernels, same reduction order)
and match the fp64 oracle within the attention tolerance.

This file is collected last so that a run stopping at the first failure has
already run every other test; it also passes when run alone.
"""
import ctypes

import numpy as np
import pytest
import torch

import paged_kv_cache_435_b200 as pa
from paged_kv_cache_435_b200 import _native as nat
from paged_kv_cache_435_b200 import inputs
from tests.helpers import assert_attn_close, bits, oracle_attention

pytestmark = pytest.mark.gpu

STATIC_WS_BYTES = 32 << 20  # PA_STATIC_WORKSPACE_BYTES in include/pa.h


@pytest.fixture(autouse=True)
def _need_gpu():
    assert torch.cuda.is_available(), "GPU test run without a CUDA device"


def call_static(out, case, partition_size, flags):
    """One call through the C ABI (ctypes, plain pointers)."""
    w = case.workload
    B, Hq, D = case.q.shape
    return nat.raw().pa_decode_attention_static_ws(
        out.data_ptr(), case.q.data_ptr(), case.k_cache.data_ptr(),
        case.v_cache.data_ptr(), case.block_tables.data_ptr(),
        case.block_tables.shape[1], case.context_lens.data_ptr(),
        case.max_context_len, B, Hq, w.num_kv_heads, D, w.block_size,
        case.k_cache.shape[0], case.scale, partition_size, flags.data_ptr(),
        torch.cuda.current_stream().cuda_stream)


def allocating_output(case, partition_size):
    w = case.workload
    B, Hq, D = case.q.shape
    nbytes = pa.pa_decode_workspace_size(B, Hq, w.num_kv_heads, D, w.block_size,
                                         case.max_context_len, partition_size)
    ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device="cuda")
    out = torch.empty(B, Hq, D, dtype=torch.float32, device="cuda")
    pa.pa_decode_attention(out, case.q, case.k_cache, case.v_cache,
                           case.block_tables, case.context_lens,
                           case.max_context_len, case.scale,
                           partition_size=partition_size, workspace=ws)
    torch.cuda.synchronize()
    return out, nbytes


def two_cases():
    # Few (sequence, kv head) units and long contexts: the split-KV path,
    # which is the one that needs scratch.  The second request has fewer
    # sequences, heads and partitions than the first, so its scratch rows
    # sit at other offsets than the first's.
    a = inputs.custom_case(4, 32, 8, 128, 16, [3000, 700, 5000, 1], seed=11,
                           device="cuda")
    b = inputs.custom_case(3, 16, 4, 128, 32, [1200, 64, 2500], seed=12,
                           device="cuda")
    return (a, 256), (b, 512)


def test_static_workspace_alternating_requests_match_allocating_call_and_oracle():
    cases = two_cases()
    expected = []
    for case, part in cases:
        ref, nbytes = allocating_output(case, part)
        assert 0 < nbytes <= STATIC_WS_BYTES
        oracle_ref = oracle_attention(case, bits(case.k_cache), bits(case.v_cache))
        expected.append((ref, oracle_ref))
    # a, b, a, b: each call follows one that left different scratch behind.
    for rnd in range(2):
        for (case, part), (ref, oracle_ref) in zip(cases, expected):
            out = torch.full_like(ref, float("nan"))
            flags = torch.zeros(1, dtype=torch.int32, device="cuda")
            n0 = pa.pa_launch_count()
            rc = call_static(out, case, part, flags)
            assert rc == pa.PA_OK, pa.status_string(rc)
            torch.cuda.synchronize()
            assert pa.pa_launch_count() - n0 == 2   # partition + merge kernels
            assert int(flags.item()) == 0
            assert torch.equal(out, ref), f"round {rnd}: differs from pa_decode_attention"
            assert_attn_close(out, oracle_ref, f"static workspace, round {rnd}")


def test_python_wrapper_and_empty_batch():
    (case, part), _ = two_cases()
    ref, _ = allocating_output(case, part)
    out = torch.empty_like(ref)
    pa.pa_decode_attention_static_ws(out, case.q, case.k_cache, case.v_cache,
                                     case.block_tables, case.context_lens,
                                     case.max_context_len, case.scale,
                                     partition_size=part)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    # num_seqs = 0: the start-up call that commits the array, no launch.
    n0 = pa.pa_launch_count()
    rc = nat.raw().pa_decode_attention_static_ws(
        None, None, None, None, None, 1, None, 0, 0, 8, 8, 128, 16, 1, 0.1, 0,
        None, None)
    assert rc == pa.PA_OK
    assert pa.pa_launch_count() == n0


def test_static_workspace_rejects_requests_beyond_its_capacity():
    # 64 sequences x 64 heads x 128 partitions of 512 tokens needs far more
    # than the built-in 32 MiB: refused before anything is enqueued.
    need = pa.pa_decode_workspace_size(64, 64, 8, 128, 16, 65536, 512)
    assert need > STATIC_WS_BYTES
    fake = 1 << 20
    n0 = pa.pa_launch_count()
    rc = nat.raw().pa_decode_attention_static_ws(
        fake, fake, fake, fake, fake, 4096, fake, 65536, 64, 64, 8, 128, 16,
        1 << 20, 0.1, 512, None, None)
    assert rc == pa.PA_ERR_WORKSPACE
    assert pa.pa_launch_count() == n0

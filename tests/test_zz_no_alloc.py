"""pa_decode_attention_static_ws: the decode entry point for callers that
cannot allocate device memory (plugin hooks handed only inputs and outputs,
processes whose device memory another allocator reserved, C callers without a
device allocator).  It must give the same output as pa_decode_attention with a
caller-allocated workspace, call after call, while itself allocating nothing.

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
from tests.helpers import TOL_MAX_ABS, TOL_REL_L2

pytestmark = pytest.mark.gpu

STATIC_WS_BYTES = 32 << 20  # PA_STATIC_WORKSPACE_BYTES in include/pa.h


@pytest.fixture(autouse=True)
def _need_gpu():
    assert torch.cuda.is_available(), "GPU test run without a CUDA device"


def static_ws_fn():
    f = nat.raw().pa_decode_attention_static_ws
    p, i32, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    f.argtypes = [p, p, p, p, p, i32, p, i32, i32, i32, i32, i32, i32, i32,
                  f32, i32, p, p]
    f.restype = i32
    return f


def call_static(f, out, case, partition_size, flags):
    w = case.workload
    B, Hq, D = case.q.shape
    return f(out.data_ptr(), case.q.data_ptr(), case.k_cache.data_ptr(),
             case.v_cache.data_ptr(), case.block_tables.data_ptr(),
             case.block_tables.shape[1], case.context_lens.data_ptr(),
             case.max_context_len, B, Hq, w.num_kv_heads, D, w.block_size,
             case.k_cache.shape[0], case.scale, partition_size,
             flags.data_ptr(), torch.cuda.current_stream().cuda_stream)


def reference_output(case, partition_size):
    w = case.workload
    B, Hq, D = case.q.shape
    nbytes = pa.pa_decode_workspace_size(B, Hq, w.num_kv_heads, D, w.block_size,
                                         case.max_context_len, partition_size)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    out = torch.empty(B, Hq, D, dtype=torch.float32, device="cuda")
    pa.pa_decode_attention(out, case.q, case.k_cache, case.v_cache,
                           case.block_tables, case.context_lens,
                           case.max_context_len, case.scale,
                           partition_size=partition_size, workspace=ws)
    return out, nbytes


def assert_close(got, ref):
    g = got.double().cpu().numpy()
    r = ref.double().cpu().numpy()
    assert np.all(np.isfinite(g))
    diff = g - r
    max_abs = float(np.abs(diff).max())
    rel_l2 = float(np.linalg.norm(diff) / np.linalg.norm(r))
    assert max_abs <= TOL_MAX_ABS and rel_l2 <= TOL_REL_L2, (max_abs, rel_l2)


@pytest.mark.parametrize("partition_size", [0, 256])
def test_static_workspace_matches_allocating_entry_point(partition_size):
    # Few (sequence, kv head) units and long contexts: the split-KV path,
    # which is the one that needs scratch memory.
    case = inputs.custom_case(4, 32, 8, 128, 16, [3000, 700, 5000, 1], seed=11,
                              device="cuda")
    ref, nbytes = reference_output(case, partition_size)
    assert 0 < nbytes <= STATIC_WS_BYTES
    f = static_ws_fn()
    for _ in range(2):  # two calls in a row share and reuse the same array
        out = torch.full_like(ref, float("nan"))
        flags = torch.zeros(1, dtype=torch.int32, device="cuda")
        n0 = pa.pa_launch_count()
        rc = call_static(f, out, case, partition_size, flags)
        assert rc == pa.PA_OK, pa.status_string(rc)
        torch.cuda.synchronize()
        assert pa.pa_launch_count() - n0 == 2      # partition + merge kernels
        assert int(flags.item()) == 0
        assert_close(out, ref)


def test_static_workspace_rejects_requests_beyond_its_capacity():
    # 64 sequences x 64 heads x 128 partitions of 512 tokens needs far more
    # than the built-in 32 MiB: refused before anything is enqueued.
    f = static_ws_fn()
    need = pa.pa_decode_workspace_size(64, 64, 8, 128, 16, 65536, 512)
    assert need > STATIC_WS_BYTES
    fake = 1 << 20
    n0 = pa.pa_launch_count()
    rc = f(fake, fake, fake, fake, fake, 4096, fake, 65536, 64, 64, 8, 128,
           16, 1 << 20, 0.1, 512, None, None)
    assert rc == pa.PA_ERR_WORKSPACE
    assert pa.pa_launch_count() == n0

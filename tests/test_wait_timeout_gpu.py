"""A bounded wait in the decode kernel that runs out.

Every mbarrier wait in the kernels gives up after a time limit, reports
PA_DEVERR_TIMEOUT in the caller's flag word and lets the CTA finish: it
skips the rest of its work, waits (with the full limit) for the copies it
already issued, and exits, so the context stays usable.  To watch that path
run without any GPU fault, the test loads libpagedattn_waittest.so, the same
sources built with PA_TEST_UNSIGNALLED_FIRST_WAIT: there every warp's first
chunk wait polls a barrier that nothing arrives on, under a 20 ms limit.
The call must still return PA_OK, the flag must carry the timeout bit, and a
following call of the product library on the same device must be correct.
"""
import ctypes

import numpy as np
import pytest
import torch

import paged_kv_cache_435_b200 as pa
from paged_kv_cache_435_b200 import build as pa_build
from paged_kv_cache_435_b200 import inputs
from tests.helpers import (assert_attn_close, bits, gpu_step, oracle_attention)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_gpu():
    assert torch.cuda.is_available(), "GPU test run without a CUDA device"


@pytest.fixture(scope="module")
def waittest_lib():
    pa_build.build()
    lib = ctypes.CDLL(pa_build.WAITTEST_LIB)
    p, i32, f32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.pa_decode_attention.argtypes = [
        p, p, p, p, p, i32, p, i32, i32, i32, i32, i32, i32, i32, f32, i32,
        p, sz, p, p]
    lib.pa_decode_attention.restype = i32
    return lib


def stalled_call(lib, case, partition_size, flags):
    w = case.workload
    B, Hq, D = case.q.shape
    nbytes = pa.pa_decode_workspace_size(B, Hq, w.num_kv_heads, D, w.block_size,
                                         case.max_context_len, partition_size)
    ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device="cuda")
    out = torch.empty(B, Hq, D, dtype=torch.float32, device="cuda")
    rc = lib.pa_decode_attention(
        out.data_ptr(), case.q.data_ptr(), case.k_cache.data_ptr(),
        case.v_cache.data_ptr(), case.block_tables.data_ptr(),
        case.block_tables.shape[1], case.context_lens.data_ptr(),
        case.max_context_len, B, Hq, w.num_kv_heads, D, w.block_size,
        case.k_cache.shape[0], case.scale, partition_size, ws.data_ptr(),
        nbytes, flags.data_ptr(), torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()   # the kernel ends: every wait is bounded
    return rc


@pytest.mark.parametrize("partition_size", [0, 128])
def test_expired_wait_reports_timeout_and_device_stays_usable(waittest_lib,
                                                              partition_size):
    # partition 0: one CTA per (kv head, sequence); 128: the persistent
    # split grid and the merge kernel.
    case = inputs.custom_case(3, 16, 2, 128, 16, [300, 40, 1000], seed=21,
                              device="cuda")
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = stalled_call(waittest_lib, case, partition_size, flags)
    assert rc == pa.PA_OK
    assert int(flags.item()) & pa.PA_DEVERR_TIMEOUT
    # The context is intact: the product library's next call is exact.
    flags.zero_()
    out = gpu_step(case, partition_size=partition_size, error_flags=flags,
                   do_write=False)
    torch.cuda.synchronize()
    assert int(flags.item()) == 0
    ref = oracle_attention(case, bits(case.k_cache), bits(case.v_cache))
    assert_attn_close(out, ref, "after an expired wait")

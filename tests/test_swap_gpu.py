"""pa_swap_blocks on the GPU: blocks swapped out to a pinned CPU pool and back
in to new block ids, bit-exact against the oracle."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_435_b200 as pa
from paged_kv_cache_435_b200 import _native as nat

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_gpu():
    assert torch.cuda.is_available(), "GPU test run without a CUDA device"


def host_bits(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16).copy()


def test_swap_out_then_in_bit_exact():
    layers, nb_gpu, nb_cpu, shape = 3, 40, 16, (16, 8, 128)
    gen = torch.Generator().manual_seed(0)
    gpu = [torch.randn(nb_gpu, *shape, generator=gen).to(torch.bfloat16).cuda()
           for _ in range(2 * layers)]
    cpu = [torch.zeros(nb_cpu, *shape, dtype=torch.bfloat16).pin_memory()
           for _ in range(2 * layers)]
    out_pairs = torch.tensor([[3, 0], [17, 5], [39, 15], [8, 1]], dtype=torch.int64)
    g_bits = [host_bits(t) for t in gpu]
    c_bits = [host_bits(t) for t in cpu]
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_swap_blocks(gpu, cpu, out_pairs.cuda(), error_flags=flags)
    torch.cuda.synchronize()
    oracle.swap_blocks(g_bits, c_bits, out_pairs.numpy())
    for t, e in zip(cpu, c_bits):
        np.testing.assert_array_equal(host_bits(t), e)
    # the GPU blocks get reused by others, then the request resumes elsewhere
    for t in gpu:
        t.normal_()
    g_bits = [host_bits(t) for t in gpu]
    in_pairs = torch.tensor([[0, 20], [5, 21], [15, 22], [1, 23]],
                            dtype=torch.int64).pin_memory()
    pa.pa_swap_blocks(cpu, gpu, in_pairs, error_flags=flags)
    torch.cuda.synchronize()
    assert int(flags.item()) == 0
    oracle.swap_blocks(c_bits, g_bits, in_pairs.numpy())
    for t, e in zip(gpu, g_bits):
        np.testing.assert_array_equal(host_bits(t), e)


def test_swap_rejects_pageable_host_memory():
    gpu = torch.zeros(4, 16, 2, 64, dtype=torch.bfloat16, device="cuda")
    pageable = torch.zeros(4, 16, 2, 64, dtype=torch.bfloat16)
    pairs = torch.tensor([[0, 1]], dtype=torch.int64, device="cuda")
    src = (ctypes.c_void_p * 1)(gpu.data_ptr())
    dst = (ctypes.c_void_p * 1)(pageable.data_ptr())
    rc = nat.raw().pa_swap_blocks(ctypes.cast(src, ctypes.c_void_p),
                                  ctypes.cast(dst, ctypes.c_void_p), 1,
                                  pairs.data_ptr(), 1, 16 * 2 * 64 * 2, 4, 4,
                                  None, None)
    assert rc == pa.PA_ERR_INVALID_ARG


def test_swap_bad_pair_sets_flag_and_skips():
    gpu = [torch.randn(6, 16, 2, 64).to(torch.bfloat16).cuda()]
    cpu = [torch.zeros(2, 16, 2, 64, dtype=torch.bfloat16).pin_memory()]
    pairs = torch.tensor([[5, 2], [1, 0]], dtype=torch.int64, device="cuda")
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_swap_blocks(gpu, cpu, pairs, error_flags=flags)
    torch.cuda.synchronize()
    assert int(flags.item()) & pa.PA_DEVERR_COPY_PAIR
    assert torch.equal(cpu[0][0], gpu[0][1].cpu())
    assert not cpu[0][1].any()

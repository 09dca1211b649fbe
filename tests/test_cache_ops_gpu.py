"""reshape_and_cache and copy_blocks on the GPU through the C ABI, bit-exact
against the oracle (whole pools compared, untouched slots included)."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_435_b200 as pa
from paged_kv_cache_435_b200 import inputs
from tests.helpers import bits

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_gpu():
    assert torch.cuda.is_available(), "GPU test run without a CUDA device"


def sentinel_pool(NB, bs, Hkv, D, fill):
    t = torch.full((NB, bs, Hkv, D), 0, dtype=torch.int16, device="cuda")
    t.fill_(fill)
    return t.view(torch.bfloat16)


@pytest.mark.parametrize("T,NB,bs,Hkv,D", [
    (4, 64, 16, 4, 64),
    (256, 300, 16, 8, 128),
    (33, 40, 32, 8, 128),
    (7, 9, 16, 3, 80),       # vector path, odd head count
    (5, 6, 16, 2, 36),       # scalar path (head_size % 8 != 0)
    (1, 1, 16, 1, 64),
])
def test_reshape_and_cache_bit_exact(T, NB, bs, Hkv, D):
    gen = torch.Generator().manual_seed(T * 7 + D)
    key = torch.randn(T, Hkv, D, generator=gen).to(torch.bfloat16)
    value = torch.randn(T, Hkv, D, generator=gen).to(torch.bfloat16)
    rng = np.random.default_rng(T)
    slots = rng.choice(NB * bs, size=T, replace=False).astype(np.int64)
    if T > 3:
        slots[[1, T - 2]] = -1                     # padding tokens
    kc = sentinel_pool(NB, bs, Hkv, D, 0x7FC1)
    vc = sentinel_pool(NB, bs, Hkv, D, 0x7F3E)
    ek, ev = bits(kc), bits(vc)
    pa.pa_reshape_and_cache(key.cuda(), value.cuda(), kc, vc,
                            torch.from_numpy(slots).cuda())
    torch.cuda.synchronize()
    oracle.reshape_and_cache(key, value, ek, ev, slots)
    np.testing.assert_array_equal(bits(kc), ek)
    np.testing.assert_array_equal(bits(vc), ev)


def test_reshape_and_cache_strided_key_from_fused_qkv():
    # key/value as views into a fused [T, (Hq + 2*Hkv) * D] projection output.
    T, Hq, Hkv, D, bs, NB = 64, 8, 2, 128, 16, 10
    gen = torch.Generator().manual_seed(3)
    qkv = torch.randn(T, (Hq + 2 * Hkv) * D, generator=gen).to(torch.bfloat16).cuda()
    key = qkv[:, Hq * D:(Hq + Hkv) * D].view(T, Hkv, D)
    value = qkv[:, (Hq + Hkv) * D:].view(T, Hkv, D)
    assert key.stride(0) == (Hq + 2 * Hkv) * D
    slots = torch.arange(T, dtype=torch.int64) * 2 + 1
    kc = sentinel_pool(NB, bs, Hkv, D, 0x1234)
    vc = sentinel_pool(NB, bs, Hkv, D, 0x4321)
    ek, ev = bits(kc), bits(vc)
    pa.pa_reshape_and_cache(key, value, kc, vc, slots.cuda())
    torch.cuda.synchronize()
    oracle.reshape_and_cache(key.cpu().contiguous(), value.cpu().contiguous(),
                             ek, ev, slots.numpy())
    np.testing.assert_array_equal(bits(kc), ek)
    np.testing.assert_array_equal(bits(vc), ev)


def test_reshape_and_cache_out_of_range_slot_sets_flag_and_skips():
    T, NB, bs, Hkv, D = 3, 4, 16, 2, 64
    key = torch.randn(T, Hkv, D).to(torch.bfloat16).cuda()
    kc = sentinel_pool(NB, bs, Hkv, D, 0x7FC1)
    vc = sentinel_pool(NB, bs, Hkv, D, 0x7FC1)
    before = bits(kc)
    slots = torch.tensor([NB * bs, NB * bs + 1000, -5], dtype=torch.int64).cuda()
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_reshape_and_cache(key, key, kc, vc, slots, error_flags=flags)
    torch.cuda.synchronize()
    assert int(flags.item()) & pa.PA_DEVERR_SLOT
    np.testing.assert_array_equal(bits(kc), before)


@pytest.mark.parametrize("layers", [1, 3, 130])
def test_copy_blocks_bit_exact(layers):
    NB, bs, Hkv, D = 24, 16, 2, 64
    gen = torch.Generator().manual_seed(layers)
    ks = [torch.randn(NB, bs, Hkv, D, generator=gen).to(torch.bfloat16).cuda()
          for _ in range(layers)]
    vs = [torch.randn(NB, bs, Hkv, D, generator=gen).to(torch.bfloat16).cuda()
          for _ in range(layers)]
    pairs = np.array([[0, 7], [3, 9], [3, 11], [15, 2], [4, 4], [23, 22]],
                     dtype=np.int64)
    ek = [bits(k) for k in ks]
    ev = [bits(v) for v in vs]
    pa.pa_copy_blocks(ks, vs, torch.from_numpy(pairs).cuda())
    torch.cuda.synchronize()
    oracle.copy_blocks(ek, ev, pairs)
    for a, b in zip(ks + vs, ek + ev):
        np.testing.assert_array_equal(bits(a), b)


def test_copy_blocks_bad_pair_sets_flag_and_skips():
    NB, bs, Hkv, D = 8, 16, 2, 64
    k = torch.randn(NB, bs, Hkv, D).to(torch.bfloat16).cuda()
    v = torch.randn(NB, bs, Hkv, D).to(torch.bfloat16).cuda()
    before_k, before_v = bits(k), bits(v)
    pairs = torch.tensor([[0, NB], [-1, 2], [1, 3]], dtype=torch.int64).cuda()
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_copy_blocks([k], [v], pairs, error_flags=flags)
    torch.cuda.synchronize()
    assert int(flags.item()) & pa.PA_DEVERR_COPY_PAIR
    oracle.copy_blocks([before_k], [before_v], np.array([[1, 3]], np.int64))
    np.testing.assert_array_equal(bits(k), before_k)
    np.testing.assert_array_equal(bits(v), before_v)


def test_shared_prefix_cow_step_pools_bit_exact():
    """The CoW workload's pool writes (256 block copies, then 256 new
    tokens) match the oracle bit for bit over the whole pool."""
    case = inputs.make_case("shared_prefix_cow", device="cuda")
    ek, ev = bits(case.k_cache), bits(case.v_cache)
    pa.pa_copy_blocks([case.k_cache], [case.v_cache], case.copy_pairs)
    pa.pa_reshape_and_cache(case.new_key, case.new_value, case.k_cache,
                            case.v_cache, case.slot_mapping)
    torch.cuda.synchronize()
    oracle.copy_blocks([ek], [ev], case.copy_pairs.cpu().numpy())
    oracle.reshape_and_cache(case.new_key.cpu(), case.new_value.cpu(), ek, ev,
                             case.slot_mapping.cpu().numpy())
    np.testing.assert_array_equal(bits(case.k_cache), ek)
    np.testing.assert_array_equal(bits(case.v_cache), ev)

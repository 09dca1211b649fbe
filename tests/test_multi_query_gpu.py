"""pa_multi_query_attention on the GPU through the C ABI against the fp64
oracle: k causal query tokens per sequence (speculative verification,
chunked-prefill chunks, whole-prompt prefill), the step's K/V written first
with pa_reshape_and_cache.  Tolerance as for decode: max-abs <= 4e-3 and
relative L2 <= 1e-3; cache writes bit-exact."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_435_b200 as pa
from paged_kv_cache_435_b200 import inputs
from tests.helpers import assert_attn_close, bits

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_gpu():
    assert torch.cuda.is_available(), "GPU test run without a CUDA device"


def gpu_mq(case, flags=None, write=True):
    if write:
        pa.pa_reshape_and_cache(case.new_key, case.new_value, case.k_cache,
                                case.v_cache, case.slot_mapping,
                                error_flags=flags)
    out = torch.empty(case.q.shape, dtype=torch.float32, device="cuda")
    pa.pa_multi_query_attention(out, case.q, case.k_cache, case.v_cache,
                                case.block_tables, case.context_lens,
                                case.query_start_loc, case.max_context_len,
                                int(case.query_lens_np.max(initial=0)),
                                case.scale, error_flags=flags)
    return out


def check(case):
    ek, ev = bits(case.k_cache), bits(case.v_cache)
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = gpu_mq(case, flags)
    torch.cuda.synchronize()
    assert int(flags.item()) == 0
    oracle.reshape_and_cache(case.new_key.cpu(), case.new_value.cpu(), ek, ev,
                             case.slot_mapping.cpu().numpy())
    np.testing.assert_array_equal(bits(case.k_cache), ek)
    ref = oracle.paged_multi_query_attention(
        case.q.cpu(), ek, ev, case.tables_np, case.lens_np.astype(np.int32),
        case.query_start_loc.cpu().numpy(), case.scale,
        case.workload.num_kv_heads)
    return assert_attn_close(out, ref, case.workload.name), out


@pytest.mark.parametrize("Hq,Hkv,D,bs,lens,qlens", [
    (64, 8, 128, 16, [300, 1000, 17, 4096], [4, 4, 4, 4]),     # spec verify
    (32, 8, 128, 32, [700, 64, 129], [5, 3, 8]),
    (16, 16, 128, 16, [257, 40, 90], [2, 1, 7]),                # MHA
    (8, 2, 64, 16, [600, 33, 512, 5], [128, 33, 100, 0]),       # chunks
    (28, 4, 64, 32, [100, 70], [100, 19]),                       # G=7, k=L
    (4, 4, 128, 16, [1, 2, 3], [1, 2, 3]),
    (32, 2, 128, 16, [2048, 300], [200, 64]),                    # G=16
])
def test_multi_query_shapes(Hq, Hkv, D, bs, lens, qlens):
    case = inputs.multi_query_case(len(lens), Hq, Hkv, D, bs, lens, qlens,
                                   seed=sum(lens) + Hq, device="cuda")
    check(case)


def test_single_query_matches_decode_kernel():
    lens = [1, 15, 16, 17, 100, 1000, 3000]
    case = inputs.multi_query_case(len(lens), 32, 8, 128, 16, lens,
                                   [1] * len(lens), seed=2, device="cuda")
    (_, _), mq = check(case)
    B, Hq, D = case.q.shape
    dec = torch.empty(B, Hq, D, dtype=torch.float32, device="cuda")
    nbytes = pa.pa_decode_workspace_size(B, Hq, 8, D, 16, case.max_context_len)
    ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device="cuda")
    pa.pa_decode_attention(dec, case.q, case.k_cache, case.v_cache,
                           case.block_tables, case.context_lens,
                           case.max_context_len, case.scale, workspace=ws)
    torch.cuda.synchronize()
    assert (mq - dec).abs().max().item() <= 2e-5


def test_speculative_verify_batch256():
    """Batch-256 GQA layer (64q/8kv, D=128, L~U[256,4096]) verifying 4 draft
    tokens per sequence; every row of every sequence compared."""
    rng = np.random.default_rng(1003)
    lens = rng.integers(256, 4097, size=256)
    case = inputs.multi_query_case(256, 64, 8, 128, 16, lens, [4] * 256,
                                   seed=77, device="cuda")
    check(case)


def test_speculative_verify_workload():
    """The benchmark's speculative-verification workload, compared in full."""
    case = inputs.make_case("spec_verify_70b_b256", device="cuda")
    check(case)


def test_run_to_run_determinism():
    case = inputs.multi_query_case(3, 32, 4, 128, 16, [500, 90, 2000],
                                   [40, 9, 6], seed=5, device="cuda")
    a = gpu_mq(case, write=False)
    b = gpu_mq(case, write=False)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_query_count_above_context_sets_flag():
    case = inputs.multi_query_case(2, 8, 2, 64, 16, [20, 30], [4, 4], seed=9,
                                   device="cuda")
    case.query_start_loc[2] = 40          # seq 1 claims 36 queries > 30 tokens
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty(40, 8, 64, dtype=torch.float32, device="cuda")
    q = torch.zeros(40, 8, 64, dtype=torch.bfloat16, device="cuda")
    pa.pa_multi_query_attention(out, q, case.k_cache, case.v_cache,
                                case.block_tables, case.context_lens,
                                case.query_start_loc, 30, 30, case.scale,
                                error_flags=flags)
    torch.cuda.synchronize()
    assert int(flags.item()) & pa.PA_DEVERR_QUERY_LEN


ROWS_SHAPES = [
    (64, 8, 128, 16, [300, 1000, 17, 4096], [4, 4, 4, 4]),      # spec verify
    (32, 8, 128, 32, [700, 64, 129], [5, 3, 8]),
    (16, 16, 128, 16, [257, 40, 90], [2, 1, 7]),                # MHA
    (4, 4, 128, 16, [1, 2, 3], [1, 2, 3]),
    (32, 2, 128, 16, [2048, 300], [200, 64]),                   # G=16, 100 tiles
    (24, 8, 128, 16, [129, 128, 127, 1000], [11, 1, 16, 3]),    # G=3, ragged tiles
]


@pytest.mark.parametrize("Hq,Hkv,D,bs,lens,qlens", ROWS_SHAPES)
def test_multi_row_kernel_shapes(monkeypatch, Hq, Hkv, D, bs, lens, qlens):
    """The tcgen05 kernel for <= 32 rows per tile (tokens as the MMA's M),
    forced for every shape: 32-row tiles of (query token, head) rows."""
    monkeypatch.setenv("PA_MULTI_QUERY_KERNEL", "rows")
    case = inputs.multi_query_case(len(lens), Hq, Hkv, D, bs, lens, qlens,
                                   seed=sum(lens) + Hq + 1, device="cuda")
    check(case)


def test_multi_row_kernel_spec_verify_batch256(monkeypatch):
    monkeypatch.setenv("PA_MULTI_QUERY_KERNEL", "rows")
    test_speculative_verify_batch256()


def test_multi_row_kernel_determinism(monkeypatch):
    monkeypatch.setenv("PA_MULTI_QUERY_KERNEL", "rows")
    test_run_to_run_determinism()


@pytest.mark.parametrize("Hq,Hkv,D,bs,lens,qlens", ROWS_SHAPES[:3])
def test_mma_kernel_head128_shapes(monkeypatch, Hq, Hkv, D, bs, lens, qlens):
    """The mma.sync kernel, forced at head_size 128 (the default there is the
    tcgen05 kernel), stays exact."""
    monkeypatch.setenv("PA_MULTI_QUERY_KERNEL", "mma")
    case = inputs.multi_query_case(len(lens), Hq, Hkv, D, bs, lens, qlens,
                                   seed=sum(lens) + Hq + 2, device="cuda")
    check(case)


def test_multi_row_kernel_long_context(monkeypatch):
    """A 131072-token sequence (1024 chunks of 128 tokens, piece windows
    walking 8192 blocks) beside short ones, 4 draft tokens each, G = 8."""
    monkeypatch.setenv("PA_MULTI_QUERY_KERNEL", "rows")
    case = inputs.multi_query_case(3, 16, 2, 128, 16, [131072, 300, 17],
                                   [4, 4, 4], seed=131, device="cuda")
    check(case)


@pytest.mark.parametrize("kernel", ["rows", "tc", "mma"])
def test_bad_first_block_id_sets_flag_without_fault(monkeypatch, kernel):
    """Sequence 1's first block id is out of range: every row of it has its
    first visible token there (the 32-row kernel's scheduler reads that K
    row for the row's reference).  The flag is set, nothing faults, and the
    other sequences' outputs stay exact."""
    monkeypatch.setenv("PA_MULTI_QUERY_KERNEL", kernel)
    case = inputs.multi_query_case(3, 32, 8, 128, 16, [300, 200, 129], [4, 4, 4],
                                   seed=77, device="cuda")
    ek, ev = bits(case.k_cache), bits(case.v_cache)
    case.block_tables[1, 0] = case.k_cache.shape[0] + 3      # out of range
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = gpu_mq(case, flags)
    torch.cuda.synchronize()
    assert int(flags.item()) & pa.PA_DEVERR_BLOCK_ID
    oracle.reshape_and_cache(case.new_key.cpu(), case.new_value.cpu(), ek, ev,
                             case.slot_mapping.cpu().numpy())
    tables = case.tables_np.copy()
    qsl = case.query_start_loc.cpu().numpy()
    ref = oracle.paged_multi_query_attention(
        case.q.cpu(), ek, ev, tables, case.lens_np.astype(np.int32), qsl,
        case.scale, case.workload.num_kv_heads)
    for s in (0, 2):
        a, b = int(qsl[s]), int(qsl[s + 1])
        assert_attn_close(out[a:b], ref[a:b], f"seq {s} beside a bad table ({kernel})")


@pytest.mark.parametrize("scale", [1.0, 4.0])
def test_multi_row_kernel_large_logits(monkeypatch, scale):
    """Scale 1 and 4 instead of 1/sqrt(D): logits of tens to hundreds (log2
    units), a sharply peaked softmax.  The 32-row kernel's reference (each
    row's logit at its first token, summed by the scheduler apart from the
    tensor core's S) and its growth check must keep every row exact."""
    monkeypatch.setenv("PA_MULTI_QUERY_KERNEL", "rows")
    case = inputs.multi_query_case(4, 64, 8, 128, 16, [300, 1000, 17, 2049],
                                   [4, 4, 4, 4], seed=4100 + int(scale), device="cuda")
    case.scale_override = scale
    (_, _), out = check(case)
    assert torch.isfinite(out).all()

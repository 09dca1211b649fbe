"""The tcgen05 multi-query kernel (128-row tiles, TMEM accumulators) against
the fp64 oracle, and against the mma.sync kernel on the same inputs.  The
kernel choice is forced with PA_MULTI_QUERY_KERNEL."""
import os

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


def run(case, kernel, write=True):
    old = os.environ.get("PA_MULTI_QUERY_KERNEL")
    os.environ["PA_MULTI_QUERY_KERNEL"] = kernel
    try:
        flags = torch.zeros(1, dtype=torch.int32, device="cuda")
        if write:
            pa.pa_reshape_and_cache(case.new_key, case.new_value, case.k_cache,
                                    case.v_cache, case.slot_mapping)
        out = torch.full(case.q.shape, float("nan"), dtype=torch.float32, device="cuda")
        pa.pa_multi_query_attention(out, case.q, case.k_cache, case.v_cache,
                                    case.block_tables, case.context_lens,
                                    case.query_start_loc, case.max_context_len,
                                    int(case.query_lens_np.max()), case.scale,
                                    error_flags=flags)
        torch.cuda.synchronize()
        assert int(flags.item()) == 0, int(flags.item())
        return out
    finally:
        if old is None:
            del os.environ["PA_MULTI_QUERY_KERNEL"]
        else:
            os.environ["PA_MULTI_QUERY_KERNEL"] = old


def oracle_out(case):
    return oracle.paged_multi_query_attention(
        case.q.cpu(), bits(case.k_cache), bits(case.v_cache), case.tables_np,
        case.lens_np.astype(np.int32), case.query_start_loc.cpu().numpy(),
        case.scale, case.workload.num_kv_heads)


@pytest.mark.parametrize("Hq,Hkv,bs,lens,qlens", [
    (8, 1, 16, [64], [16]),                        # one tile, one chunk
    (64, 8, 16, [300, 1000, 40], [64, 200, 17]),  # chunks, partial tiles
    (32, 8, 32, [700, 129], [96, 129]),           # bs 32, whole-prompt prefill
    (16, 2, 16, [2049, 513], [512, 300]),         # long causal ranges
])
def test_tc_kernel_matches_oracle(Hq, Hkv, bs, lens, qlens):
    case = inputs.multi_query_case(len(lens), Hq, Hkv, 128, bs, lens, qlens,
                                   seed=sum(lens) + 5 * Hq, device="cuda")
    out = run(case, "tc")
    assert torch.isfinite(out).all()
    assert_attn_close(out, oracle_out(case), "tcgen05 multi-query")


def test_tc_and_mma_kernels_agree():
    case = inputs.multi_query_case(3, 64, 8, 128, 16, [1500, 260, 700],
                                   [128, 64, 300], seed=31, device="cuda")
    a = run(case, "tc")
    b = run(case, "mma", write=False)
    assert (a - b).abs().max().item() <= 2e-4


def test_tc_large_logits_rescale_path():
    # scale 1.0 makes logits large and forces the O rescale in TMEM.
    case = inputs.multi_query_case(2, 16, 2, 128, 16, [900, 400], [128, 64],
                                   seed=12, device="cuda")
    case.scale_override = 1.0
    out = run(case, "tc")
    assert torch.isfinite(out).all()
    assert_attn_close(out, oracle_out(case), "tcgen05 rescale")


@pytest.mark.parametrize("kernel", ["tc", "rows"])
def test_late_dominant_keys_force_the_rescale(kernel):
    """Keys of all 64 at token 300 and of all 128 at token 700 (after the
    first chunk sets the softmax reference) give every row whose query sums
    to a positive value a logit tens of powers of two above that reference:
    the tcgen05 kernel's chunk-sum check must take the exact path (max, O and
    sums rescaled) once or twice per row; the 32-row kernel's rescale too."""
    case = inputs.multi_query_case(2, 16, 2, 128, 16, [900, 400], [128, 64],
                                   seed=44, device="cuda")
    bs = case.workload.block_size
    for s, t, val in [(0, 300, 64.0), (0, 700, 128.0), (1, 200, 64.0)]:
        blk = int(case.tables_np[s][t // bs])
        case.k_cache[blk, t % bs] = val
    out = run(case, kernel)
    assert torch.isfinite(out).all()
    assert_attn_close(out, oracle_out(case), f"{kernel}: late dominant keys")

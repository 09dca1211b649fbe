"""pa_decode_attention on the GPU through the C ABI against the fp64 oracle.

Every named workload runs as a whole decode step (copy_blocks when it has CoW
pairs, reshape_and_cache, attention) in the launch configuration the
benchmark uses; the oracle recomputes the step on the host from the same
pre-step pool.  Every workload is compared in full: every output element of
every sequence and head.  Tolerance: max-abs <= 4e-3 and relative L2 <= 1e-3
over the whole output; cache writes bit-exact over the whole pool.
"""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_435_b200 as pa
from paged_kv_cache_435_b200 import inputs
from tests.helpers import (assert_attn_close, bits, gpu_step, oracle_attention,
                           oracle_pools_after_step)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_gpu():
    assert torch.cuda.is_available(), "GPU test run without a CUDA device"


def run_and_check(case, seqs=None, partition_size=0, check_pools=True):
    ek, ev = bits(case.k_cache), bits(case.v_cache)
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    launches0 = pa.pa_launch_count()
    out = gpu_step(case, partition_size=partition_size, error_flags=flags)
    torch.cuda.synchronize()
    assert pa.pa_launch_count() > launches0
    assert int(flags.item()) == 0
    oracle_pools_after_step(case, ek, ev)
    if check_pools:
        np.testing.assert_array_equal(bits(case.k_cache), ek)
        np.testing.assert_array_equal(bits(case.v_cache), ev)
    ref = oracle_attention(case, ek, ev, seqs)
    got = out if seqs is None else out[torch.from_numpy(np.asarray(seqs)).cuda()]
    return assert_attn_close(got, ref, case.workload.name), out


# ---------------------------------------------------------------- workloads
def test_tiny_workload_full():
    case = inputs.make_case("tiny", device="cuda")
    (max_abs, rel), out = run_and_check(case)
    # context length 1: the output is that token's value, exactly
    v1 = case.new_value[0].float()                  # seq 0 has L = 1
    G = case.workload.num_heads // case.workload.num_kv_heads
    for h in range(case.workload.num_heads):
        assert torch.equal(out[0, h], v1[h // G])


def test_llama2_7b_mha_workload():
    case = inputs.make_case("llama2_7b_mha", device="cuda")
    run_and_check(case)


def test_llama2_70b_gqa_batch256_workload():
    # The benchmark's workload in the benchmark's launch configuration (the
    # library's partition heuristic), all 256 sequences x 64 heads compared.
    case = inputs.make_case("llama2_70b_gqa_b256", device="cuda")
    run_and_check(case)


def test_shared_prefix_cow_workload():
    # The plain decode call on the copy-on-write workload, every sequence.
    case = inputs.make_case("shared_prefix_cow", device="cuda")
    run_and_check(case)


@pytest.mark.parametrize("name", ["long_skew_bs16", "long_skew_bs32"])
def test_long_skew_split_kv_workload(name):
    case = inputs.make_case(name, device="cuda")
    w = case.workload
    part = pa.pa_decode_partition_size(w.num_seqs, w.num_heads, w.num_kv_heads,
                                       w.head_size, w.block_size,
                                       case.max_context_len, w.partition_size)
    assert part == 512
    run_and_check(case, partition_size=w.partition_size)


# ---------------------------------------------------------------- shapes
@pytest.mark.parametrize("Hq,Hkv,D,bs", [
    (4, 4, 64, 16), (8, 4, 64, 32), (16, 4, 128, 16), (16, 2, 128, 32),
    (24, 3, 128, 16), (7, 7, 128, 16), (6, 2, 64, 16), (5, 1, 128, 32),
])
def test_shapes_and_ragged_lengths(Hq, Hkv, D, bs):
    lens = [1, 15, 16, 17, 31, 32, 33, 63, 64, 65, 100, 257, 1000, 0, 2]
    case = inputs.custom_case(len(lens), Hq, Hkv, D, bs, lens,
                              seed=Hq * 100 + D + bs, device="cuda")
    (_, _), out = run_and_check(case)
    # the empty context gives zeros
    assert torch.count_nonzero(out[13]) == 0


@pytest.mark.parametrize("partition", [16, 32, 64, 128, 512])
def test_forced_partitions_agree_with_oracle(partition):
    lens = [1, 16, 17, 100, 511, 512, 513, 2000, 4097]
    bs = 32 if partition % 32 == 0 else 16
    case = inputs.custom_case(len(lens), 16, 2, 128, bs, lens, seed=partition,
                              device="cuda")
    run_and_check(case, partition_size=partition)


@pytest.mark.parametrize("D,bs,partition", [(128, 16, 256), (64, 32, 128)])
def test_split_grid_beyond_the_persistent_limit(D, bs, partition):
    # More than 768 sequences with a split: the partition kernel runs on the
    # plain grid (one CTA per kv head, partition and sequence, early exit past
    # a sequence's end) instead of the persistent compact-item grid.
    rng = np.random.default_rng(800 + D)
    lens = rng.integers(1, 1300, size=800)
    lens[:4] = [0, 1, partition, partition + 1]
    case = inputs.custom_case(len(lens), 16, 2, D, bs, lens, seed=900 + D,
                              device="cuda")
    run_and_check(case, partition_size=partition)


def test_split_and_unsplit_agree():
    lens = [3000, 5, 700, 1601]
    outs = []
    for part in (0, 64, 512):
        case = inputs.custom_case(len(lens), 32, 8, 128, 16, lens, seed=77,
                                  device="cuda")
        outs.append(gpu_step(case, partition_size=part, do_write=False))
    torch.cuda.synchronize()
    for o in outs[1:]:
        diff = (o - outs[0]).abs().max().item()
        assert diff <= 2e-5, diff


def test_run_to_run_bitwise_determinism():
    case = inputs.custom_case(8, 64, 8, 128, 16, [4096, 1, 300, 2222, 17, 999,
                                                   3000, 64], seed=5,
                              device="cuda")
    a = gpu_step(case, do_write=False)
    b = gpu_step(case, do_write=False)
    c = gpu_step(case, partition_size=256, do_write=False)
    d = gpu_step(case, partition_size=256, do_write=False)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    assert torch.equal(c, d)


def test_single_token_contexts_return_value_exactly():
    lens = [1] * 6
    case = inputs.custom_case(6, 32, 8, 128, 16, lens, seed=9, device="cuda")
    out = gpu_step(case)
    torch.cuda.synchronize()
    for s in range(6):
        for h in range(32):
            assert torch.equal(out[s, h], case.new_value[s, h // 4].float())


def test_large_logits_stay_finite_and_accurate():
    # Scale 1.0 instead of 1/sqrt(D): logits of magnitude ~10, a peaked
    # softmax; the online rescaling must keep everything finite.
    lens = [700, 33, 2048]
    case = inputs.custom_case(3, 16, 2, 128, 16, lens, seed=31, device="cuda")
    case.scale_override = 1.0
    run_and_check(case)


# ---------------------------------------------------------------- errors
def test_bad_block_id_sets_flag_without_fault():
    lens = [40, 40]
    case = inputs.custom_case(2, 8, 2, 64, 16, lens, seed=3, device="cuda")
    case.block_tables[1, 1] = case.k_cache.shape[0] + 5       # out of range
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = gpu_step(case, error_flags=flags, do_write=False)
    torch.cuda.synchronize()
    assert int(flags.item()) & pa.PA_DEVERR_BLOCK_ID
    # the untouched sequence is still right
    ek, ev = bits(case.k_cache), bits(case.v_cache)
    ref = oracle_attention(case, ek, ev, seqs=[0])
    assert_attn_close(out[:1], ref, "seq 0 beside a bad table")


def test_context_len_above_bound_sets_flag():
    lens = [40, 20]
    case = inputs.custom_case(2, 8, 2, 64, 16, lens, seed=4, device="cuda")
    case.context_lens[1] = 10_000                           # > max_context_len
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    B, Hq, D = case.q.shape
    out = torch.empty(B, Hq, D, device="cuda")
    pa.pa_decode_attention(out, case.q, case.k_cache, case.v_cache,
                           case.block_tables, case.context_lens, 40,
                           case.scale, error_flags=flags)
    torch.cuda.synchronize()
    assert int(flags.item()) & pa.PA_DEVERR_CONTEXT_LEN


def test_workspace_too_small_is_rejected_before_launch():
    lens = [600, 700]
    case = inputs.custom_case(2, 8, 2, 64, 16, lens, seed=6, device="cuda")
    out = torch.empty(2, 8, 64, device="cuda")
    ws = torch.empty(64, dtype=torch.uint8, device="cuda")
    n0 = pa.pa_launch_count()
    with pytest.raises(pa.PAError) as e:
        pa.pa_decode_attention(out, case.q, case.k_cache, case.v_cache,
                               case.block_tables, case.context_lens, 700,
                               case.scale, partition_size=64, workspace=ws)
    assert e.value.status == pa.PA_ERR_WORKSPACE
    assert pa.pa_launch_count() == n0


@pytest.mark.parametrize("seed", range(4))
def test_random_split_batches(seed):
    """Randomised long-context batches on the persistent split path: a few
    long sequences (so their merge runs as CTA slices, more than 16 candidate
    rows) among many short ones that straddle worker boundaries (merged
    whole by one warp each), with random head shapes, head size, block size
    and a forced partition size.  Every output is compared with the oracle."""
    rng = np.random.default_rng(6000 + seed)
    Hkv = int(rng.choice([1, 2, 4, 8]))
    G = int(rng.choice([1, 2, 4, 8]))
    D = int(rng.choice([64, 128]))
    bs = int(rng.choice([16, 32]))
    part = int(rng.choice([128, 256, 512]))
    n_long = int(rng.integers(1, 4))
    lens = list(rng.integers(8000, 40000, size=n_long)) + \
        list(rng.integers(0, 1200, size=int(rng.integers(20, 200))))
    rng.shuffle(lens)
    case = inputs.custom_case(len(lens), G * Hkv, Hkv, D, bs, lens, seed=7000 + seed,
                              device="cuda")
    run_and_check(case, partition_size=part)

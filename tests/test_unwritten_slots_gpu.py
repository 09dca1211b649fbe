"""Cache slots that hold no token of any context (the rows after the last
token of a sequence's last block, blocks no table reaches) may contain
anything: a pool is allocated, not cleared ("PagedAttention": a block is
filled left to right, so the last block of a sequence is partly empty).
These tests fill every such slot of K and V with NaN and infinities and
compare the attention of every kernel with the fp64 oracle, which reads
only the first L tokens of each sequence.  Tolerance as for decode:
max-abs <= 4e-3 and relative L2 <= 1e-3, and every output finite."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_435_b200 as pa
from paged_kv_cache_435_b200 import inputs
from tests.helpers import (assert_attn_close, bits, gpu_step, oracle_attention,
                           poison_unwritten_slots)

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_gpu():
    assert torch.cuda.is_available(), "GPU test run without a CUDA device"


RAGGED = [1, 15, 17, 31, 33, 100, 257, 1000, 0, 2, 4095, 130]


@pytest.mark.parametrize("Hq,Hkv,D,bs,partition", [
    (32, 32, 128, 16, 0),      # MHA, whole sequences
    (64, 8, 128, 16, 0),       # GQA 8
    (64, 8, 128, 32, 512),     # forced split + merge
    (16, 2, 128, 16, 64),      # many partitions per sequence
    (16, 4, 64, 16, 0),        # head size 64
    (16, 4, 64, 32, 128),      # head size 64, split
])
def test_decode_ignores_unwritten_slots(Hq, Hkv, D, bs, partition):
    case = inputs.custom_case(len(RAGGED), Hq, Hkv, D, bs, RAGGED,
                              seed=7000 + Hq + D + bs + partition, device="cuda")
    assert poison_unwritten_slots(case) > 0
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = gpu_step(case, partition_size=partition, error_flags=flags,
                   do_copy=False, do_write=False)
    torch.cuda.synchronize()
    assert int(flags.item()) == 0
    ref = oracle_attention(case, bits(case.k_cache), bits(case.v_cache))
    assert_attn_close(out, ref, "decode")


@pytest.mark.parametrize("kernel", ["rows", "tc", "mma"])
@pytest.mark.parametrize("Hq,Hkv,bs,lens,qlens", [
    (64, 8, 16, [300, 1000, 17, 4095, 129], [4, 4, 4, 4, 1]),    # spec verify
    (32, 8, 32, [700, 65, 129, 31], [5, 3, 8, 31]),
    (24, 8, 16, [129, 127, 1000, 2], [11, 16, 3, 2]),            # G = 3
])
def test_multi_query_ignores_unwritten_slots(monkeypatch, kernel, Hq, Hkv, bs, lens, qlens):
    run_multi_query(monkeypatch, kernel, Hq, Hkv, 128, bs, lens, qlens)


@pytest.mark.parametrize("bs", [16, 32])
def test_multi_query_head64_ignores_unwritten_slots(monkeypatch, bs):
    """Head size 64 runs on the mma.sync kernel."""
    run_multi_query(monkeypatch, "mma", 16, 4, 64, bs, [300, 65, 129, 31, 1000],
                    [5, 3, 8, 31, 64])


def run_multi_query(monkeypatch, kernel, Hq, Hkv, D, bs, lens, qlens):
    monkeypatch.setenv("PA_MULTI_QUERY_KERNEL", kernel)
    case = inputs.multi_query_case(len(lens), Hq, Hkv, D, bs, lens, qlens,
                                   seed=7100 + sum(lens) + Hq + D, device="cuda")
    assert poison_unwritten_slots(case) > 0
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_reshape_and_cache(case.new_key, case.new_value, case.k_cache,
                            case.v_cache, case.slot_mapping, error_flags=flags)
    out = torch.empty(case.q.shape, dtype=torch.float32, device="cuda")
    pa.pa_multi_query_attention(out, case.q, case.k_cache, case.v_cache,
                                case.block_tables, case.context_lens,
                                case.query_start_loc, case.max_context_len,
                                int(case.query_lens_np.max(initial=0)),
                                case.scale, error_flags=flags)
    torch.cuda.synchronize()
    assert int(flags.item()) == 0
    ref = oracle.paged_multi_query_attention(
        case.q.cpu(), bits(case.k_cache), bits(case.v_cache), case.tables_np,
        case.lens_np.astype(np.int32), case.query_start_loc.cpu().numpy(),
        case.scale, case.workload.num_kv_heads)
    assert_attn_close(out, ref, f"multi-query {kernel}")


def _shared_prefix(case):
    B, Hq, D = case.q.shape
    Hkv, bs = case.workload.num_kv_heads, case.workload.block_size
    out = torch.full((B, Hq, D), float("nan"), dtype=torch.float32, device="cuda")
    nbytes = pa.pa_shared_prefix_workspace_size(B, Hq, Hkv, D, bs,
                                                case.max_context_len, 0)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_decode_attention_shared_prefix(
        out, case.q, case.k_cache, case.v_cache, case.block_tables,
        case.context_lens, case.group_start.cuda(), case.prefix_lens.cuda(),
        case.max_context_len, case.max_group_size, case.scale, ws,
        error_flags=flags)
    torch.cuda.synchronize()
    assert int(flags.item()) == 0
    return out


@pytest.mark.parametrize("G,Hkv,bs,split", [
    (4, 8, 16, False),     # the parallel-sampling shape
    (8, 2, 32, False),
    (4, 2, 16, True),      # one dominant group: its pass is cut into pieces
])
def test_shared_prefix_ignores_unwritten_slots(G, Hkv, bs, split):
    """Groups whose members end inside the prefix, members with empty and
    one-token tails, tails that end mid-block, lone sequences between the
    groups: the shared blocks past the longest member and every tail's
    padding are poisoned."""
    rng = np.random.default_rng(7200 + G + Hkv + bs)
    lens, gs, pl = [], [], []
    for gi in range(12):
        m = int(rng.integers(1, 32 // G + 1))
        P = int(rng.integers(1, 30)) * bs
        tails = rng.integers(0, 3000 if (split and gi == 0) else 200, size=m)
        start = len(lens)
        lens += [int(P + t) for t in tails]
        if m > 1:
            lens[start] = int(rng.integers(1, P))           # ends inside the prefix
        if m > 2:
            lens[start + 1] = P + 1                         # one-token tail
        gs.append(start)
        pl.append(P)
        if gi % 4 == 3:
            lens.append(int(rng.integers(1, 700)))          # a lone sequence
    gs.append(len(lens))
    lens.append(77)
    case = inputs.grouped_case(G * Hkv, Hkv, 128, bs, lens, gs, pl,
                               seed=7300 + G + bs, device="cuda")
    assert poison_unwritten_slots(case) > 0
    out = _shared_prefix(case)
    ref = oracle.paged_decode_attention(
        case.q.cpu(), bits(case.k_cache), bits(case.v_cache), case.tables_np,
        case.lens_np.astype(np.int32), case.scale, Hkv)
    assert_attn_close(out, ref, "shared prefix")

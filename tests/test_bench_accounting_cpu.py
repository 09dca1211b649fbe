"""bench.py's accounting, which every roofline figure divides by, against
counts made independently: the per-token formula written out by hand for
the tiny workload, distinct cached positions counted from the block tables,
and (query, visible token) pairs enumerated one by one."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from paged_kv_cache_435_b200 import inputs  # noqa: E402


def test_tiny_workload_bytes_by_hand():
    """B = 4, L = {1, 16, 17, 100}, Hq = Hkv = 4, D = 64, bs = 16; one new
    token per sequence written first.  KV: 134 tokens x (K and V) x 4 heads
    x 64 x 2 bytes = 137216; q 4 x 4 x 64 x 2 = 2048; fp32 out 4096; block
    table entries 1 + 1 + 2 + 7 = 11 x 4 = 44; lengths 16.  The cache write
    reads and writes 4 rows of K and of V (4 x 512 bytes each way) and reads
    4 int64 slots."""
    case = inputs.make_case("tiny")
    assert list(case.lens_np) == [1, 16, 17, 100]
    assert bench.attention_bytes(case) == 137216 + 2048 + 4096 + 44 + 16
    assert bench.step_bytes(case) == 143420 + 2 * 2 * 4 * 512 + 4 * 8
    assert bench.attention_flops(case) == 134 * 4 * 4 * 64


def test_unique_tokens_are_the_distinct_cached_positions():
    """Shared prefixes are counted once: compare with the number of distinct
    (block, offset) positions the block tables reach."""
    bs = 16
    lens = [64 + 5, 64 + 40, 30, 64, 200, 17]
    case = inputs.grouped_case(8, 2, 64, bs, lens, [0, 4], [64], seed=9)
    seen = set()
    for s, L in enumerate(case.lens_np):
        for t in range(int(L)):
            seen.add((int(case.tables_np[s, t // bs]), t % bs))
    assert case.unique_tokens == len(seen) < int(case.lens_np.sum())
    w = case.workload
    kv = len(seen) * 2 * w.num_kv_heads * w.head_size * 2
    B = len(lens)
    blocks = sum(-(-L // bs) for L in lens)
    assert bench.attention_bytes(case) == (kv + B * 8 * 64 * 2 + B * 8 * 64 * 4
                                           + blocks * 4 + B * 4)


def test_multi_query_flops_count_causal_pairs():
    lens, qlens = [40, 300, 7], [8, 128, 7]
    case = inputs.multi_query_case(3, 16, 4, 64, 16, lens, qlens, seed=3)
    pairs = 0
    for L, k in zip(lens, qlens):
        for j in range(k):               # query j sits at position L - k + j
            pairs += sum(1 for u in range(L) if u <= L - k + j)
    assert bench.attention_flops(case) == pairs * 4 * 16 * 64
    nq = sum(qlens)
    kv = sum(lens) * 2 * 4 * 64 * 2
    assert bench.attention_bytes(case) == (kv + nq * 16 * 64 * 2 + nq * 16 * 64 * 4
                                           + sum(-(-L // 16) for L in lens) * 4 + 3 * 4)


def test_traffic_is_used_only_for_its_kernel_source_and_workload(tmp_path, monkeypatch):
    dk, mk = "paged_decode_kernel", "paged_multi_row_kernel"
    good = tmp_path / "traffic.txt"
    good.write_text(f"# note\nworkload = w1\nkernel = {dk}\nkernel_sha = {bench.kernel_sha(dk)}\n"
                    "dram_bytes_per_launch = 1234.5\n\n"
                    f"workload = w2\nkernel = {mk}\nkernel_sha = {bench.kernel_sha(mk)}\n"
                    "dram_bytes_per_launch = 99\n")
    monkeypatch.setattr(bench, "PROFILE_TRAFFIC", str(good))
    assert bench.read_traffic("w1", dk) == 1234.5
    assert bench.read_traffic("w2", mk) == 99.0
    assert bench.read_traffic("w2", dk) is None   # another kernel's record
    assert bench.read_traffic("w3", dk) is None
    stale = tmp_path / "stale.txt"
    stale.write_text(f"workload = w1\nkernel = {dk}\nkernel_sha = 0000000000000000\n"
                     "dram_bytes_per_launch = 1234.5\n")
    monkeypatch.setattr(bench, "PROFILE_TRAFFIC", str(stale))
    assert bench.read_traffic("w1", dk) is None
    for k in bench.KERNEL_SOURCES:
        sha = bench.kernel_sha(k)
        assert len(sha) == 16 and all(c in "0123456789abcdef" for c in sha)
    assert bench.kernel_sha(dk) != bench.kernel_sha(mk)


def test_shared_prefix_workload_unique_tokens():
    """32 prompts x 8 samples: 63 shared blocks per prompt, each sample's
    private copy of block 63 and its own tail, counted position by position."""
    case = inputs.make_case("shared_prefix_cow")
    bs = case.workload.block_size
    seen = set()
    for s, L in enumerate(case.lens_np):
        row = case.tables_np[s]
        seen.update((int(row[t // bs]), t % bs) for t in range(int(L)))
    assert case.unique_tokens == len(seen)
    assert case.logical_tokens == int(case.lens_np.sum()) > 4 * len(seen)

"""The seeded input builders that both the oracle and the CUDA path read:
a workload rebuilt from its seeds is bit-identical, block tables are a
permutation of pool ids with -1 past each sequence's last block, and the
structural promises of each workload hold (shared prefixes, copy-on-write
pairs, query placement)."""
import numpy as np
import torch

from paged_kv_cache_435_b200 import inputs


def _same(a, b):
    assert a.shape == b.shape and a.dtype == b.dtype
    assert torch.equal(a.view(torch.int16) if a.dtype == torch.bfloat16 else a,
                       b.view(torch.int16) if b.dtype == torch.bfloat16 else b)


def test_rebuilt_workload_is_bit_identical():
    a = inputs.make_case("tiny")
    b = inputs.make_case("tiny")
    for name in ("q", "k_cache", "v_cache", "new_key", "new_value", "slot_mapping",
                 "block_tables", "context_lens"):
        _same(getattr(a, name), getattr(b, name))
    assert np.array_equal(a.tables_np, b.tables_np)


def test_tables_are_scattered_distinct_pool_ids():
    case = inputs.make_case("tiny")
    bs = case.workload.block_size
    NB = case.k_cache.shape[0]
    used = []
    for s, L in enumerate(case.lens_np):
        nb = -(-int(L) // bs)
        row = case.tables_np[s]
        assert (row[:nb] >= 0).all() and (row[:nb] < NB).all()
        assert (row[nb:] == -1).all()
        used.extend(row[:nb].tolist())
    assert len(used) == len(set(used))          # no sharing outside config 4
    # the step's new token of sequence s goes to logical position L - 1
    for s, L in enumerate(case.lens_np):
        slot = int(case.slot_mapping[s])
        assert slot == int(case.tables_np[s][(L - 1) // bs]) * bs + (L - 1) % bs


def test_shared_prefix_workload_structure():
    case = inputs.make_case("shared_prefix_cow")
    w = case.workload
    bs = w.block_size
    gs = case.group_start.numpy()
    pl = case.prefix_lens.numpy()
    assert len(gs) == 33 and gs[-1] == w.num_seqs and (np.diff(gs) == 8).all()
    assert (pl == 63 * bs).all()
    pairs = case.copy_pairs.cpu().numpy()
    assert pairs.shape == (w.num_seqs, 2)
    for i in range(len(pl)):
        rows = case.tables_np[gs[i]:gs[i + 1]]
        assert (rows[:, :63] == rows[0, :63]).all()          # 63 shared blocks
        assert len(set(rows[:, 63].tolist())) == 8          # private block 64
        for j, s in enumerate(range(gs[i], gs[i + 1])):
            # copy-on-write: the prompt's block 63 into the sample's own copy
            assert pairs[s, 1] == case.tables_np[s, 63]
    assert (case.lens_np >= 64 * bs).all() and (case.lens_np <= 64 * bs + 256).all()


def test_skewed_shared_prefix_workload_structure():
    """Prompt 0 shares 2047 blocks (its last block is each sample's copy);
    the other prompts as in the uniform workload; unique tokens count every
    shared block once."""
    case = inputs.make_case("shared_prefix_skew")
    w = case.workload
    bs = w.block_size
    gs = case.group_start.numpy()
    pl = case.prefix_lens.numpy()
    assert pl[0] == 2047 * bs and (pl[1:] == 63 * bs).all()
    rows = case.tables_np[gs[0]:gs[1]]
    assert (rows[:, :2047] == rows[0, :2047]).all()
    assert len(set(rows[:, 2047].tolist())) == 8
    assert (case.lens_np[:8] >= 2048 * bs).all() and (case.lens_np[8:] < 2048 * bs).all()
    # Every distinct (block, offset) position read: each group's shared
    # blocks once, every sample's copied block and tail.
    tails = case.lens_np - np.repeat(np.where(np.arange(32) == 0, 2048, 64) * bs, 8)
    assert case.unique_tokens == int(pl.sum()) + w.num_seqs * bs + int(tails.sum())
    # The uniform workload's draws are unchanged by the skewed one's field.
    assert inputs.make_case("shared_prefix_cow").unique_tokens == 69927


def test_multi_query_case_places_queries_at_the_end():
    lens, qlens = [40, 300, 7], [8, 128, 7]
    case = inputs.multi_query_case(3, 16, 4, 64, 16, lens, qlens, seed=3)
    qsl = case.query_start_loc.numpy()
    assert list(qsl) == [0, 8, 136, 143]
    bs = 16
    for s, (L, k) in enumerate(zip(lens, qlens)):
        for j in range(k):
            pos = L - k + j
            slot = int(case.slot_mapping[qsl[s] + j])
            assert slot == int(case.tables_np[s][pos // bs]) * bs + pos % bs

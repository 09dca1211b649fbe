"""Host block manager (C++ in the library, CPU only): the page's block-table
example, on-demand growth, copy-on-write of a shared partial block, prefix
caching and eviction, swap bookkeeping, and invariants under random use."""
import os

import numpy as np
import pytest

from paged_kv_cache_435_b200 import _native as nat
from paged_kv_cache_435_b200 import build as pa_build
from paged_kv_cache_435_b200.block_manager import (BlockManager,
                                                   prefix_block_hash,
                                                   prefix_hash_seed)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module", autouse=True)
def _built():
    pa_build.build()


def toks(n, start=0):
    return np.arange(start, start + n, dtype=np.int32)


def test_page_example_block_tables():
    m = BlockManager(64, 16)
    rows = [l.split() for l in open(os.path.join(GOLDEN, "block_manager_tables.txt"))
            if l.strip() and not l.startswith("#")]
    ids = {}
    for name, n, *blocks in rows:
        sid, slots, cached = m.add_sequence(toks(int(n)))
        ids[name] = sid
        assert list(m.block_table(sid)) == [int(b) for b in blocks]
        assert cached == 0 and len(slots) == int(n)
        # slot of token t = block(t // 16) * 16 + t % 16
        tbl = m.block_table(sid)
        t = np.arange(int(n))
        assert np.array_equal(slots, tbl[t // 16] * 16 + t % 16)
    # R1 holds tokens 0..47; token 48 needs a new block, the next free (B9).
    slots, pairs = m.append_slots(ids["R1"], 1, toks(1, 48))
    assert list(m.block_table(ids["R1"])) == [0, 1, 2, 9] and slots[0] == 9 * 16
    assert len(pairs) == 0
    # A finished request returns its blocks to the free pool.
    free0 = m.num_free_blocks
    m.free(ids["R2"])
    assert m.num_free_blocks == free0 + 2


def test_fork_shares_blocks_and_copies_only_the_diverging_block():
    m = BlockManager(16, 16)
    parent, _, _ = m.add_sequence(toks(20))            # blocks [0, 1]; 1 partial
    child = m.fork(parent)
    assert list(m.block_table(child)) == [0, 1]
    assert m.refcount(0) == 2 and m.refcount(1) == 2
    slots, pairs = m.append_slots(child, 1, toks(1, 100))
    assert pairs.tolist() == [[1, 2]]                  # copy of block 1 only
    assert list(m.block_table(child)) == [0, 2] and slots[0] == 2 * 16 + 4
    assert m.refcount(1) == 1 and m.refcount(0) == 2
    slots, pairs = m.append_slots(parent, 1, toks(1, 200))
    assert len(pairs) == 0 and slots[0] == 1 * 16 + 4  # parent writes in place
    m.free(parent)
    assert m.refcount(0) == 1 and m.refcount(1) == 0


def test_full_shared_block_needs_no_copy():
    m = BlockManager(8, 16)
    a, _, _ = m.add_sequence(toks(32))
    b = m.fork(a)
    _, pairs = m.append_slots(b, 1, toks(1, 7))
    assert len(pairs) == 0 and list(m.block_table(b)) == [0, 1, 2]


def test_prefix_caching_reuses_and_evicts():
    m = BlockManager(6, 16, prefix_caching=True)
    a, _, _ = m.add_sequence(toks(40))                 # [0, 1, 2], 0 and 1 full
    b, slots, cached = m.add_sequence(np.concatenate([toks(32), toks(5, 900)]))
    assert cached == 32 and list(m.block_table(b)) == [0, 1, 3]
    assert len(slots) == 5 and m.refcount(0) == 2
    m.free(a)
    m.free(b)
    assert m.num_free_blocks == 6
    # Freed blocks stay findable: the same prefix is still cached.
    c, _, cached = m.add_sequence(toks(33))
    assert cached == 32 and list(m.block_table(c))[:2] == [0, 1]
    m.free(c)
    # A different prefix gets different blocks; once the pool cycles through
    # every block the cached ones are handed out and forgotten.
    d, _, cached = m.add_sequence(toks(96, 5000))
    assert cached == 0 and m.num_free_blocks == 0
    m.free(d)
    e, _, cached = m.add_sequence(toks(33))
    assert cached == 0


def test_prefix_hash_chains_on_the_parent():
    s = prefix_hash_seed()
    h1 = prefix_block_hash(s, toks(16))
    assert h1 == prefix_block_hash(s, toks(16))
    assert h1 != prefix_block_hash(s, toks(16, 1))
    assert prefix_block_hash(h1, toks(16)) != h1
    assert prefix_block_hash(h1, toks(16)) != prefix_block_hash(s ^ 1, toks(16))


_FNV64_PRIME = 0x100000001b3
_FNV64_BASIS = 0xcbf29ce484222325


def _fnv1a64(h, data: bytes) -> int:
    """FNV-1a, 64 bit: for each byte, xor it in, then multiply by the prime."""
    for c in data:
        h = ((h ^ c) * _FNV64_PRIME) & ((1 << 64) - 1)
    return h


def test_fnv1a_reference_matches_published_vectors():
    # Test vectors of the FNV-1a 64-bit hash as published with the algorithm.
    assert _fnv1a64(_FNV64_BASIS, b"") == 0xcbf29ce484222325
    assert _fnv1a64(_FNV64_BASIS, b"a") == 0xaf63dc4c8601ec8c
    assert _fnv1a64(_FNV64_BASIS, b"foobar") == 0x85944171f73967e8


@pytest.mark.parametrize("tokens", [
    [], [0x61], [0x626f6f66, 0x7261], [1, 2, 3, 4, 5, 6, 7, 8, 9, 10, 11, 12,
                                       13, 14, 15, 16], [-1, 2**31 - 1, 0]])
def test_prefix_hash_known_answers(tokens):
    # The block hash is FNV-1a over the block's token ids (little-endian
    # int32 bytes) started from the parent hash, xor the parent times the
    # prime; the seed of a first block is the FNV offset basis.
    assert prefix_hash_seed() == _FNV64_BASIS
    t = np.asarray(tokens, dtype=np.int32)
    for parent in (_FNV64_BASIS, 0, 0x0123456789abcdef):
        want = _fnv1a64(parent, t.astype("<i4").tobytes()) ^ \
            ((parent * _FNV64_PRIME) & ((1 << 64) - 1))
        assert prefix_block_hash(parent, t) == want


def test_prefix_hash_of_ascii_tokens_is_published_fnv1a():
    # "a" as one token id 0x61 hashes the bytes 61 00 00 00: the published
    # value of "a" continued over three zero bytes.
    h_a = _fnv1a64(_FNV64_BASIS, b"a")
    assert h_a == 0xaf63dc4c8601ec8c
    want = _fnv1a64(h_a, b"\0\0\0") ^ ((_FNV64_BASIS * _FNV64_PRIME) & ((1 << 64) - 1))
    assert prefix_block_hash(_FNV64_BASIS, np.array([0x61], np.int32)) == want


def test_out_of_blocks_changes_nothing():
    m = BlockManager(4, 16)
    a, _, _ = m.add_sequence(toks(48))
    with pytest.raises(nat.PAError) as e:
        m.add_sequence(toks(40))
    assert e.value.status == nat.PA_ERR_NO_BLOCKS
    assert m.num_free_blocks == 1
    m.append_slots(a, 16, toks(16))                    # uses the last block
    with pytest.raises(nat.PAError):
        m.append_slots(a, 1, toks(1))
    assert m.seq_len(a) == 64


def test_swap_out_and_in_bookkeeping():
    m = BlockManager(8, 16, num_cpu_blocks=4)
    a, _, _ = m.add_sequence(toks(40))                 # 3 blocks
    out = m.swap_out(a)
    assert out[:, 0].tolist() == [0, 1, 2] and out[:, 1].tolist() == [0, 1, 2]
    assert m.num_free_blocks == 8 and m.num_free_cpu_blocks == 1
    other, _, _ = m.add_sequence(toks(48, 100))        # takes GPU blocks 3,4,5
    back = m.swap_in(a)
    assert back[:, 0].tolist() == [0, 1, 2] and back[:, 1].tolist() == [6, 7, 0]
    assert list(m.block_table(a)) == [6, 7, 0] and m.num_free_cpu_blocks == 4
    b = m.fork(other)
    with pytest.raises(nat.PAError):
        m.swap_out(b)                                  # shared blocks stay


def test_random_operations_keep_refcounts_consistent():
    rng = np.random.default_rng(0)
    nb = 64
    m = BlockManager(nb, 16, prefix_caching=True)
    live = []
    for step in range(600):
        op = rng.integers(0, 4)
        try:
            if op == 0 or not live:
                sid, _, _ = m.add_sequence(rng.integers(0, 4, rng.integers(1, 60)))
                live.append(sid)
            elif op == 1:
                live.append(m.fork(live[rng.integers(len(live))]))
            elif op == 2:
                sid = live[rng.integers(len(live))]
                n = int(rng.integers(1, 20))
                m.append_slots(sid, n, rng.integers(0, 4, n))
            else:
                m.free(live.pop(rng.integers(len(live))))
        except nat.PAError as e:
            assert e.status == nat.PA_ERR_NO_BLOCKS
        counts = np.zeros(nb, dtype=int)
        for sid in live:
            tbl = m.block_table(sid)
            assert len(tbl) == -(-m.seq_len(sid) // 16)
            np.add.at(counts, tbl, 1)
        assert all(m.refcount(b) == counts[b] for b in range(nb))
        assert m.num_free_blocks == int((counts == 0).sum())


def shared_blocks(m, ids):
    """Leading blocks that every sequence of ids maps to the same block."""
    tables = [list(m.block_table(s)) for s in ids]
    n = 0
    while all(len(t) > n for t in tables) and len({t[n] for t in tables}) == 1:
        n += 1
    return n


def test_shared_prefix_groups_follow_forks_and_copy_on_write():
    m = BlockManager(64, 16)
    a, _, _ = m.add_sequence(toks(40))            # 2 full blocks + 8 tokens
    samples = [a] + [m.fork(a) for _ in range(3)]
    b, _, _ = m.add_sequence(toks(20, 500))       # unrelated prompt
    c = m.fork(b)
    lone, _, _ = m.add_sequence(toks(7, 900))
    batch = samples + [b, c, lone]
    gs, pl, mg = m.shared_prefix_groups(batch)
    # the four samples share all 3 blocks (the partial one too, before CoW)
    assert list(gs) == [0, 4, 6, 7] and list(pl) == [48, 32, 0] and mg == 4
    for i in range(len(pl)):
        members = batch[gs[i]:gs[i + 1]]
        if len(members) > 1:
            assert pl[i] == 16 * shared_blocks(m, members)
    # every sample appends a token: copy-on-write of the partial block
    for s in samples:
        m.append_slots(s, 1, np.array([7], dtype=np.int32))
    gs, pl, _ = m.shared_prefix_groups(batch)
    assert list(gs) == [0, 4, 6, 7] and list(pl) == [32, 32, 0]
    # interleaved order: runs only, a non-sharing neighbour ends a group
    gs, pl, _ = m.shared_prefix_groups([samples[0], b, samples[1], c])
    assert list(gs) == [0, 1, 2, 3, 4] and list(pl) == [0, 0, 0, 0]
    # a stricter threshold splits groups whose common prefix is too short
    gs, pl, _ = m.shared_prefix_groups(batch, min_shared_blocks=3)
    assert list(gs) == [0, 1, 2, 3, 4, 5, 6, 7] and not any(pl)


def test_shared_prefix_groups_reject_bad_sequences():
    m = BlockManager(16, 16, num_cpu_blocks=8)
    a, _, _ = m.add_sequence(toks(20))
    with pytest.raises(nat.PAError):
        m.shared_prefix_groups([a, 99])
    m.swap_out(a)
    with pytest.raises(nat.PAError):
        m.shared_prefix_groups([a])
    gs, pl, mg = m.shared_prefix_groups([])
    assert list(gs) == [0] and len(pl) == 0 and mg == 1

"""Pins for the fp64 oracle (CPU only).

Each check ties the oracle to something other than itself: a library routine
on the special case it reduces to (torch's scaled_dot_product_attention on the
contiguous logical sequence, numpy fancy indexing for the cache ops), closed
forms, invariants the paged layout must satisfy ("Block-Level Management" and
"Memory Sharing via Copy-on-Write (CoW)" on "vLLM: Anatomy and Mechanisms of
High-Throughput LLM Inference"), brute force on tiny inputs, and the numbers
the pages print (tests/golden).  ``tests/test_oracle_mutants.py`` plants
plausible mistakes in the oracle's C source and checks these pins catch them.
"""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from paged_kv_cache_435_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------------
# helpers that build paged inputs from contiguous logical data
# --------------------------------------------------------------------------
def bf16(shape, gen):
    return torch.randn(*shape, generator=gen).to(torch.bfloat16)


def scatter_to_pool(k_seqs, v_seqs, block_size, num_blocks, rng, fill=None):
    """Lay logical per-sequence K/V ([L_s, Hkv, D] each) into a pool through a
    random table.  Returns k_pool, v_pool (bf16), tables (int32), lens."""
    Hkv, D = k_seqs[0].shape[1:]
    lens = np.array([k.shape[0] for k in k_seqs], dtype=np.int32)
    nblk = -(-lens // block_size)
    MB = max(1, int(nblk.max()))
    perm = rng.permutation(num_blocks)
    assert nblk.sum() <= num_blocks
    if fill is None:
        k_pool = torch.zeros(num_blocks, block_size, Hkv, D, dtype=torch.bfloat16)
        v_pool = torch.zeros_like(k_pool)
    else:
        k_pool, v_pool = fill
    tables = np.full((len(k_seqs), MB), -1, dtype=np.int32)
    cur = 0
    for s, (k, v) in enumerate(zip(k_seqs, v_seqs)):
        for b in range(int(nblk[s])):
            phys = int(perm[cur]); cur += 1
            tables[s, b] = phys
            lo, hi = b * block_size, min((b + 1) * block_size, k.shape[0])
            k_pool[phys, : hi - lo] = k[lo:hi]
            v_pool[phys, : hi - lo] = v[lo:hi]
    return k_pool, v_pool, tables, lens


def sdpa_reference(q, k_seqs, v_seqs, scale):
    """torch's fp64 scaled_dot_product_attention on each contiguous sequence
    (GQA via enable_gqa: query head h uses kv head h // G)."""
    out = []
    for s in range(q.shape[0]):
        qs = q[s].double()[None, :, None, :]                    # [1,Hq,1,D]
        ks = k_seqs[s].double().permute(1, 0, 2)[None]          # [1,Hkv,L,D]
        vs = v_seqs[s].double().permute(1, 0, 2)[None]
        if k_seqs[s].shape[0] == 0:
            out.append(torch.zeros(q.shape[1], q.shape[2], dtype=torch.float64))
            continue
        o = F.scaled_dot_product_attention(qs, ks, vs, scale=scale,
                                           enable_gqa=True)
        out.append(o[0, :, 0, :])
    return torch.stack(out).numpy()


def random_problem(lens, Hq, Hkv, D, bs, seed, slack=5):
    gen = torch.Generator().manual_seed(seed)
    rng = np.random.default_rng(seed)
    q = bf16((len(lens), Hq, D), gen)
    k_seqs = [bf16((L, Hkv, D), gen) for L in lens]
    v_seqs = [bf16((L, Hkv, D), gen) for L in lens]
    nb = int(sum(-(-L // bs) for L in lens)) + slack
    k_pool, v_pool, tables, lens_a = scatter_to_pool(k_seqs, v_seqs, bs, nb, rng)
    return q, k_seqs, v_seqs, k_pool, v_pool, tables, lens_a


# --------------------------------------------------------------------------
# attention: library special case
# --------------------------------------------------------------------------
@pytest.mark.parametrize("Hq,Hkv,D,bs,lens", [
    (4, 4, 64, 16, [1, 16, 17, 100]),       # MHA, ragged block tails
    (8, 2, 32, 16, [5, 33, 48, 0, 64]),     # G=4, an empty context
    (16, 2, 16, 32, [31, 32, 33, 70]),      # G=8, bs=32
    (6, 3, 8, 16, [200, 1, 2]),             # G=2, odd head counts
])
def test_attention_matches_sdpa_on_logical_sequence(Hq, Hkv, D, bs, lens):
    q, ks, vs, kp, vp, tables, lens_a = random_problem(lens, Hq, Hkv, D, bs,
                                                       seed=11 + len(lens))
    scale = 1.0 / math.sqrt(D)
    got = oracle.paged_decode_attention(q, kp, vp, tables, lens_a, scale, Hkv)
    ref = sdpa_reference(q, ks, vs, scale)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-13)


def test_scale_is_applied_to_logits():
    # A different scale must change the result exactly as SDPA's scale does.
    q, ks, vs, kp, vp, tables, lens_a = random_problem([40, 9], 4, 2, 16, 16, 5)
    for scale in (0.03, 0.5, 2.0):
        got = oracle.paged_decode_attention(q, kp, vp, tables, lens_a, scale, 2)
        np.testing.assert_allclose(got, sdpa_reference(q, ks, vs, scale),
                                   rtol=1e-12, atol=1e-13)


# --------------------------------------------------------------------------
# attention: closed forms and brute force
# --------------------------------------------------------------------------
def test_single_token_context_returns_its_value_exactly():
    q, ks, vs, kp, vp, tables, lens_a = random_problem([1, 1], 8, 2, 64, 16, 3)
    got = oracle.paged_decode_attention(q, kp, vp, tables, lens_a, 0.125, 2)
    for s in range(2):
        for h in range(8):
            np.testing.assert_array_equal(got[s, h], vs[s][0, h // 4].double().numpy())


def test_zero_query_gives_mean_of_values():
    q, ks, vs, kp, vp, tables, lens_a = random_problem([37, 100], 4, 4, 32, 16, 4)
    q = torch.zeros_like(q)
    got = oracle.paged_decode_attention(q, kp, vp, tables, lens_a, 0.2, 4)
    for s in range(2):
        mean = vs[s].double().mean(dim=0).numpy()                  # [Hkv, D]
        np.testing.assert_allclose(got[s], mean, rtol=1e-13, atol=1e-14)


def test_equal_keys_give_mean_of_values():
    gen = torch.Generator().manual_seed(9)
    L, Hkv, D = 50, 2, 16
    k = bf16((1, Hkv, D), gen).expand(L, Hkv, D).contiguous()
    v = bf16((L, Hkv, D), gen)
    q = bf16((1, 4, D), gen)
    kp, vp, tables, lens = scatter_to_pool([k], [v], 16, 8, np.random.default_rng(0))
    got = oracle.paged_decode_attention(q, kp, vp, tables, lens, 0.3, Hkv)
    np.testing.assert_allclose(got[0], v.double().mean(0).numpy()[[0, 0, 1, 1]],
                               rtol=1e-13, atol=1e-14)


def test_dominant_key_selects_its_value():
    # One key aligned with q with a logit gap >= 50: weight of the others is
    # below e^-50 relative, so the output is that key's value to ~1e-20.
    D, L = 16, 40
    gen = torch.Generator().manual_seed(2)
    q = torch.zeros(1, 1, D); q[0, 0, 3] = 8.0
    k = bf16((L, 1, D), gen) * 0.01
    k[17, 0, 3] = 8.0
    v = bf16((L, 1, D), gen)
    kp, vp, tables, lens = scatter_to_pool([k.to(torch.bfloat16)], [v], 16, 4,
                                           np.random.default_rng(1))
    got = oracle.paged_decode_attention(q.to(torch.bfloat16), kp, vp, tables,
                                        lens, 1.0, 1)
    np.testing.assert_allclose(got[0, 0], v[17, 0].double().numpy(),
                               rtol=0, atol=1e-12)


def test_empty_context_gives_zeros():
    q, ks, vs, kp, vp, tables, lens_a = random_problem([0, 3], 2, 2, 8, 16, 6)
    got = oracle.paged_decode_attention(q, kp, vp, tables, lens_a, 1.0, 2)
    assert np.all(got[0] == 0.0)
    assert np.any(got[1] != 0.0)


def test_brute_force_tiny():
    # Hand-expanded softmax with exact float sums (math.fsum) on L<=4, D=4.
    gen = torch.Generator().manual_seed(21)
    for trial in range(6):
        L = 1 + trial % 4
        Hq, Hkv, D = 2, 1, 4
        q = bf16((1, Hq, D), gen)
        k = bf16((L, Hkv, D), gen)
        v = bf16((L, Hkv, D), gen)
        kp, vp, tables, lens = scatter_to_pool([k], [v], 16, 3,
                                               np.random.default_rng(trial))
        scale = 0.7
        got = oracle.paged_decode_attention(q, kp, vp, tables, lens, scale, Hkv)
        qf, kf, vf = q.double().tolist(), k.double().tolist(), v.double().tolist()
        for h in range(Hq):
            z = [scale * math.fsum(qf[0][h][d] * kf[t][0][d] for d in range(D))
                 for t in range(L)]
            m = max(z)
            w = [math.exp(x - m) for x in z]
            den = math.fsum(w)
            for d in range(D):
                want = math.fsum(w[t] * vf[t][0][d] for t in range(L)) / den
                assert abs(got[0, h, d] - want) <= 1e-14 * max(1.0, abs(want))


# --------------------------------------------------------------------------
# attention: invariants of the paged layout
# --------------------------------------------------------------------------
def test_physical_block_permutation_invariance():
    q, ks, vs, kp, vp, tables, lens = random_problem([70, 3, 129], 8, 2, 32, 16, 7)
    base = oracle.paged_decode_attention(q, kp, vp, tables, lens, 0.17, 2)
    NB = kp.shape[0]
    perm = np.random.default_rng(3).permutation(NB)       # new id of block i
    kp2 = torch.empty_like(kp); vp2 = torch.empty_like(vp)
    kp2[torch.from_numpy(perm)] = kp
    vp2[torch.from_numpy(perm)] = vp
    tables2 = np.where(tables >= 0, perm[np.maximum(tables, 0)], -1).astype(np.int32)
    moved = oracle.paged_decode_attention(q, kp2, vp2, tables2, lens, 0.17, 2)
    np.testing.assert_array_equal(base, moved)


def test_block_size_invariance():
    gen = torch.Generator().manual_seed(8)
    lens = [1, 31, 32, 33, 95]
    Hq, Hkv, D = 8, 4, 16
    q = bf16((len(lens), Hq, D), gen)
    ks = [bf16((L, Hkv, D), gen) for L in lens]
    vs = [bf16((L, Hkv, D), gen) for L in lens]
    outs = []
    for bs in (16, 32):
        nb = sum(-(-L // bs) for L in lens) + 3
        kp, vp, tables, la = scatter_to_pool(ks, vs, bs, nb, np.random.default_rng(bs))
        outs.append(oracle.paged_decode_attention(q, kp, vp, tables, la, 0.25, Hkv))
    # Same logical order of accumulation in both layouts: bitwise equal.
    np.testing.assert_array_equal(outs[0], outs[1])


def test_shared_prefix_equals_separate_copies():
    """Sequences whose tables point at the same prefix blocks get the same
    result as sequences holding private copies of those blocks."""
    gen = torch.Generator().manual_seed(12)
    bs, Hkv, D, Hq = 16, 2, 16, 4
    prefix_k = bf16((48, Hkv, D), gen)
    prefix_v = bf16((48, Hkv, D), gen)
    tails = [5, 0, 17]
    ks = [torch.cat([prefix_k, bf16((t, Hkv, D), gen)]) for t in tails]
    vs = [torch.cat([prefix_v, bf16((t, Hkv, D), gen)]) for t in tails]
    q = bf16((len(tails), Hq, D), gen)
    # separate copies
    kp, vp, tables, lens = scatter_to_pool(ks, vs, bs, 20, np.random.default_rng(0))
    sep = oracle.paged_decode_attention(q, kp, vp, tables, lens, 0.3, Hkv)
    # shared: all three tables use the first sequence's three prefix blocks
    shared_tables = tables.copy()
    shared_tables[1:, :3] = tables[0, :3]
    shared = oracle.paged_decode_attention(q, kp, vp, shared_tables, lens, 0.3, Hkv)
    np.testing.assert_array_equal(sep, shared)
    # and the copies are no longer needed: wiping them does not change it
    for s in (1, 2):
        for b in range(3):
            kp[int(tables[s, b])] = 0
            vp[int(tables[s, b])] = 0
    again = oracle.paged_decode_attention(q, kp, vp, shared_tables, lens, 0.3, Hkv)
    np.testing.assert_array_equal(sep, again)


def test_threads_do_not_change_results():
    q, ks, vs, kp, vp, tables, lens = random_problem([300, 7, 64, 65], 8, 2, 64, 16, 13)
    one = oracle.paged_decode_attention(q, kp, vp, tables, lens, 0.1, 2, threads=1)
    many = oracle.paged_decode_attention(q, kp, vp, tables, lens, 0.1, 2, threads=5)
    np.testing.assert_array_equal(one, many)


def test_out_of_range_block_id_is_an_error():
    q, ks, vs, kp, vp, tables, lens = random_problem([20], 2, 2, 8, 16, 14)
    tables = tables.copy()
    tables[0, 1] = kp.shape[0]
    with pytest.raises(ValueError):
        oracle.paged_decode_attention(q, kp, vp, tables, lens, 1.0, 2)


# --------------------------------------------------------------------------
# reshape_and_cache
# --------------------------------------------------------------------------
def _cache_bits(NB, bs, Hkv, D, sentinel=0x7FC1):
    return (np.full((NB, bs, Hkv, D), sentinel, dtype=np.uint16),
            np.full((NB, bs, Hkv, D), sentinel ^ 0x00FF, dtype=np.uint16))


@pytest.mark.parametrize("bs", [16, 32])
def test_reshape_and_cache_matches_flat_slot_indexing(bs):
    gen = torch.Generator().manual_seed(bs)
    NB, Hkv, D, T = 12, 4, 32, 30
    key = bf16((T, Hkv, D), gen)
    value = bf16((T, Hkv, D), gen)
    rng = np.random.default_rng(bs)
    slots = rng.choice(NB * bs, size=T, replace=False).astype(np.int64)
    if 0 not in slots:
        slots[5] = 0                                      # slot 0 is a real slot
    slots[[3, 17]] = -1                                   # padding tokens
    kc, vc = _cache_bits(NB, bs, Hkv, D)
    oracle.reshape_and_cache(key, value, kc, vc, slots)
    # numpy special case: a [NB*bs, Hkv, D] view indexed by slot
    ek, ev = _cache_bits(NB, bs, Hkv, D)
    keep = slots >= 0
    kb = key.view(torch.int16).numpy().view(np.uint16)
    vb = value.view(torch.int16).numpy().view(np.uint16)
    ek.reshape(NB * bs, Hkv, D)[slots[keep]] = kb[keep]
    ev.reshape(NB * bs, Hkv, D)[slots[keep]] = vb[keep]
    np.testing.assert_array_equal(kc, ek)
    np.testing.assert_array_equal(vc, ev)


def test_reshape_and_cache_round_trip_through_block_table():
    case = inputs.make_case("tiny")
    kc = case.k_cache.view(torch.int16).numpy().view(np.uint16).copy()
    vc = case.v_cache.view(torch.int16).numpy().view(np.uint16).copy()
    oracle.reshape_and_cache(case.new_key, case.new_value, kc, vc, case.slot_mapping)
    bs = case.workload.block_size
    nk = case.new_key.view(torch.int16).numpy().view(np.uint16)
    for s, L in enumerate(case.lens_np):
        pos = int(L) - 1
        blk = case.tables_np[s, pos // bs]
        np.testing.assert_array_equal(kc[blk, pos % bs], nk[s])


def test_reshape_and_cache_rejects_out_of_range_slot():
    gen = torch.Generator().manual_seed(1)
    key = bf16((2, 1, 8), gen)
    kc, vc = _cache_bits(2, 16, 1, 8)
    with pytest.raises(ValueError):
        oracle.reshape_and_cache(key, key, kc, vc, np.array([0, 32], np.int64))


# --------------------------------------------------------------------------
# copy_blocks
# --------------------------------------------------------------------------
def test_copy_blocks_matches_numpy_block_assignment():
    rng = np.random.default_rng(5)
    NB, bs, Hkv, D, layers = 20, 16, 2, 16, 3
    ks = [rng.integers(0, 65535, (NB, bs, Hkv, D), dtype=np.uint16) for _ in range(layers)]
    vs = [rng.integers(0, 65535, (NB, bs, Hkv, D), dtype=np.uint16) for _ in range(layers)]
    pairs = np.array([[0, 7], [3, 9], [3, 11], [15, 2], [4, 4]], dtype=np.int64)
    ek = [k.copy() for k in ks]; ev = [v.copy() for v in vs]
    for e in ek + ev:
        e[pairs[:, 1]] = e[pairs[:, 0]]
    oracle.copy_blocks(ks, vs, pairs)
    for a, b in zip(ks + vs, ek + ev):
        np.testing.assert_array_equal(a, b)


def test_copy_blocks_rejects_out_of_range():
    z = [np.zeros((4, 16, 1, 8), np.uint16)]
    with pytest.raises(ValueError):
        oracle.copy_blocks(z, [z[0].copy()], np.array([[0, 4]], np.int64))


# --------------------------------------------------------------------------
# swap_blocks
# --------------------------------------------------------------------------
def test_swap_blocks_matches_numpy_and_round_trips():
    rng = np.random.default_rng(11)
    gpu = [rng.integers(0, 65535, (12, 16, 2, 8), dtype=np.uint16) for _ in range(4)]
    cpu = [np.zeros((5, 16, 2, 8), dtype=np.uint16) for _ in range(4)]
    out_pairs = np.array([[3, 0], [7, 4], [11, 2]], dtype=np.int64)
    expect = [c.copy() for c in cpu]
    for e, g in zip(expect, gpu):
        e[out_pairs[:, 1]] = g[out_pairs[:, 0]]
    oracle.swap_blocks(gpu, cpu, out_pairs)                    # swap out
    for a, b in zip(cpu, expect):
        np.testing.assert_array_equal(a, b)
    back = [np.zeros_like(g) for g in gpu]
    in_pairs = out_pairs[:, ::-1].copy()
    in_pairs[:, 1] = [1, 5, 9]                                 # new block ids
    oracle.swap_blocks(cpu, back, in_pairs)                    # swap in
    for b, g in zip(back, gpu):
        np.testing.assert_array_equal(b[[1, 5, 9]], g[[3, 7, 11]])
        assert not b[[0, 2, 3]].any()


def test_swap_blocks_rejects_out_of_range():
    a = [np.zeros((4, 16), np.uint16)]
    b = [np.zeros((2, 16), np.uint16)]
    with pytest.raises(ValueError):
        oracle.swap_blocks(a, b, np.array([[3, 2]], np.int64))


# --------------------------------------------------------------------------
# numbers the pages print
# --------------------------------------------------------------------------
def _golden_rows(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


def test_block_manager_example_block_counts():
    rows = _golden_rows("block_manager_example.txt")
    assert len(rows) == 4
    for _, bs, tokens, blocks in rows:
        assert int(inputs.blocks_for(int(tokens), int(bs))) == int(blocks)


def test_pool_layout_bytes_match_block_formula():
    """A pool block (K plus V) of the layout both sides use occupies exactly the
    bytes the KV-cache manager formula gives."""
    for bs, hkv, d, nbytes, want in _golden_rows("block_bytes.txt"):
        bs, hkv, d, nbytes, want = map(int, (bs, hkv, d, nbytes, want))
        k = torch.empty(3, bs, hkv, d, dtype=torch.bfloat16)
        assert nbytes == k.element_size()
        assert k[0].nbytes + torch.empty_like(k)[0].nbytes == want


def test_named_workloads_are_well_formed():
    c = inputs.make_case("tiny")
    assert list(c.lens_np) == [1, 16, 17, 100]
    assert c.k_cache.shape == (64, 16, 4, 64)
    used = c.tables_np[c.tables_np >= 0]
    assert len(np.unique(used)) == used.size                # distinct ids
    assert used.size == int(inputs.blocks_for(c.lens_np, 16).sum())
    s = inputs.make_case("shared_prefix_cow")
    assert s.copy_pairs.shape == (256, 2)
    # the 8 samples of a prompt share blocks 0..62 and own block 63
    t = s.tables_np
    assert np.all(t[0:8, :63] == t[0, :63])
    assert len(np.unique(t[0:8, 63])) == 8
    assert np.all(s.copy_pairs[:, 1].numpy() == t[:, 63])

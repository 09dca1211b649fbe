"""pa_decode_attention_shared_prefix on the GPU through the C ABI against the
fp64 oracle.  The oracle knows nothing of groups: it attends every sequence
over its whole block table, so these tests check that the group pass (shared
blocks read once for all members' rows, tcgen05) plus the per-sequence pass
and their merge reproduce plain paged attention ("Memory Sharing via
Copy-on-Write (CoW)": parallel samples share the prompt's blocks).
Tolerance as for decode: max-abs <= 4e-3 and relative L2 <= 1e-3."""
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


def run(case, flags=None, partition_size=0, group_start=None, prefix_lens=None,
        max_group_size=None):
    B, Hq, D = case.q.shape
    Hkv, bs = case.workload.num_kv_heads, case.workload.block_size
    gs = case.group_start if group_start is None else group_start
    pl = case.prefix_lens if prefix_lens is None else prefix_lens
    mgs = case.max_group_size if max_group_size is None else max_group_size
    out = torch.full((B, Hq, D), float("nan"), dtype=torch.float32, device="cuda")
    nbytes = pa.pa_shared_prefix_workspace_size(B, Hq, Hkv, D, bs,
                                                case.max_context_len,
                                                partition_size)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    pa.pa_decode_attention_shared_prefix(
        out, case.q, case.k_cache, case.v_cache, case.block_tables,
        case.context_lens, gs.cuda(), pl.cuda(), case.max_context_len, mgs,
        case.scale, ws, partition_size=partition_size, error_flags=flags)
    return out


def reference(case):
    return oracle.paged_decode_attention(
        case.q.cpu(), bits(case.k_cache), bits(case.v_cache), case.tables_np,
        case.lens_np.astype(np.int32), case.scale, case.workload.num_kv_heads)


def check(case, expect_flags=0, **kw):
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = run(case, flags, **kw)
    torch.cuda.synchronize()
    assert int(flags.item()) == expect_flags
    return assert_attn_close(out, reference(case), case.workload.name), out


@pytest.mark.parametrize("name", ["shared_prefix_cow", "shared_prefix_skew"])
def test_parallel_sampling_workload(name):
    """32 prompts x 8 samples (32q/8kv, D=128, bs=16): the copy-on-write step
    and the new token's write run first; groups share their prompt's blocks
    but the last (each sample's private copy).  In the skewed batch prompt 0
    has 32768 tokens, so its group's pass is cut into pieces across CTAs;
    every output is compared."""
    case = inputs.make_case(name, device="cuda")
    ek, ev = bits(case.k_cache), bits(case.v_cache)
    pa.pa_copy_blocks([case.k_cache], [case.v_cache], case.copy_pairs)
    pa.pa_reshape_and_cache(case.new_key, case.new_value, case.k_cache,
                            case.v_cache, case.slot_mapping)
    oracle.copy_blocks([ek], [ev], case.copy_pairs.cpu().numpy())
    oracle.reshape_and_cache(case.new_key.cpu(), case.new_value.cpu(), ek, ev,
                             case.slot_mapping.cpu().numpy())
    (_, _), out = check(case)
    # The plain decode call on the same inputs agrees within rounding.
    B, Hq, D = case.q.shape
    plain = torch.empty_like(out)
    pa.pa_decode_attention(plain, case.q, case.k_cache, case.v_cache,
                           case.block_tables, case.context_lens,
                           case.max_context_len, case.scale)
    torch.cuda.synchronize()
    assert (plain - out).abs().max().item() <= 2e-5


@pytest.mark.parametrize("Hq,Hkv,bs", [(32, 8, 16), (64, 8, 16), (8, 8, 32),
                                       (24, 8, 16), (64, 8, 32)])
def test_group_shapes(Hq, Hkv, bs):
    """G = 4, 8, 1, 3 and both block sizes.  Groups of 8, 5, 1 and 12 members
    (G=8 x 12 members = 3 row tiles), a member shorter than its prefix, two
    whose context ends exactly at the prefix, a group with prefix 0 in the
    middle of the batch and sequences after the last group."""
    P0, P1, P2, P3 = 20 * bs, 6 * bs, 3 * bs, 40 * bs
    lens = ([P0 + t for t in (1, 17, 200, 0, 33, 5, 64, 129)] +   # [0, 8)
            [P1 + 3, P1 - bs - 3, P1 + 90, P1, P1 + 1] +            # [8, 13)
            [555] +                                                 # [13, 14), P=0
            [P2 + 7] +                                              # [14, 15)
            [P3 + 11 * t for t in range(12)] +                      # [15, 27)
            [42, 1])                                                # no group
    gs = [0, 8, 13, 14, 15, 27]
    pl = [P0, P1, 0, P2, P3]
    case = inputs.grouped_case(Hq, Hkv, 128, bs, lens, gs, pl, seed=Hq + bs,
                               device="cuda")
    check(case)


def test_split_suffix_and_determinism():
    """Long private tails with 64-token partitions: the split merge kernel
    folds in the group pass's partial; repeated calls are bitwise equal."""
    bs = 16
    lens = [512 + 700, 512 + 1, 512 + 333, 300, 512 + 64]
    case = inputs.grouped_case(32, 8, 128, bs, lens, [0, 3], [512], seed=77,
                               device="cuda")
    (_, _), a = check(case, partition_size=64)
    b = run(case, partition_size=64)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_invalid_groups_are_flagged_and_still_exact():
    """A prefix that is not a multiple of the block size, a group larger than
    max_group_size and an inverted group all fall back to the per-sequence
    pass (PA_DEVERR_PREFIX) with exact results."""
    bs = 16
    lens = [200, 210, 220, 230, 240, 250, 260, 270]
    case = inputs.grouped_case(32, 8, 128, bs, lens, [0, 2, 5, 8], [64, 64, 48],
                               seed=3, device="cuda")
    check(case, expect_flags=pa.PA_DEVERR_PREFIX,
          prefix_lens=torch.tensor([64, 72, 48], dtype=torch.int32))
    check(case, expect_flags=pa.PA_DEVERR_PREFIX, max_group_size=2)
    check(case, expect_flags=pa.PA_DEVERR_PREFIX,
          group_start=torch.tensor([0, 2, 1, 8], dtype=torch.int32),
          prefix_lens=torch.tensor([64, 0, 0], dtype=torch.int32))


def test_no_groups_is_plain_decode():
    case = inputs.custom_case(6, 32, 8, 128, 16, [1, 16, 17, 100, 1000, 3000],
                              seed=11, device="cuda")
    out = torch.empty(case.q.shape, dtype=torch.float32, device="cuda")
    B, Hq, D = case.q.shape
    ws = torch.empty(pa.pa_shared_prefix_workspace_size(
        B, Hq, 8, D, 16, case.max_context_len), dtype=torch.uint8, device="cuda")
    empty = torch.zeros(1, dtype=torch.int32, device="cuda")
    pa.pa_decode_attention_shared_prefix(
        out, case.q, case.k_cache, case.v_cache, case.block_tables,
        case.context_lens, empty, empty[:0], case.max_context_len, 1,
        case.scale, ws)
    torch.cuda.synchronize()
    assert_attn_close(out, reference(case), "no groups")


def test_block_manager_groups_drive_the_shared_prefix_call():
    """Parallel sampling end to end: the block manager forks samples from
    three prompts, two decode steps append a token to every sample (with the
    copy-on-write copies and new-token writes on the GPU), and the manager's
    groups feed the shared-prefix call, checked against the fp64 oracle."""
    from paged_kv_cache_435_b200.block_manager import BlockManager
    NB, BS, HKV, HQ, D = 256, 16, 4, 16, 128
    gen = torch.Generator().manual_seed(21)

    def rows(n):
        return (torch.randn(n, HKV, D, generator=gen).to(torch.bfloat16),
                torch.randn(n, HKV, D, generator=gen).to(torch.bfloat16))

    k = torch.randn(NB, BS, HKV, D, generator=gen).to(torch.bfloat16).cuda()
    v = torch.randn(NB, BS, HKV, D, generator=gen).to(torch.bfloat16).cuda()
    m = BlockManager(NB, BS)
    batch = []
    for pi, plen in enumerate([300, 130, 77]):
        p, slots, _ = m.add_sequence(np.arange(plen, dtype=np.int32) + 1000 * pi)
        nk, nv = rows(plen)
        pa.pa_reshape_and_cache(nk.cuda(), nv.cuda(), k, v, torch.from_numpy(slots).cuda())
        batch += [p] + [m.fork(p) for _ in range(pi + 2)]
    for step in range(2):
        slots, pairs = [], []
        for s in batch:
            sl, pr = m.append_slots(s, 1, np.array([7 + step], dtype=np.int32))
            slots.append(sl)
            pairs.append(pr)
        pairs = np.concatenate(pairs).astype(np.int64)
        if len(pairs):
            pa.pa_copy_blocks([k], [v], torch.from_numpy(pairs).cuda())
        nk, nv = rows(len(batch))
        pa.pa_reshape_and_cache(nk.cuda(), nv.cuda(), k, v,
                                torch.from_numpy(np.concatenate(slots)).cuda())
    tables = [m.block_table(s) for s in batch]
    MB = max(len(t) for t in tables)
    bt = np.full((len(batch), MB), -1, dtype=np.int32)
    for i, t in enumerate(tables):
        bt[i, :len(t)] = t
    lens = np.array([m.seq_len(s) for s in batch], dtype=np.int32)
    gs, pl, mg = m.shared_prefix_groups(batch)
    assert len(gs) == 4 and pl.min() > 0 and mg == 5

    q = torch.randn(len(batch), HQ, D, generator=gen).to(torch.bfloat16).cuda()
    maxlen = int(lens.max())
    out = torch.empty(len(batch), HQ, D, dtype=torch.float32, device="cuda")
    ws = torch.empty(pa.pa_shared_prefix_workspace_size(len(batch), HQ, HKV, D, BS, maxlen),
                     dtype=torch.uint8, device="cuda")
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    bt_d, lens_d = torch.from_numpy(bt).cuda(), torch.from_numpy(lens).cuda()
    pa.pa_decode_attention_shared_prefix(
        out, q, k, v, bt_d, lens_d, torch.from_numpy(gs).cuda(),
        torch.from_numpy(pl).cuda(), maxlen, mg, 0.088, ws, error_flags=flags)
    plain = torch.empty_like(out)
    pa.pa_decode_attention(plain, q, k, v, bt_d, lens_d, maxlen, 0.088)
    torch.cuda.synchronize()
    assert int(flags.item()) == 0
    ref = oracle.paged_decode_attention(q.cpu(), bits(k), bits(v), bt, lens, 0.088, HKV)
    assert_attn_close(out, ref, "block-manager groups")
    assert (plain - out).abs().max().item() <= 2e-5


def test_first_member_shorter_than_prefix():
    """The group's first member ends inside the prefix (its table stops
    there): the shared blocks are read through a member that covers them."""
    lens = [40, 300, 256, 9, 511]
    case = inputs.grouped_case(32, 8, 128, 16, lens, [0, 5], [256], seed=91,
                               device="cuda")
    check(case)


def test_long_prefix_and_tails():
    """A 16384-token prefix shared by 6 samples with tails of 0..1000 tokens
    (G = 4), and a 5000-token prefix shared by 3 samples (bs 16)."""
    P0, P1 = 16384, 5000 // 16 * 16
    lens = [P0 + t for t in (0, 1, 999, 1000, 517, 64)] + [P1 + t for t in (3, 700, 0)]
    case = inputs.grouped_case(32, 8, 128, 16, lens, [0, 6, 9], [P0, P1], seed=16,
                               device="cuda")
    check(case)


@pytest.mark.parametrize("partition_size", [0, 256])
def test_more_than_768_sequences(partition_size):
    """800 sequences: 96 groups of 8 samples sharing a 512-token prefix, then
    32 sequences outside every group.  Past 768 sequences the per-sequence
    pass skips the groups' members on the plain grid (one CTA per kv head,
    partition and sequence) instead of the persistent compact-item grid; with
    256-token partitions the ungrouped sequences are split and merged."""
    rng = np.random.default_rng(768)
    grouped = 512 + rng.integers(0, 201, size=768)
    lone = rng.integers(1, 1500, size=32)
    lens = np.concatenate([grouped, lone])
    gs = np.arange(0, 769, 8)
    pl = np.full(96, 512)
    case = inputs.grouped_case(32, 8, 128, 16, lens, gs, pl, seed=800,
                               device="cuda")
    check(case, partition_size=partition_size)


@pytest.mark.parametrize("Hq,Hkv,bs,scale", [(32, 8, 16, None), (32, 8, 16, 1.0),
                                             (8, 8, 32, None)])
def test_items_cut_across_ctas(Hq, Hkv, bs, scale):
    """One group with long private tails among many short groups: the items
    are dealt by chunks, so the long one is cut into pieces on several CTAs,
    most of which start inside the tails, where a row's first visible token
    lies chunks into the piece.  The group also holds a member shorter than
    its prefix and one that ends exactly at it.  Scale 1.0 makes the logits
    spread far beyond the rescale threshold.  The piece merge order is fixed,
    so repeated calls are bitwise equal."""
    import dataclasses
    G = Hq // Hkv
    members = 32 // G if G > 1 else 20
    P0 = 4 * bs
    rng = np.random.default_rng(Hq * 7 + bs)
    tails = rng.integers(900, 1800, size=members)
    tails[2] = -(P0 - 24)          # ends inside the prefix
    tails[3] = 0                   # ends exactly at the prefix
    tails[5] = 17
    lens = list(P0 + tails)
    gs, pl = [0, members], [P0]
    for i in range(20):
        lens += list(bs + rng.integers(0, 60, size=2))
        gs.append(gs[-1] + 2)
        pl.append(bs)
    lens += [700, 5]               # outside every group
    case = inputs.grouped_case(Hq, Hkv, 128, bs, lens, gs, pl, seed=Hq + bs + 5,
                               device="cuda")
    if scale is not None:
        case = dataclasses.replace(case, scale_override=scale)
    (_, _), a = check(case)
    b = run(case)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_cut_items_with_invalid_group_and_empty_member():
    """G = 8 (four members per 32-row tile).  A dominant group whose pass is
    cut into pieces holds an empty member (context 0: no visible token in
    any piece, output 0) and a member shorter than the prefix; an invalid
    group (prefix not a multiple of the block size) falls back to the
    per-sequence pass and is flagged; twenty small groups and two lone
    sequences fill the batch."""
    bs, P0 = 16, 160
    lens = [P0 + 1500, 0, 100, P0 + 1777]              # group 0 (dominant)
    lens += [300, 320]                                  # group 1 (made invalid below)
    gs, pl = [0, 4, 6], [P0, 48]
    rng = np.random.default_rng(64)
    for i in range(20):
        lens += list(bs + rng.integers(0, 40, size=2))
        gs.append(gs[-1] + 2)
        pl.append(bs)
    lens += [900, 3]
    case = inputs.grouped_case(64, 8, 128, bs, lens, gs, pl, seed=64, device="cuda")
    bad = torch.tensor([P0, 40] + pl[2:], dtype=torch.int32)   # 40: not whole blocks
    (_, _), out = check(case, expect_flags=pa.PA_DEVERR_PREFIX, prefix_lens=bad)
    assert torch.count_nonzero(out[1]).item() == 0


@pytest.mark.parametrize("Hkv", [1, 2, 4])
def test_cut_items_fewer_kv_heads(Hkv):
    """The split deal with 148, 74 and 37 CTAs per kv head (G = 4): one group
    with long tails among thirty short groups, so its pass is cut into many
    pieces, most of them inside the tails."""
    G, bs, P0 = 4, 16, 64
    rng = np.random.default_rng(100 + Hkv)
    lens = list(P0 + rng.integers(800, 2400, size=8))
    gs, pl = [0, 8], [P0]
    for i in range(30):
        lens += list(bs + rng.integers(0, 50, size=2))
        gs.append(gs[-1] + 2)
        pl.append(bs)
    lens += [333]
    case = inputs.grouped_case(G * Hkv, Hkv, 128, bs, lens, gs, pl, seed=200 + Hkv,
                               device="cuda")
    check(case)


@pytest.mark.parametrize("seed", range(6))
def test_random_grouped_batches(seed):
    """Randomised grouped batches: G in 1..8 with 1, 2, 4 or 8 kv heads,
    block size 16 or 32, groups of random size (one 32-row tile each) with
    prefixes of 0..40 blocks and tails of 0..1500 tokens, lone sequences
    between them, and in most seeds one group whose pass dominates (a long
    prefix or long tails), which takes the split deal.  Every output is
    compared with the oracle."""
    rng = np.random.default_rng(4000 + seed)
    Hkv = int(rng.choice([1, 2, 4, 8]))
    G = int(rng.integers(1, 9))
    bs = int(rng.choice([16, 32]))
    mpt = 32 // G if G > 1 else 16
    lens, gs, pl = [], [], []
    for gi in range(int(rng.integers(5, 30))):
        if rng.random() < 0.2:
            lens.append(int(rng.integers(0, 900)))        # a lone sequence
        m = int(rng.integers(1, mpt + 1))
        P = int(rng.integers(0, 41)) * bs
        dominant = gi == 0 and seed % 3 != 2
        tails = rng.integers(0, 2500 if dominant else 300, size=m)
        if dominant and seed % 2 == 0:
            P = int(rng.integers(150, 400)) * bs          # a long shared prefix
        start = len(lens)
        lens += [int(P + t) for t in tails]
        if rng.random() < 0.3 and m > 1:
            lens[start + 1] = int(rng.integers(0, P + 1))  # ends inside the prefix
        gs.append(start)
        pl.append(P)
    gs.append(len(lens))
    lens.append(int(rng.integers(1, 500)))               # one after the last group
    case = inputs.grouped_case(G * Hkv, Hkv, 128, bs, lens, gs, pl, seed=5000 + seed,
                               device="cuda")
    check(case)


@pytest.mark.parametrize("lone_last", [False, True])
def test_every_sequence_grouped_ragged_batch(lone_last):
    """37 sequences (the grouped bitmap's last word is partial), G = 4: every
    sequence in a valid group, one of them empty, so the per-sequence pass
    has nothing to answer; with `lone_last` the 37th sequence is outside
    every group and that pass must attend it."""
    G, Hkv, bs = 4, 8, 16
    rng = np.random.default_rng(37 + lone_last)
    lens, gs, pl = [], [], []
    while len(lens) < 37:
        m = min(int(rng.integers(1, 9)), 37 - len(lens))
        P = int(rng.integers(1, 20)) * bs
        gs.append(len(lens))
        pl.append(P)
        lens += [int(P + t) for t in rng.integers(0, 300, size=m)]
    lens[5] = 0                                              # an empty member
    if lone_last:
        if gs[-1] == 36:                                     # the last group is that one sequence
            gs.pop()
            pl.pop()
        lens[36] = 901
        gs.append(36)
    else:
        gs.append(37)
    case = inputs.grouped_case(G * Hkv, Hkv, 128, bs, lens, gs, pl, seed=370 + lone_last,
                               device="cuda")
    (_, _), out = check(case)
    assert torch.count_nonzero(out[5]).item() == 0


@pytest.mark.parametrize("scale", [1.0, 4.0])
def test_large_logits_grouped_batch(scale):
    """Scale 1 and 4: sharply peaked rows through the group pass, whole and
    cut into pieces (one long group), against the oracle."""
    G, Hkv, bs, P0 = 4, 2, 16, 64
    rng = np.random.default_rng(4200 + int(scale))
    lens = list(P0 + rng.integers(800, 2400, size=8))
    gs, pl = [0, 8], [P0]
    for i in range(12):
        lens += list(bs + rng.integers(0, 50, size=2))
        gs.append(gs[-1] + 2)
        pl.append(bs)
    case = inputs.grouped_case(G * Hkv, Hkv, 128, bs, lens, gs, pl, seed=4300 + int(scale),
                               device="cuda")
    case.scale_override = scale
    (_, _), out = check(case)
    assert torch.isfinite(out).all()

"""Seeded synthetic inputs for paged decode attention.

This module only builds inputs: shapes, context lengths, block tables laid
over a physical pool, slot mappings for the new token, copy-on-write pairs and
N(0,1) bf16 values.  It holds none of the attention, cache-write or block-copy
arithmetic, so both the CUDA library's tests/benchmark and the fp64 oracle can
draw from it.

Recipe (every draw is seeded):
  * lengths and block ids: ``numpy.random.default_rng(1000 + workload_id)``;
  * values (q, pool, new K/V): ``torch.Generator(...).manual_seed(2000 +
    workload_id)``, drawn N(0,1) in fp32 and rounded to bf16 by torch.
  * pool = (blocks the tables need) * 1.10, rounded up; the tables are a
    random permutation of pool ids, so a sequence's blocks are scattered
    ("Block-Level Management": logical blocks map to arbitrary physical
    blocks through a block table).  Table entries past a sequence's last
    block are -1.
  * the new token of sequence s sits at logical position context_lens[s]-1;
    its slot is table[s][pos // bs] * bs + pos % bs (what a block manager's
    slot allocation hands the cache write).  A sequence of length 0 gets slot
    -1 (padding).

The named workloads follow the decode shapes the pages discuss (Llama-2 7B
MHA, Llama-2 70B GQA at batch 256 from "vLLM Internals" / "Production
Performance", shared-prefix parallel sampling from "Memory Sharing via
Copy-on-Write (CoW)", and a long-context skew).  No dataset is used; these
synthetic draws stand in for real prompts.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch

POOL_SLACK = 0.10


@dataclasses.dataclass
class Workload:
    """Shape description of one decode workload."""
    name: str
    wid: int                  # seed offset
    num_seqs: int
    num_heads: int
    num_kv_heads: int
    head_size: int
    block_size: int
    lengths: str              # how to draw context lengths (see draw_lengths)
    num_blocks: Optional[int] = None   # fixed pool size (else sized + slack)
    partition_size: int = 0            # 0: library heuristic
    # shared-prefix parallel sampling
    prompts: int = 0
    samples: int = 0
    prefix_tokens: int = 0
    tail_max: int = 0
    first_prefix_tokens: int = 0      # prompt 0's prefix (0: prefix_tokens)
    # multi-query workloads: the last query_len tokens of each context are
    # the step's queries (0: decode, one query per sequence)
    query_len: int = 0
    description: str = ""

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_size)


WORKLOADS = {
    "tiny": Workload(
        "tiny", 1, 4, 4, 4, 64, 16, "fixed:1,16,17,100", num_blocks=64,
        description="4 seqs, lens {1,16,17,100}, 4q/4kv heads, D=64, bs=16, "
                    "64-block pool"),
    "llama2_7b_mha": Workload(
        "llama2_7b_mha", 2, 64, 32, 32, 128, 16, "uniform:128,2048",
        description="batch 64, 32q/32kv heads, D=128, bs=16, L~U[128,2048]"),
    "llama2_70b_gqa_b256": Workload(
        "llama2_70b_gqa_b256", 3, 256, 64, 8, 128, 16, "uniform:256,4096",
        description="batch 256, 64q/8kv heads (group 8), D=128, bs=16, "
                    "L~U[256,4096]"),
    "shared_prefix_cow": Workload(
        "shared_prefix_cow", 4, 256, 32, 8, 128, 16, "shared",
        prompts=32, samples=8, prefix_tokens=1024, tail_max=256,
        description="32 prompts x 8 samples, 1024-token shared prefix "
                    "(64 blocks, refcount 8), CoW copy of prefix block 63 per "
                    "sample, tails U[0,256]; 32q/8kv, D=128, bs=16"),
    "shared_prefix_skew": Workload(
        "shared_prefix_skew", 8, 256, 32, 8, 128, 16, "shared",
        prompts=32, samples=8, prefix_tokens=1024, tail_max=256,
        first_prefix_tokens=32768,
        description="as shared_prefix_cow, but prompt 0's prefix is 32768 "
                    "tokens (2048 blocks shared by its 8 samples): one "
                    "group's pass is several CTAs' share"),
    "long_skew_bs16": Workload(
        "long_skew_bs16", 5, 32, 32, 8, 128, 16, "skew:131072;64,1024",
        partition_size=512,
        description="32 seqs: one of 131072 tokens, 31 of U[64,1024]; "
                    "32q/8kv, D=128, bs=16, 512-token partitions"),
    "long_skew_bs32": Workload(
        "long_skew_bs32", 5, 32, 32, 8, 128, 32, "skew:131072;64,1024",
        partition_size=512,
        description="as long_skew_bs16 with bs=32"),
    "spec_verify_70b_b256": Workload(
        "spec_verify_70b_b256", 6, 256, 64, 8, 128, 16, "uniform:256,4096",
        query_len=4,
        description="speculative verification of 4 draft tokens per sequence "
                    "on the batch-256 GQA layer (64q/8kv, D=128, bs=16, "
                    "L~U[256,4096])"),
    "chunked_prefill_70b": Workload(
        "chunked_prefill_70b", 7, 16, 64, 8, 128, 16, "uniform:1024,4096",
        query_len=512,
        description="512-token prefill chunks of 16 sequences (64q/8kv, "
                    "D=128, bs=16, L~U[1024,4096] including the chunk)"),
}


@dataclasses.dataclass
class DecodeCase:
    """One decode step's inputs (pool state before the step's writes)."""
    workload: Workload
    q: torch.Tensor              # bf16 [B, Hq, D]
    k_cache: torch.Tensor        # bf16 [NB, bs, Hkv, D]
    v_cache: torch.Tensor        # bf16 [NB, bs, Hkv, D]
    block_tables: torch.Tensor   # int32 [B, MB], -1 past the last used block
    context_lens: torch.Tensor   # int32 [B]
    new_key: torch.Tensor        # bf16 [B, Hkv, D]
    new_value: torch.Tensor      # bf16 [B, Hkv, D]
    slot_mapping: torch.Tensor   # int64 [B]
    copy_pairs: torch.Tensor     # int64 [N, 2] (src, dst); N may be 0
    lens_np: np.ndarray          # int64 [B] (host copy)
    tables_np: np.ndarray        # int32 [B, MB] (host copy, after CoW remap)
    unique_tokens: int           # distinct (block, offset) positions read
    logical_tokens: int          # sum of context lengths
    scale_override: Optional[float] = None
    # multi-query cases: the last k_s context tokens of sequence s are its
    # queries; q / new_key / new_value / slot_mapping then have sum(k_s) rows
    query_start_loc: Optional[torch.Tensor] = None   # int32 [B+1]
    query_lens_np: Optional[np.ndarray] = None        # int64 [B]
    # shared-prefix cases: sequences group_start[i] .. group_start[i+1]-1
    # share their first prefix_lens[i] tokens (whole blocks)
    group_start: Optional[torch.Tensor] = None        # int32 [G+1]
    prefix_lens: Optional[torch.Tensor] = None        # int32 [G]
    max_group_size: int = 0

    @property
    def scale(self) -> float:
        if self.scale_override is not None:
            return self.scale_override
        return self.workload.scale

    @property
    def max_context_len(self) -> int:
        return int(self.lens_np.max()) if self.lens_np.size else 0


def draw_lengths(spec: str, num_seqs: int, rng: np.random.Generator) -> np.ndarray:
    kind, _, arg = spec.partition(":")
    if kind == "fixed":
        vals = [int(x) for x in arg.split(",")]
        assert len(vals) == num_seqs
        return np.array(vals, dtype=np.int64)
    if kind == "uniform":
        lo, hi = (int(x) for x in arg.split(","))
        return rng.integers(lo, hi + 1, size=num_seqs).astype(np.int64)
    if kind == "skew":
        big, rest = arg.split(";")
        lo, hi = (int(x) for x in rest.split(","))
        lens = np.empty(num_seqs, dtype=np.int64)
        lens[0] = int(big)
        lens[1:] = rng.integers(lo, hi + 1, size=num_seqs - 1)
        return lens
    raise ValueError(spec)


def blocks_for(tokens, block_size: int):
    """Number of blocks that hold ``tokens`` tokens (ceil division)."""
    return -(-np.asarray(tokens) // block_size)


def _randn_bf16(shape, gen: torch.Generator, device) -> torch.Tensor:
    return torch.randn(*shape, generator=gen, device=device,
                       dtype=torch.float32).to(torch.bfloat16)


def _generator(device, seed: int) -> torch.Generator:
    dev = torch.device(device)
    g = torch.Generator(device=dev) if dev.type == "cuda" else torch.Generator()
    g.manual_seed(seed)
    return g


def build_case(w: Workload, lens: np.ndarray, device="cpu",
               seed: Optional[int] = None, num_blocks: Optional[int] = None,
               pool_device=None,
               rng: Optional[np.random.Generator] = None) -> DecodeCase:
    """Independent (non-shared) sequences scattered over a random pool."""
    B, bs = w.num_seqs, w.block_size
    if rng is None:
        rng = np.random.default_rng(1000 + w.wid if seed is None else seed)
    nblk = blocks_for(lens, bs)
    need = int(nblk.sum())
    NB = num_blocks or w.num_blocks or max(1, math.ceil(need * (1 + POOL_SLACK)))
    if need > NB:
        raise ValueError(f"pool of {NB} blocks cannot hold {need}")
    MB = max(1, int(nblk.max()) if B else 1)
    perm = rng.permutation(NB).astype(np.int32)
    tables = np.full((B, MB), -1, dtype=np.int32)
    cursor = 0
    for s in range(B):
        n = int(nblk[s])
        tables[s, :n] = perm[cursor:cursor + n]
        cursor += n
    return _finish(w, lens, tables, NB, np.zeros((0, 2), np.int64), device,
                   2000 + w.wid if seed is None else seed + 1,
                   pool_device, unique_tokens=int(lens.sum()))


def build_shared_prefix_case(w: Workload, device="cpu",
                             seed: Optional[int] = None,
                             pool_device=None) -> DecodeCase:
    """Parallel sampling: ``samples`` sequences per prompt share the prompt's
    blocks; the prompt's last block is duplicated per sample (copy-on-write)
    before the step, and each sample's table then points at its own copy."""
    rng = np.random.default_rng(1000 + w.wid if seed is None else seed)
    bs = w.block_size
    P, S = w.prompts, w.samples
    B = P * S
    first = w.first_prefix_tokens or w.prefix_tokens
    assert B == w.num_seqs and w.prefix_tokens % bs == 0 and first % bs == 0
    prefix = np.full(P, w.prefix_tokens, dtype=np.int64)
    prefix[0] = first
    pblks = prefix // bs
    tails = rng.integers(0, w.tail_max + 1, size=B).astype(np.int64)
    lens = np.repeat(prefix, S) + tails
    tail_blocks = blocks_for(tails, bs)
    need = int(pblks.sum()) + B + int(tail_blocks.sum())
    NB = max(1, math.ceil(need * (1 + POOL_SLACK)))
    perm = rng.permutation(NB).astype(np.int32)
    cursor = 0
    prompt_blocks = []
    for p in range(P):
        prompt_blocks.append(perm[cursor:cursor + int(pblks[p])])
        cursor += int(pblks[p])
    MB = int(pblks.max()) + int(tail_blocks.max())
    tables = np.full((B, MB), -1, dtype=np.int32)
    pairs = np.zeros((B, 2), dtype=np.int64)
    for p in range(P):
        pblk = int(pblks[p])
        for j in range(S):
            s = p * S + j
            tables[s, :pblk] = prompt_blocks[p]
            private = int(perm[cursor]); cursor += 1
            pairs[s] = (prompt_blocks[p][pblk - 1], private)
            tables[s, pblk - 1] = private
            n = int(tail_blocks[s])
            tables[s, pblk:pblk + n] = perm[cursor:cursor + n]
            cursor += n
    unique = int(((pblks - 1) * bs).sum()) + B * bs + int(tails.sum())
    case = _finish(w, lens, tables, NB, pairs, device,
                   2000 + w.wid if seed is None else seed + 1, pool_device,
                   unique_tokens=unique)
    # The samples of a prompt share its blocks up to the copied last one.
    dev = torch.device(device)
    gs = (np.arange(P + 1) * S).astype(np.int32)
    pl = ((pblks - 1) * bs).astype(np.int32)
    return dataclasses.replace(case, group_start=torch.from_numpy(gs).to(dev),
                               prefix_lens=torch.from_numpy(pl).to(dev),
                               max_group_size=S)


def _finish(w: Workload, lens, tables, NB, pairs, device, vseed, pool_device,
            unique_tokens: int) -> DecodeCase:
    B, Hq, Hkv, D, bs = (w.num_seqs, w.num_heads, w.num_kv_heads, w.head_size,
                         w.block_size)
    small = _generator("cpu", vseed)
    q = _randn_bf16((B, Hq, D), small, "cpu")
    new_key = _randn_bf16((B, Hkv, D), small, "cpu")
    new_value = _randn_bf16((B, Hkv, D), small, "cpu")
    pdev = torch.device(pool_device if pool_device is not None else device)
    pg = _generator(pdev, vseed + 7)
    k_cache = _randn_bf16((NB, bs, Hkv, D), pg, pdev)
    v_cache = _randn_bf16((NB, bs, Hkv, D), pg, pdev)
    slots = np.full(B, -1, dtype=np.int64)
    for s in range(B):
        L = int(lens[s])
        if L > 0:
            pos = L - 1
            slots[s] = int(tables[s, pos // bs]) * bs + pos % bs
    dev = torch.device(device)
    return DecodeCase(
        workload=w,
        q=q.to(dev),
        k_cache=k_cache.to(dev),
        v_cache=v_cache.to(dev),
        block_tables=torch.from_numpy(tables).to(dev),
        context_lens=torch.from_numpy(lens.astype(np.int32)).to(dev),
        new_key=new_key.to(dev),
        new_value=new_value.to(dev),
        slot_mapping=torch.from_numpy(slots).to(dev),
        copy_pairs=torch.from_numpy(pairs.astype(np.int64)).to(dev),
        lens_np=lens.astype(np.int64),
        tables_np=tables,
        unique_tokens=unique_tokens,
        logical_tokens=int(lens.sum()),
    )


def make_case(name: str, device="cpu", pool_device=None,
              num_seqs: Optional[int] = None) -> DecodeCase:
    """The named workload with its fixed seeds.  ``num_seqs`` keeps only the
    first sequences of its length draw (same shapes; a smaller case)."""
    w = WORKLOADS[name]
    if w.lengths == "shared":
        if num_seqs is not None and num_seqs != w.num_seqs:
            raise ValueError("the shared-prefix workload cannot be truncated")
        return build_shared_prefix_case(w, device=device,
                                        pool_device=pool_device)
    rng = np.random.default_rng(1000 + w.wid)
    lens = draw_lengths(w.lengths, w.num_seqs, rng)
    if num_seqs is not None and num_seqs != w.num_seqs:
        lens = lens[:num_seqs]
        w = dataclasses.replace(w, num_seqs=len(lens),
                                name=f"{w.name}_first{len(lens)}")
    if w.query_len > 0:
        qlens = np.minimum(lens, w.query_len)
        case = multi_query_case(w.num_seqs, w.num_heads, w.num_kv_heads,
                                w.head_size, w.block_size, lens, qlens,
                                seed=2000 + w.wid, device=device,
                                pool_device=pool_device, name=w.name)
        return dataclasses.replace(case, workload=w)
    return build_case(w, lens, device=device, pool_device=pool_device,
                      seed=None, rng=rng)


def custom_case(num_seqs: int, num_heads: int, num_kv_heads: int,
                head_size: int, block_size: int, lens, seed: int,
                device="cpu", num_blocks: Optional[int] = None) -> DecodeCase:
    """A small ad-hoc case (tests): explicit lengths, seeded pool."""
    w = Workload(f"custom{seed}", 0, num_seqs, num_heads, num_kv_heads,
                 head_size, block_size, "fixed")
    lens = np.asarray(lens, dtype=np.int64)
    return build_case(w, lens, device=device, seed=seed,
                      num_blocks=num_blocks)


def multi_query_case(num_seqs: int, num_heads: int, num_kv_heads: int,
                     head_size: int, block_size: int, lens, query_lens,
                     seed: int, device="cpu", pool_device=None,
                     name: str = "multi_query") -> DecodeCase:
    """k_s new query tokens per sequence (chunked prefill or speculative
    verification): they occupy logical positions L_s - k_s .. L_s - 1, and
    their K/V rows are the step's new tokens with slots from the tables."""
    lens = np.asarray(lens, dtype=np.int64)
    qlens = np.asarray(query_lens, dtype=np.int64)
    assert lens.shape == qlens.shape == (num_seqs,) and np.all(qlens <= lens)
    w = Workload(name, 0, num_seqs, num_heads, num_kv_heads, head_size,
                 block_size, "fixed")
    base = build_case(w, lens, device=device, seed=seed,
                      pool_device=pool_device)
    T = int(qlens.sum())
    g = _generator("cpu", seed + 3)
    q = _randn_bf16((T, num_heads, head_size), g, "cpu")
    nk = _randn_bf16((T, num_kv_heads, head_size), g, "cpu")
    nv = _randn_bf16((T, num_kv_heads, head_size), g, "cpu")
    qsl = np.zeros(num_seqs + 1, dtype=np.int32)
    qsl[1:] = np.cumsum(qlens)
    slots = np.empty(T, dtype=np.int64)
    for s in range(num_seqs):
        for j in range(int(qlens[s])):
            pos = int(lens[s] - qlens[s] + j)
            slots[qsl[s] + j] = int(base.tables_np[s, pos // block_size]) * \
                block_size + pos % block_size
    dev = torch.device(device)
    return dataclasses.replace(
        base, q=q.to(dev), new_key=nk.to(dev), new_value=nv.to(dev),
        slot_mapping=torch.from_numpy(slots).to(dev),
        query_start_loc=torch.from_numpy(qsl).to(dev), query_lens_np=qlens)


def grouped_case(num_heads: int, num_kv_heads: int, head_size: int,
                 block_size: int, lens, group_start, prefix_lens, seed: int,
                 device="cpu", max_group_size: Optional[int] = None) -> DecodeCase:
    """Sequences whose block tables share leading blocks.  Sequence s of
    group i (group_start[i] <= s < group_start[i+1]) maps its first
    min(L_s, P_i) tokens (P_i = prefix_lens[i], whole blocks) to the group's
    blocks and the rest to private blocks; sequences outside every group
    have private blocks only.  Block ids are a seeded permutation of the
    pool.  No step writes: only the attention inputs are meaningful."""
    lens = np.asarray(lens, dtype=np.int64)
    gs = np.asarray(group_start, dtype=np.int32)
    pl = np.asarray(prefix_lens, dtype=np.int32)
    B, bs = len(lens), block_size
    rng = np.random.default_rng(seed)
    shared_of = np.zeros(B, dtype=np.int64)   # tokens mapped to group blocks
    owner = np.full(B, -1)
    for i in range(len(pl)):
        for s in range(int(gs[i]), int(gs[i + 1])):
            owner[s] = i
            shared_of[s] = min(int(lens[s]), int(pl[i]))
    group_blocks = [int(pl[i]) // bs for i in range(len(pl))]
    private = [int(blocks_for(np.array([lens[s] - shared_of[s]]), bs)[0])
               for s in range(B)]
    need = sum(group_blocks) + sum(private)
    NB = max(1, math.ceil(need * (1 + POOL_SLACK)) + 1)
    perm = rng.permutation(NB).astype(np.int32)
    cursor = 0
    gblk = []
    for n in group_blocks:
        gblk.append(perm[cursor:cursor + n])
        cursor += n
    MB = max(1, int(max(blocks_for(lens, bs).max(initial=0), 1)))
    tables = np.full((B, MB), -1, dtype=np.int32)
    for s in range(B):
        nsh = int(blocks_for(np.array([shared_of[s]]), bs)[0])
        if owner[s] >= 0 and nsh:
            tables[s, :nsh] = gblk[owner[s]][:nsh]
        n = private[s]
        tables[s, nsh:nsh + n] = perm[cursor:cursor + n]
        cursor += n
    w = Workload(f"grouped{seed}", 0, B, num_heads, num_kv_heads, head_size,
                 block_size, "fixed")
    # Distinct cached positions: each group's shared tokens once (as far as
    # its longest member reaches into them), every private token.
    unique = int((lens - shared_of).sum())
    for i in range(len(pl)):
        members = shared_of[int(gs[i]):int(gs[i + 1])]
        unique += int(members.max(initial=0))
    case = _finish(w, lens, tables, NB, np.zeros((0, 2), dtype=np.int64),
                   device, seed + 1, None, unique_tokens=unique)
    dev = torch.device(device)
    mgs = int(np.max(np.diff(gs), initial=1)) if max_group_size is None else max_group_size
    return dataclasses.replace(case, group_start=torch.from_numpy(gs).to(dev),
                               prefix_lens=torch.from_numpy(pl).to(dev),
                               max_group_size=max(1, mgs))

"""The method end to end on the GPU, driven by the library's block manager:
prompts with a prefix-cache hit, parallel samples forked from them, decode
steps whose copy-on-write pairs, slots and block tables come from the
manager, a finished sample, and a sample swapped out to pinned CPU memory and
back.  After every step the GPU pool equals the oracle's mirror of it bit for
bit, every sample's logical K/V history reads back through its block table,
and decode attention matches the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_435_b200 as pa
from paged_kv_cache_435_b200.block_manager import BlockManager
from tests.helpers import assert_attn_close

pytestmark = pytest.mark.gpu

NB, BS, HKV, HQ, D = 96, 16, 2, 8, 64


@pytest.fixture(autouse=True)
def _need_gpu():
    assert torch.cuda.is_available(), "GPU test run without a CUDA device"


def u16(t):
    return t.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


class Model:
    """GPU pool + host mirror + the logical K/V history of every sequence."""

    def __init__(self):
        self.gen = torch.Generator().manual_seed(7)
        self.k = torch.zeros(NB, BS, HKV, D, dtype=torch.bfloat16, device="cuda")
        self.v = torch.zeros_like(self.k)
        self.mk, self.mv = u16(self.k).copy(), u16(self.v).copy()
        self.hist = {}            # seq -> list of (k_row, v_row) uint16 [HKV, D]
        self.m = BlockManager(NB, BS, num_cpu_blocks=16, prefix_caching=True)
        self.cpu_k = torch.zeros(16, BS, HKV, D, dtype=torch.bfloat16).pin_memory()
        self.cpu_v = torch.zeros_like(self.cpu_k).pin_memory()
        self.mck, self.mcv = u16(self.cpu_k).copy(), u16(self.cpu_v).copy()

    def swap(self, pairs, out: bool):
        """pa_swap_blocks on the GPU, the oracle on the mirrors."""
        gpu, cpu = [self.k, self.v], [self.cpu_k, self.cpu_v]
        mg, mc = [self.mk, self.mv], [self.mck, self.mcv]
        src, dst = (gpu, cpu) if out else (cpu, gpu)
        msrc, mdst = (mg, mc) if out else (mc, mg)
        pa.pa_swap_blocks(src, dst, torch.from_numpy(pairs).cuda())
        oracle.swap_blocks(msrc, mdst, pairs)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(u16(self.cpu_k), self.mck)
        np.testing.assert_array_equal(u16(self.cpu_v), self.mcv)

    def rows(self, n):
        k = torch.randn(n, HKV, D, generator=self.gen).to(torch.bfloat16)
        v = torch.randn(n, HKV, D, generator=self.gen).to(torch.bfloat16)
        return k, v

    def write(self, k, v, slots):
        """pa_reshape_and_cache on the GPU, the oracle on the mirror."""
        pa.pa_reshape_and_cache(k.cuda(), v.cuda(), self.k, self.v,
                                torch.from_numpy(slots).cuda())
        oracle.reshape_and_cache(k, v, self.mk, self.mv, slots)

    def copy(self, pairs):
        if len(pairs):
            pa.pa_copy_blocks([self.k], [self.v], torch.from_numpy(pairs).cuda())
            oracle.copy_blocks([self.mk], [self.mv], pairs)

    def check(self, seqs):
        torch.cuda.synchronize()
        np.testing.assert_array_equal(u16(self.k), self.mk)
        np.testing.assert_array_equal(u16(self.v), self.mv)
        for s in seqs:
            tbl = self.m.block_table(s)
            hist = self.hist[s]
            assert self.m.seq_len(s) == len(hist)
            for t, (kr, vr) in enumerate(hist):
                b, o = tbl[t // BS], t % BS
                np.testing.assert_array_equal(self.mk[b, o], kr)
                np.testing.assert_array_equal(self.mv[b, o], vr)

    def attend(self, seqs):
        B = len(seqs)
        tables = [self.m.block_table(s) for s in seqs]
        MB = max(len(t) for t in tables)
        bt = np.full((B, MB), -1, dtype=np.int32)
        for i, t in enumerate(tables):
            bt[i, :len(t)] = t
        lens = np.array([self.m.seq_len(s) for s in seqs], dtype=np.int32)
        q = torch.randn(B, HQ, D, generator=self.gen).to(torch.bfloat16)
        out = torch.empty(B, HQ, D, dtype=torch.float32, device="cuda")
        maxlen = int(lens.max())
        ws_bytes = pa.pa_decode_workspace_size(B, HQ, HKV, D, BS, maxlen)
        ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device="cuda")
        pa.pa_decode_attention(out, q.cuda(), self.k, self.v,
                               torch.from_numpy(bt).cuda(),
                               torch.from_numpy(lens).cuda(), maxlen, 0.125,
                               workspace=ws)
        torch.cuda.synchronize()
        ref = oracle.paged_decode_attention(q, self.mk, self.mv, bt, lens, 0.125, HKV)
        assert_attn_close(out, ref, "manager-driven decode")


def test_manager_driven_decode_with_sharing_cow_and_swap():
    M = Model()
    prompt_a = np.arange(40, dtype=np.int32)
    prompt_b = np.concatenate([np.arange(32), 1000 + np.arange(9)]).astype(np.int32)

    a, slots, cached = M.m.add_sequence(prompt_a)
    assert cached == 0
    k, v = M.rows(40)
    M.write(k, v, slots)
    M.hist[a] = [(u16(k[i]).copy(), u16(v[i]).copy()) for i in range(40)]

    # The second prompt shares the first two full blocks through the cache.
    b, slots, cached = M.m.add_sequence(prompt_b)
    assert cached == 32 and len(slots) == 9
    k, v = M.rows(9)
    M.write(k, v, slots)
    M.hist[b] = M.hist[a][:32] + [(u16(k[i]).copy(), u16(v[i]).copy()) for i in range(9)]
    M.check([a, b])

    # Parallel sampling: 4 samples per prompt share the prompt's blocks.
    samples = [a, b]
    for p in (a, b):
        for _ in range(3):
            c = M.m.fork(p)
            M.hist[c] = list(M.hist[p])
            samples.append(c)
    # An unshared request, the one that will be preempted by swapping.
    lone, slots, _ = M.m.add_sequence(5000 + np.arange(20, dtype=np.int32))
    k, v = M.rows(20)
    M.write(k, v, slots)
    M.hist[lone] = [(u16(k[i]).copy(), u16(v[i]).copy()) for i in range(20)]
    samples.append(lone)
    M.check(samples)

    for step in range(6):
        if step == 2:                       # a sample finishes
            gone = samples.pop(3)
            M.m.free(gone)
            del M.hist[gone]
        if step == 3:                       # preempt: swap out to CPU RAM
            M.swap(M.m.swap_out(lone), out=True)
            samples.remove(lone)
        if step == 5:                       # resume into fresh GPU blocks
            M.swap(M.m.swap_in(lone), out=False)
            samples.append(lone)
            M.check(samples)
        all_slots, all_pairs, ks, vs = [], [], [], []
        for s_ in samples:
            toks = np.array([2000 + 17 * step + s_], dtype=np.int32)
            slots, pairs = M.m.append_slots(s_, 1, toks)
            all_slots.append(slots)
            all_pairs.append(pairs)
            kr, vr = M.rows(1)
            ks.append(kr)
            vs.append(vr)
            M.hist[s_].append((u16(kr[0]).copy(), u16(vr[0]).copy()))
        pairs = np.concatenate(all_pairs).astype(np.int64)
        M.copy(pairs)                       # copies read the pre-step blocks
        M.write(torch.cat(ks), torch.cat(vs), np.concatenate(all_slots))
        M.check(samples)
        M.attend(samples)
    assert len(samples) == 8

"""Pins for the oracle's multi-query (causal chunk) paged attention (CPU).

Query token j of a sequence with L cached tokens and k queries sits at
position L-k+j and sees tokens 0..L-k+j ("Chunked Prefill" and "Speculative
Decoding" on "vLLM: Anatomy and Mechanisms of High-Throughput LLM
Inference").  Pinned to torch's scaled_dot_product_attention with that mask
on the contiguous sequence, to the decode oracle at k = 1 and under
truncation, and to brute force.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from tests.test_oracle import bf16, scatter_to_pool


def problem(lens, qlens, Hq, Hkv, D, bs, seed):
    gen = torch.Generator().manual_seed(seed)
    rng = np.random.default_rng(seed)
    ks = [bf16((L, Hkv, D), gen) for L in lens]
    vs = [bf16((L, Hkv, D), gen) for L in lens]
    T = int(sum(qlens))
    q = bf16((T, Hq, D), gen)
    nb = int(sum(-(-L // bs) for L in lens)) + 3
    kp, vp, tables, lens_a = scatter_to_pool(ks, vs, bs, nb, rng)
    qsl = np.zeros(len(lens) + 1, dtype=np.int32)
    qsl[1:] = np.cumsum(qlens)
    return q, ks, vs, kp, vp, tables, lens_a, qsl


def sdpa_causal(q, ks, vs, qsl, scale):
    outs = []
    for s in range(len(ks)):
        L = ks[s].shape[0]
        k = int(qsl[s + 1] - qsl[s])
        if k == 0:
            continue
        qs = q[qsl[s]:qsl[s + 1]].double().permute(1, 0, 2)[None]   # [1,Hq,k,D]
        kk = ks[s].double().permute(1, 0, 2)[None]                   # [1,Hkv,L,D]
        vv = vs[s].double().permute(1, 0, 2)[None]
        pos = torch.arange(L)
        qpos = torch.arange(L - k, L)
        mask = pos[None, :] <= qpos[:, None]                        # [k, L]
        o = F.scaled_dot_product_attention(qs, kk, vv, attn_mask=mask,
                                           scale=scale, enable_gqa=True)
        outs.append(o[0].permute(1, 0, 2))                           # [k,Hq,D]
    return torch.cat(outs).numpy()


@pytest.mark.parametrize("Hq,Hkv,D,bs,lens,qlens", [
    (8, 2, 32, 16, [20, 40, 17], [4, 1, 7]),            # speculative verify
    (4, 4, 16, 32, [64, 33], [64, 33]),                 # whole-prompt prefill
    (16, 2, 16, 16, [100, 5, 48], [16, 5, 0]),          # chunk, full, none
    (6, 3, 8, 16, [31, 32, 33], [2, 3, 31]),
])
def test_multi_query_matches_masked_sdpa(Hq, Hkv, D, bs, lens, qlens):
    q, ks, vs, kp, vp, tables, lens_a, qsl = problem(lens, qlens, Hq, Hkv, D,
                                                     bs, seed=sum(lens))
    scale = 1.0 / math.sqrt(D)
    got = oracle.paged_multi_query_attention(q, kp, vp, tables, lens_a, qsl,
                                             scale, Hkv)
    ref = sdpa_causal(q, ks, vs, qsl, scale)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-13)


def test_single_query_equals_decode_oracle():
    lens = [1, 16, 17, 100, 250]
    q, ks, vs, kp, vp, tables, lens_a, qsl = problem(lens, [1] * 5, 8, 2, 64,
                                                     16, seed=3)
    mq = oracle.paged_multi_query_attention(q, kp, vp, tables, lens_a, qsl,
                                            0.125, 2)
    dec = oracle.paged_decode_attention(q, kp, vp, tables, lens_a, 0.125, 2)
    np.testing.assert_array_equal(mq, dec)


def test_query_j_equals_decode_of_truncated_sequence():
    lens, qlens = [90, 37], [6, 5]
    q, ks, vs, kp, vp, tables, lens_a, qsl = problem(lens, qlens, 4, 2, 32,
                                                     16, seed=8)
    mq = oracle.paged_multi_query_attention(q, kp, vp, tables, lens_a, qsl,
                                            0.2, 2)
    for s in range(2):
        for j in range(qlens[s]):
            trunc = np.array([lens[s] - qlens[s] + j + 1], dtype=np.int32)
            one = oracle.paged_decode_attention(
                q[qsl[s] + j:qsl[s] + j + 1], kp, vp, tables[s:s + 1], trunc,
                0.2, 2)
            np.testing.assert_array_equal(mq[qsl[s] + j], one[0])


def test_brute_force_tiny_causal():
    gen = torch.Generator().manual_seed(4)
    L, k, Hq, Hkv, D = 5, 3, 2, 1, 4
    kk = bf16((L, Hkv, D), gen)
    vv = bf16((L, Hkv, D), gen)
    q = bf16((k, Hq, D), gen)
    kp, vp, tables, lens_a = scatter_to_pool([kk], [vv], 16, 2,
                                             np.random.default_rng(0))
    qsl = np.array([0, k], dtype=np.int32)
    got = oracle.paged_multi_query_attention(q, kp, vp, tables, lens_a, qsl,
                                             0.9, Hkv)
    qf, kf, vf = q.double().tolist(), kk.double().tolist(), vv.double().tolist()
    for j in range(k):
        for h in range(Hq):
            last = L - k + j
            z = [0.9 * math.fsum(qf[j][h][d] * kf[t][0][d] for d in range(D))
                 for t in range(last + 1)]
            m = max(z)
            w = [math.exp(x - m) for x in z]
            for d in range(D):
                want = math.fsum(w[t] * vf[t][0][d] for t in range(last + 1)) / math.fsum(w)
                assert abs(got[j, h, d] - want) <= 1e-14 * max(1.0, abs(want))


def test_more_queries_than_context_is_an_error():
    q, ks, vs, kp, vp, tables, lens_a, qsl = problem([4], [4], 2, 2, 8, 16, 1)
    qsl = np.array([0, 5], dtype=np.int32)
    q = torch.cat([q, q[:1]])
    with pytest.raises(ValueError):
        oracle.paged_multi_query_attention(q, kp, vp, tables, lens_a, qsl, 1.0, 2)

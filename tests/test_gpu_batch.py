"""GPU checks of attn_fwd_partial_batch: each pair's result is bit-identical to the
single-pair call (keys outside a chunk weigh exactly zero either way), matches the
oracle, and the batched ring schedules match the unchunked oracle."""

from __future__ import annotations

import math

import pytest
import torch

import oracle
from parity_util import compare, to_np
from workloads import attention_inputs, get, randn_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def osx():
    import online_softmax_exact_b200 as m

    return m


PAIRS = [  # q_start, q_len, kv_start, kv_len
    (0, 300, 0, 300), (300, 500, 0, 800), (100, 129, 650, 350), (700, 300, 200, 257),
    (0, 1000, 999, 1), (512, 256, 512, 256), (37, 600, 37, 600),
]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("accumulate", [False, True])
def test_batch_equals_single_pair_calls(osx, d, causal, accumulate):
    q, k, v = (randn_bf16((2, 4, 1000, d), 13 + d, i) if i == 0 else
               randn_bf16((2, 2, 1000, d), 13 + d, i) for i in range(3))
    qg, kg, vg = q.cuda(), k.cuda(), v.cuda()
    scale = 1 / math.sqrt(d)
    g = torch.Generator(device="cuda").manual_seed(5)
    pairs, singles = [], []
    for qs, ql, ks, kl in PAIRS:
        o0 = torch.randn((2, 4, ql, d), device="cuda", generator=g)
        l0 = torch.randn((2, 4, ql), device="cuda", generator=g) * 5
        pairs.append(dict(q_start=qs, q_len=ql, kv_start=ks, kv_len=kl, o=o0.clone(),
                          lse=l0.clone()))
        o1, l1 = o0.clone(), l0.clone()
        fn = osx.attn_fwd_partial_acc if accumulate else osx.attn_fwd_partial
        fn(qg, kg, vg, q_start=qs, q_len=ql, kv_start=ks, kv_len=kl, causal=causal,
           scale=scale, o=o1, lse=l1)
        singles.append((o1, l1))
    osx.attn_fwd_partial_batch(qg, kg, vg, pairs, causal=causal, scale=scale,
                               accumulate=accumulate)
    assert osx.attn_device_status() == osx.ATTN_OK
    for pr, (o1, l1) in zip(pairs, singles):
        assert torch.equal(pr["o"], o1) and torch.equal(pr["lse"], l1)
    if not accumulate:
        for pr in pairs[:3]:
            qs, ql, ks, kl = pr["q_start"], pr["q_len"], pr["kv_start"], pr["kv_len"]
            o_ref, l_ref = oracle.attention(q[:, :, qs:qs + ql].contiguous(),
                                            k[:, :, ks:ks + kl].contiguous(),
                                            v[:, :, ks:ks + kl].contiguous(), causal=causal,
                                            scale=scale, q_off=qs, kv_off=ks)
            compare(to_np(pr["o"]), to_np(pr["lse"]), o_ref, l_ref)


@pytest.mark.parametrize("fused", [False, True])
def test_batched_ring_small(osx, fused):
    from online_softmax_exact_b200.schedules import chunks_to_sequence, ring_attention

    q, k, v = (randn_bf16((1, 4, 2048, 128), 31, i) for i in range(3))
    oc, lc = ring_attention(q.cuda(), k.cuda(), v.cuda(), n_chunks=8, causal=True,
                            batched=True, fused_merge=fused)
    o, lse = chunks_to_sequence(oc, lc)
    o_ref, l_ref = oracle.attention(q, k, v, causal=True, scale=128 ** -0.5)
    compare(to_np(o), to_np(lse), o_ref, l_ref)


@pytest.mark.parametrize("fused", [False, True])
def test_batched_ring_32k(osx, fused):
    from online_softmax_exact_b200.schedules import chunks_to_sequence, ring_attention
    from workloads import sample_rows

    w = get("ring_32k")
    q, k, v = attention_inputs(w)
    oc, lc = ring_attention(q.cuda(), k.cuda(), v.cuda(), n_chunks=w.n_chunks, causal=True,
                            scale=w.scale, batched=True, fused_merge=fused)
    assert osx.attn_device_status() == osx.ATTN_OK
    o, lse = chunks_to_sequence(oc, lc)
    rows = sample_rows(w.N, w.chunk, 48, seed=w.seed + 1)
    rt = torch.from_numpy(rows).cuda()
    o_ref, l_ref = oracle.attention_rows(q, k, v, causal=True, scale=w.scale, rows=rows)
    compare(to_np(o.index_select(2, rt)), to_np(lse.index_select(2, rt)), o_ref, l_ref)


@pytest.mark.parametrize("causal", [False, True])
def test_grouped_pairs_equal_single_pair_calls(osx, causal):
    """Pairs with equal units that read one key/value chunk run as a group, head by head
    across the group; each pair's result is still the single call's, bit for bit."""
    d = 128
    q = randn_bf16((2, 4, 2048, d), 71, 0)
    k = randn_bf16((2, 2, 2048, d), 71, 1)
    v = randn_bf16((2, 2, 2048, d), 71, 2)
    qg, kg, vg = q.cuda(), k.cuda(), v.cuda()
    spec = [(1024, 256, 512, 384), (512, 256, 512, 384), (1280, 256, 512, 384),
            (1536, 256, 512, 384), (0, 256, 512, 384), (1792, 256, 512, 384),
            (1792, 256, 0, 384)]
    pairs, singles = [], []
    for qs, ql, ks, kl in spec:
        o1, l1 = osx.attn_fwd_partial(qg, kg, vg, q_start=qs, q_len=ql, kv_start=ks,
                                      kv_len=kl, causal=causal)
        singles.append((o1, l1))
        pairs.append(dict(q_start=qs, q_len=ql, kv_start=ks, kv_len=kl,
                          o=torch.empty_like(o1), lse=torch.empty_like(l1)))
    osx.attn_fwd_partial_batch(qg, kg, vg, pairs, causal=causal)
    assert osx.attn_device_status() == osx.ATTN_OK
    for pr, (o1, l1) in zip(pairs, singles):
        assert torch.equal(pr["o"], o1) and torch.equal(pr["lse"], l1)
    pr = pairs[3]
    o_ref, l_ref = oracle.attention(q[:, :, 1536:1792].contiguous(),
                                    k[:, :, 512:896].contiguous(), v[:, :, 512:896].contiguous(),
                                    causal=causal, scale=d ** -0.5, q_off=1536, kv_off=512)
    compare(to_np(pr["o"]), to_np(pr["lse"]), o_ref, l_ref)

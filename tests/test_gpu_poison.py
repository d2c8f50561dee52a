"""Rows outside a pair's chunks never reach its result.

A batched launch maps whole parent tensors, so a pair whose chunk ends inside a key
tile reads the parent's next rows into that tile (and a query tile past the chunk's
end reads the next query rows). Those rows may hold anything: uninitialised memory,
or, in the host-buffer ring call, a chunk whose copy is still in flight. Here they
are NaN, and every result must still equal the oracle's ("Ring Attention with
Blockwise Parallel Transformers", section 3: each block's attention is computed
exactly; nothing outside the block enters it).
"""

from __future__ import annotations

import math

import pytest
import torch

import oracle
from parity_util import compare, to_np
from workloads import randn_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def osx():
    import online_softmax_exact_b200 as m

    return m


def _poisoned_parent(shape, live, seed, tensor_id):
    """bf16 [B, H, L, d] that is NaN except on the row ranges in ``live``, where it
    holds N(0, 1) draws."""
    t = torch.full(shape, math.nan, dtype=torch.bfloat16)
    full = randn_bf16(shape, seed, tensor_id)
    for a, b in live:
        t[:, :, a:b] = full[:, :, a:b]
    return t


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n_chunks,N", [(4, 1000), (3, 390), (5, 1285)])
def test_ring_host_with_nan_staging(osx, d, causal, n_chunks, N):
    """attn_ring_fwd_host with chunks that are not multiples of the 128-row tile and
    device staging buffers full of NaN before the call: under the causal mask a pair
    launches as soon as its query chunk has arrived, while the next chunk's rows,
    which its last tiles read, are still NaN or in flight."""
    B, Hq, Hkv = 1, 4, 2
    q = randn_bf16((B, Hq, N, d), 61 + d, 0)
    k = randn_bf16((B, Hkv, N, d), 61 + d, 1)
    v = randn_bf16((B, Hkv, N, d), 61 + d, 2)
    bufs = osx.RingHostBuffers(B, Hq, Hkv, N, d, n_chunks, torch.device("cuda"))
    for t in bufs.tensors():
        t.fill_(math.nan)
    qh, kh, vh = q.pin_memory(), k.pin_memory(), v.pin_memory()
    o_h, l_h = osx.attn_ring_fwd_host(qh, kh, vh, n_chunks=n_chunks, causal=causal,
                                      buffers=bufs)
    torch.cuda.synchronize()
    assert osx.attn_device_status() == osx.ATTN_OK
    from online_softmax_exact_b200.schedules import chunks_to_sequence

    o, lse = chunks_to_sequence(o_h, l_h)
    o_ref, l_ref = oracle.attention(q, k, v, causal=causal, scale=d ** -0.5)
    compare(o.numpy(), lse.numpy(), o_ref, l_ref)


# (q_start, q_len, kv_start, kv_len, q_off, kv_off): chunk ends fall inside 128-row
# tiles next to NaN rows of the parents
PAIRS = [
    (64, 300, 50, 333, 400, 100),
    (500, 257, 600, 130, 700, 600),
    (64, 300, 800, 257, 1100, 800),
    (380, 100, 0, 1, 380, 0),
]
LQ, LKV = 900, 1100


def _parents(d, seed):
    q_live = sorted({(p[0], p[0] + p[1]) for p in PAIRS})
    kv_live = sorted({(p[2], p[2] + p[3]) for p in PAIRS})
    q = _poisoned_parent((2, 4, LQ, d), q_live, seed, 0)
    k = _poisoned_parent((2, 2, LKV, d), kv_live, seed, 1)
    v = _poisoned_parent((2, 2, LKV, d), kv_live, seed, 2)
    return q, k, v


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_batched_pairs_in_nan_parents(osx, d, causal):
    q, k, v = _parents(d, 70 + d)
    qg, kg, vg = q.cuda(), k.cuda(), v.cuda()
    scale = d ** -0.5
    outs = []
    pairs = []
    for qs, ql, ks, kl, qo, ko in PAIRS:
        o = torch.full((2, 4, ql, d), math.nan, device="cuda")
        lse = torch.full((2, 4, ql), math.nan, device="cuda")
        outs.append((o, lse))
        pairs.append(dict(q_start=qs, q_len=ql, kv_start=ks, kv_len=kl, q_off=qo, kv_off=ko,
                          o=o, lse=lse))
    osx.attn_fwd_partial_batch(qg, kg, vg, pairs, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert osx.attn_device_status() == osx.ATTN_OK
    for (qs, ql, ks, kl, qo, ko), (o, lse) in zip(PAIRS, outs):
        o_ref, l_ref = oracle.attention(q[:, :, qs:qs + ql].contiguous(),
                                        k[:, :, ks:ks + kl].contiguous(),
                                        v[:, :, ks:ks + kl].contiguous(), causal=causal,
                                        scale=scale, q_off=qo, kv_off=ko)
        compare(to_np(o), to_np(lse), o_ref, l_ref)


@pytest.mark.parametrize("d", [64, 128])
def test_batched_accumulate_in_nan_parents(osx, d):
    """accumulate=1: each pair folds a second key chunk, read from inside NaN parents,
    into an accumulator that already holds the first chunk's partial."""
    q, k, v = _parents(d, 80 + d)
    qg, kg, vg = q.cuda(), k.cuda(), v.cuda()
    scale = d ** -0.5
    first = (50, 333)     # keys every pair has seen already
    second = [(600, 130), (800, 257), (0, 1)]
    qs, ql = 64, 300
    accs, pairs = [], []
    for ks, kl in second:
        o, lse = osx.attn_fwd_partial(qg, kg, vg, q_start=qs, q_len=ql, kv_start=first[0],
                                      kv_len=first[1], causal=False, scale=scale)
        accs.append((o, lse))
        pairs.append(dict(q_start=qs, q_len=ql, kv_start=ks, kv_len=kl, o=o, lse=lse))
    # pairs writing to distinct accumulators, all reading query rows [64, 364)
    osx.attn_fwd_partial_batch(qg, kg, vg, pairs, causal=False, scale=scale, accumulate=True)
    torch.cuda.synchronize()
    assert osx.attn_device_status() == osx.ATTN_OK
    qc = q[:, :, qs:qs + ql].contiguous()
    for (ks, kl), (o, lse) in zip(second, accs):
        kk = torch.cat([k[:, :, first[0]:first[0] + first[1]], k[:, :, ks:ks + kl]], dim=2)
        vv = torch.cat([v[:, :, first[0]:first[0] + first[1]], v[:, :, ks:ks + kl]], dim=2)
        o_ref, l_ref = oracle.attention(qc, kk.contiguous(), vv.contiguous(), causal=False,
                                        scale=scale)
        compare(to_np(o), to_np(lse), o_ref, l_ref)

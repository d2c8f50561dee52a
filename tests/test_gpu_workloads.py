"""GPU parity at the full sizes of the five workloads, in the launch configuration the
benchmark times, on sampled rows the oracle computes one by one (every chunk's first
and last rows, rows around 128-row tile boundaries, plus seeded uniform rows)."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from parity_util import compare, to_np
from workloads import attention_inputs, get, grid_merge_orders, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def osx():
    import online_softmax_exact_b200 as m

    return m


def check_sampled(o_seq, lse_seq, q, k, v, w, rows_per_head):
    rows = sample_rows(w.N, w.chunk, rows_per_head, seed=w.seed)
    rows_t = torch.from_numpy(rows).to(o_seq.device)
    o_s = to_np(o_seq.index_select(2, rows_t))
    l_s = to_np(lse_seq.index_select(2, rows_t))
    o_ref, l_ref = oracle.attention_rows(q, k, v, causal=w.causal, scale=w.scale, rows=rows)
    do, dl = compare(o_s, l_s, o_ref, l_ref)
    print(f"{w.name}: {len(rows)} rows/head, max|dO|={do:.2e} max|dLSE|={dl:.2e}")


def test_causal_4k_single_pass(osx):
    w = get("causal_4k")
    q, k, v = attention_inputs(w)
    o, lse = osx.attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=w.causal, scale=w.scale)
    assert osx.attn_device_status() == osx.ATTN_OK
    check_sampled(o, lse, q, k, v, w, 256)


def test_ring_32k(osx):
    from online_softmax_exact_b200.schedules import chunks_to_sequence, ring_attention

    w = get("ring_32k")
    q, k, v = attention_inputs(w)
    oc, lc = ring_attention(q.cuda(), k.cuda(), v.cuda(), n_chunks=w.n_chunks, causal=w.causal,
                            scale=w.scale)
    assert osx.attn_device_status() == osx.ATTN_OK
    o, lse = chunks_to_sequence(oc, lc)
    check_sampled(o, lse, q, k, v, w, 96)


def test_ring_32k_fused_merge(osx):
    from online_softmax_exact_b200.schedules import chunks_to_sequence, ring_attention

    w = get("ring_32k")
    q, k, v = attention_inputs(w)
    oc, lc = ring_attention(q.cuda(), k.cuda(), v.cuda(), n_chunks=w.n_chunks, causal=w.causal,
                            scale=w.scale, fused_merge=True, n_streams=2)
    assert osx.attn_device_status() == osx.ATTN_OK
    o, lse = chunks_to_sequence(oc, lc)
    check_sampled(o, lse, q, k, v, w, 64)


def test_gqa_128k_single_pass(osx):
    w = get("gqa_128k")
    q, k, v = attention_inputs(w)
    o, lse = osx.attn_fwd(q.cuda(), k.cuda(), v.cuda(), causal=w.causal, scale=w.scale)
    assert osx.attn_device_status() == osx.ATTN_OK
    check_sampled(o, lse, q, k, v, w, 48)


def test_grid2d_64k_stress(osx):
    from online_softmax_exact_b200.schedules import chunks_to_sequence, grid2d_attention

    w = get("grid2d_64k_stress")
    q, k, v = attention_inputs(w)
    qg, kg, vg = q.cuda(), k.cuda(), v.cuda()
    # per-cell launches and the batched launch the benchmark times, each with partial
    # buffers and merges and with the fused running merge
    for batched in (False, True):
        for fused in (False, True):
            oc, lc = grid2d_attention(qg, kg, vg, n_chunks=w.n_chunks,
                                      merge_orders=grid_merge_orders(w.n_chunks, w.seed),
                                      causal=w.causal, scale=w.scale, fused_merge=fused,
                                      batched=batched)
            assert osx.attn_device_status() == osx.ATTN_OK
            o, lse = chunks_to_sequence(oc, lc)
            check_sampled(o, lse, q, k, v, w, 96 if batched and not fused else 32)


def test_large_causal_gqa_over_key_value_head_bands(osx):
    """A one-pair causal call whose K/V exceed L2 is launched over bands of key/value
    heads (here B = 2, 8 key/value heads of 4 query heads, N = 65536: one key/value head
    per launch, sixteen launches). Every band's O and LSE rows, in both batches, must equal
    the oracle's; a partial on a chunk of the parents with global offsets, folded into an
    accumulator, goes the same way."""
    from workloads.gen import randn_bf16

    B, Hq, Hkv, N, d = 2, 32, 8, 65536, 128
    q = randn_bf16((B, Hq, N, d), 21, 0)
    k = randn_bf16((B, Hkv, N, d), 21, 1)
    v = randn_bf16((B, Hkv, N, d), 21, 2)
    qg, kg, vg = q.cuda(), k.cuda(), v.cuda()
    scale = d ** -0.5
    launches = osx.attn_launch_count()
    o, lse = osx.attn_fwd(qg, kg, vg, causal=True, scale=scale)
    assert osx.attn_device_status() == osx.ATTN_OK
    assert osx.attn_launch_count() - launches == 16
    rows = sample_rows(N, 16384, 40, seed=21)
    rows_t = torch.from_numpy(rows).cuda()
    o_ref, l_ref = oracle.attention_rows(q, k, v, causal=True, scale=scale, rows=rows)
    do, dl = compare(to_np(o.index_select(2, rows_t)), to_np(lse.index_select(2, rows_t)),
                     o_ref, l_ref)
    print(f"banded GQA B=2: {len(rows)} rows/head, max|dO|={do:.2e} max|dLSE|={dl:.2e}")
    # the second half of the keys folded into the first half's partial: the whole result
    h = N // 2
    acc_o, acc_l = osx.attn_fwd_partial(qg, kg, vg, q_start=0, q_len=N, kv_start=0, kv_len=h,
                                        causal=True, scale=scale)
    osx.attn_fwd_partial_acc(qg, kg, vg, q_start=0, q_len=N, kv_start=h, kv_len=h,
                             causal=True, scale=scale, o=acc_o, lse=acc_l)
    assert osx.attn_device_status() == osx.ATTN_OK
    compare(to_np(acc_o.index_select(2, rows_t)), to_np(acc_l.index_select(2, rows_t)),
            o_ref, l_ref)

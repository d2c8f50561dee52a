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

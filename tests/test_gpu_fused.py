"""GPU parity of the fused running merge (attn_fwd_partial_acc) and of the ring and 2-D
grid schedules run with it, against the fp64 oracle."""

from __future__ import annotations

import math

import numpy as np
import pytest
import torch

import oracle
from parity_util import MERGE_LSE_ULPS, TOL_MERGE, compare, to_np
from workloads import grid_merge_orders, randn_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def osx():
    import online_softmax_exact_b200 as m

    return m


def inputs(B, Hq, Hkv, Nq, Nkv, d, seed):
    return (randn_bf16((B, Hq, Nq, d), seed, 0), randn_bf16((B, Hkv, Nkv, d), seed, 1),
            randn_bf16((B, Hkv, Nkv, d), seed, 2))


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal,q_start", [(False, 0), (True, 500), (True, 128)])
def test_two_chunks_accumulated_equal_the_unchunked_result(osx, d, causal, q_start):
    q, k, v = inputs(1, 4, 2, 800, 900, d, seed=d + q_start)
    qg, kg, vg = q.cuda(), k.cuda(), v.cuda()
    scale = 1 / math.sqrt(d)
    Nq = 300
    o, lse = osx.attn_fwd_partial(qg, kg, vg, q_start=q_start, q_len=Nq, kv_start=0,
                                  kv_len=411, causal=causal, scale=scale)
    osx.attn_fwd_partial_acc(qg, kg, vg, q_start=q_start, q_len=Nq, kv_start=411, kv_len=489,
                             causal=causal, scale=scale, o=o, lse=lse)
    assert osx.attn_device_status() == osx.ATTN_OK
    o_ref, l_ref = oracle.attention(q[:, :, q_start:q_start + Nq].contiguous(), k, v,
                                    causal=causal, scale=scale, q_off=q_start)
    compare(to_np(o), to_np(lse), o_ref, l_ref)


def test_accumulate_matches_the_merge_of_the_same_partials(osx):
    q, k, v = inputs(1, 4, 4, 512, 512, 128, seed=3)
    qg, kg, vg = q.cuda(), k.cuda(), v.cuda()
    a = osx.attn_fwd_partial(qg, kg, vg, q_start=0, q_len=512, kv_start=0, kv_len=200,
                             causal=False)
    b = osx.attn_fwd_partial(qg, kg, vg, q_start=0, q_len=512, kv_start=200, kv_len=312,
                             causal=False)
    acc_o, acc_l = a[0].clone(), a[1].clone()
    osx.attn_fwd_partial_acc(qg, kg, vg, q_start=0, q_len=512, kv_start=200, kv_len=312,
                             causal=False, o=acc_o, lse=acc_l)
    o64, l64 = oracle.merge([to_np(a[0]), to_np(b[0])], [to_np(a[1]), to_np(b[1])])
    # The accumulating call forms the same scores, the same bf16 P and the same TMEM
    # accumulator and denominator l as the plain partial b, so the two paths differ only
    # in their final fp32 operations: the fused epilogue computes
    # a * O_acc + (w_new / (w_acc + w_new) / l) * O_tmem, the merge w-weights the stored
    # O_tmem / l. That is a handful of roundings of 2^-24 relative each, plus the
    # ex2/lg2 approximations (2^-22 relative) in the weights, on |O| of order 1: far
    # below 1e-5, so the merge's own bound applies.
    compare(to_np(acc_o), to_np(acc_l), o64, l64, tol_o=TOL_MERGE, tol_lse=TOL_MERGE,
            lse_ulps=MERGE_LSE_ULPS)


@pytest.mark.parametrize("d", [64, 128])
def test_empty_accumulator_gives_the_plain_partial(osx, d):
    """At d = 128 the plain partial stores O through the shared-memory staging buffer and
    the accumulating call stores it row by row: the two store paths must agree."""
    q, k, v = inputs(2, 4, 2, 384, 384, d, seed=9)
    qg, kg, vg = q.cuda(), k.cuda(), v.cuda()
    plain = osx.attn_fwd_partial(qg, kg, vg, q_start=0, q_len=384, kv_start=0, kv_len=384,
                                 causal=True)
    o = torch.zeros_like(plain[0])
    lse = torch.full_like(plain[1], -math.inf)
    osx.attn_fwd_partial_acc(qg, kg, vg, q_start=0, q_len=384, kv_start=0, kv_len=384,
                             causal=True, o=o, lse=lse)
    compare(to_np(o), to_np(lse), to_np(plain[0]), to_np(plain[1]), tol_o=1e-6,
            tol_lse=1e-6, lse_ulps=MERGE_LSE_ULPS)


def test_chunk_hidden_by_the_mask_leaves_the_accumulator_unchanged(osx):
    q, k, v = inputs(1, 2, 2, 512, 512, 128, seed=4)
    qg, kg, vg = q.cuda(), k.cuda(), v.cuda()
    o, lse = osx.attn_fwd_partial(qg, kg, vg, q_start=0, q_len=256, kv_start=0, kv_len=256,
                                  causal=True)
    o0, l0 = o.clone(), lse.clone()
    osx.attn_fwd_partial_acc(qg, kg, vg, q_start=0, q_len=256, kv_start=256, kv_len=256,
                             causal=True, o=o, lse=lse)
    assert torch.equal(o, o0) and torch.equal(lse, l0)


@pytest.mark.parametrize("n_streams", [1, 2])
def test_ring_with_fused_merge(osx, n_streams):
    from online_softmax_exact_b200.schedules import chunks_to_sequence, ring_attention

    q, k, v = inputs(1, 4, 4, 1024, 1024, 128, seed=21)
    oc, lc = ring_attention(q.cuda(), k.cuda(), v.cuda(), n_chunks=4, causal=True,
                            fused_merge=True, n_streams=n_streams)
    o, lse = chunks_to_sequence(oc, lc)
    o_ref, l_ref = oracle.attention(q, k, v, causal=True, scale=128 ** -0.5)
    compare(to_np(o), to_np(lse), o_ref, l_ref)


def test_grid2d_with_fused_merge(osx):
    from online_softmax_exact_b200.schedules import chunks_to_sequence, grid2d_attention

    q, k, v = inputs(1, 2, 2, 1024, 1024, 64, seed=22)
    q = q * 8
    oc, lc = grid2d_attention(q.cuda(), k.cuda(), v.cuda(), n_chunks=4,
                              merge_orders=grid_merge_orders(4, 7), causal=False,
                              fused_merge=True)
    o, lse = chunks_to_sequence(oc, lc)
    o_ref, l_ref = oracle.attention(q, k, v, causal=False, scale=64 ** -0.5)
    compare(to_np(o), to_np(lse), o_ref, l_ref)

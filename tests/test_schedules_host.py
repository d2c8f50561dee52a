"""Host logic of the one-GPU chunk schedules (schedules.py), without a GPU: the chunk
split, the ring order ("Ring Attention with Blockwise Parallel Transformers", section 3:
at step s query block i holds key/value block (i - s) mod P), the partial-slot counts,
the stream balancing and the chunk-major to sequence layout."""

from __future__ import annotations

import itertools

import pytest
import torch

from online_softmax_exact_b200 import schedules


@pytest.mark.parametrize("N,P", [(256, 4), (32768, 8), (12, 3), (7, 1)])
def test_chunk_bounds_tile_the_sequence(N, P):
    b = schedules.chunk_bounds(N, P)
    assert len(b) == P and b[0][0] == 0 and b[-1][1] == N
    assert all(e - s == N // P for s, e in b)
    assert all(b[i][1] == b[i + 1][0] for i in range(P - 1))


@pytest.mark.parametrize("N,P", [(10, 3), (8, 0)])
def test_chunk_bounds_reject_unequal_chunks(N, P):
    with pytest.raises(ValueError):
        schedules.chunk_bounds(N, P)


@pytest.mark.parametrize("P", [1, 2, 3, 8])
def test_ring_order_non_causal_visits_every_chunk_once_in_ring_order(P):
    order = schedules.ring_order(P, causal=False)
    for i, visit in enumerate(order):
        assert visit == [(i - s) % P for s in range(P)]
        assert sorted(visit) == list(range(P))


@pytest.mark.parametrize("P", [1, 2, 3, 8])
def test_ring_order_causal_skips_exactly_the_later_chunks(P):
    order = schedules.ring_order(P, causal=True)
    for i, visit in enumerate(order):
        # step 0 is the diagonal, then chunks i-1, i-2, ... 0: the hidden ones are gone
        assert visit == list(range(i, -1, -1))
    # 8 chunks: 36 visible pairs (28 full + 8 diagonal), the ring_32k step
    if P == 8:
        assert sum(len(v) for v in order) == 36


@pytest.mark.parametrize("P,causal", [(8, True), (8, False), (4, True), (1, False)])
def test_ring_slots(P, causal):
    order = schedules.ring_order(P, causal)
    batched = schedules.ring_slots(P, causal, batched=True)
    assert batched == sum(len(v) for v in order if len(v) > 1)
    for n_streams in (1, 2, 4):
        s = schedules.ring_slots(P, causal, batched=False, n_streams=n_streams)
        assert s == max(len(v) for v in order) * min(n_streams, P)


def test_balance_streams_is_greedy_heaviest_first():
    costs = [8.0, 7.0, 6.0, 5.0, 4.0, 3.0, 2.0, 1.0]
    assign = schedules.balance_streams(costs, 2)
    loads = [sum(c for c, a in zip(costs, assign) if a == s) for s in range(2)]
    assert sorted(loads) == [18.0, 18.0]
    # the greedy rule never leaves a stream idle while another holds two or more chunks
    assign = schedules.balance_streams([1.0] * 3, 4)
    assert len(set(assign)) == 3


def test_balance_streams_bounded_by_the_optimum_plus_the_largest_cost():
    costs = [float(c) for c in (9, 7, 7, 5, 3, 3, 2, 1)]
    for n in (1, 2, 3):
        assign = schedules.balance_streams(costs, n)
        loads = [sum(c for c, a in zip(costs, assign) if a == s) for s in range(n)]
        best = min(max(sum(c for c, a in zip(costs, p) if a == s) for s in range(n))
                   for p in itertools.product(range(n), repeat=len(costs)))
        assert max(loads) <= best + max(costs)


def test_chunks_to_sequence_places_each_chunk_at_its_rows():
    P, B, Hq, C, d = 3, 2, 2, 4, 5
    o = torch.arange(P * B * Hq * C * d, dtype=torch.float32).reshape(P, B, Hq, C, d)
    lse = torch.arange(P * B * Hq * C, dtype=torch.float32).reshape(P, B, Hq, C)
    so, sl = schedules.chunks_to_sequence(o, lse)
    assert so.shape == (B, Hq, P * C, d) and sl.shape == (B, Hq, P * C)
    for c in range(P):
        assert torch.equal(so[:, :, c * C:(c + 1) * C], o[c])
        assert torch.equal(sl[:, :, c * C:(c + 1) * C], lse[c])

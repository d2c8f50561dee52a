"""GPU checks of attn_ring_fwd_host (Ring Attention's schedule from host buffers to host
buffers, copies pipelined with the compute): its result is bit-identical to the same
schedule run on device buffers (ring_attention, batched), and matches the oracle."""

from __future__ import annotations

import pytest
import torch

import oracle
from parity_util import compare, to_np
from workloads import attention_inputs, get, randn_bf16, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def osx():
    import online_softmax_exact_b200 as m

    return m


def _device_ring(q, k, v, n_chunks, causal, scale):
    from online_softmax_exact_b200.schedules import ring_attention

    return ring_attention(q.cuda(), k.cuda(), v.cuda(), n_chunks=n_chunks, causal=causal,
                          scale=scale, batched=True)


@pytest.mark.parametrize("shape,n_chunks,causal,pinned", [
    ((1, 4, 2, 2048, 128), 4, True, True),
    ((2, 2, 2, 1024, 64), 4, False, True),
    ((1, 4, 4, 1536, 128), 3, True, False),   # pageable host memory: copies unoverlapped
    ((1, 2, 1, 768, 64), 1, True, True),      # one chunk: no merge, no partial buffers
])
def test_ring_host_equals_device_schedule(osx, shape, n_chunks, causal, pinned):
    from online_softmax_exact_b200.schedules import chunks_to_sequence

    B, Hq, Hkv, N, d = shape
    q = randn_bf16((B, Hq, N, d), 41 + d, 0)
    k = randn_bf16((B, Hkv, N, d), 41 + d, 1)
    v = randn_bf16((B, Hkv, N, d), 41 + d, 2)
    scale = d ** -0.5
    qh, kh, vh = (t.pin_memory() if pinned else t for t in (q, k, v))
    o_h, l_h = osx.attn_ring_fwd_host(qh, kh, vh, n_chunks=n_chunks, causal=causal, scale=scale)
    torch.cuda.synchronize()
    assert osx.attn_device_status() == osx.ATTN_OK
    oc, lc = _device_ring(q, k, v, n_chunks, causal, scale)
    assert torch.equal(o_h, oc.cpu()) and torch.equal(l_h, lc.cpu())
    o, lse = chunks_to_sequence(o_h, l_h)
    o_ref, l_ref = oracle.attention(q, k, v, causal=causal, scale=scale)
    compare(o.numpy(), lse.numpy(), o_ref, l_ref)


def test_ring_host_reuses_buffers_and_streams(osx):
    """Two calls back to back with the same device buffers and copy streams, on inputs
    that differ, each give their own result."""
    B, Hq, Hkv, N, d, P = 1, 2, 2, 1024, 128, 4
    bufs = osx.RingHostBuffers(B, Hq, Hkv, N, d, P, torch.device("cuda"))
    outs = []
    for seed in (3, 4):
        q, k, v = (randn_bf16((B, Hq, N, d), seed, i).pin_memory() for i in range(3))
        outs.append((osx.attn_ring_fwd_host(q, k, v, n_chunks=P, causal=True, buffers=bufs),
                     (q, k, v)))
    torch.cuda.synchronize()
    for (o_h, l_h), (q, k, v) in outs:
        oc, lc = _device_ring(q, k, v, P, True, d ** -0.5)
        assert torch.equal(o_h, oc.cpu()) and torch.equal(l_h, lc.cpu())


def test_ring_host_32k(osx):
    """The ring_32k step from host buffers: bit-identical to the device schedule, and
    sampled rows against the oracle."""
    from online_softmax_exact_b200.schedules import chunks_to_sequence

    w = get("ring_32k")
    q, k, v = attention_inputs(w)
    o_h, l_h = osx.attn_ring_fwd_host(q.pin_memory(), k.pin_memory(), v.pin_memory(),
                                      n_chunks=w.n_chunks, causal=True, scale=w.scale)
    torch.cuda.synchronize()
    assert osx.attn_device_status() == osx.ATTN_OK
    oc, lc = _device_ring(q, k, v, w.n_chunks, True, w.scale)
    assert torch.equal(o_h, oc.cpu()) and torch.equal(l_h, lc.cpu())
    o, lse = chunks_to_sequence(o_h, l_h)
    rows = sample_rows(w.N, w.chunk, 32, seed=w.seed + 2)
    rt = torch.from_numpy(rows)
    o_ref, l_ref = oracle.attention_rows(q, k, v, causal=True, scale=w.scale, rows=rows)
    compare(to_np(o.index_select(2, rt)), to_np(lse.index_select(2, rt)), o_ref, l_ref)

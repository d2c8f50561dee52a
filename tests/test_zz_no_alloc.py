"""attn_ring_fwd_host_noalloc, the host-buffer ring call that allocates no device memory,
against attn_ring_fwd_host on the same inputs.

The entry point is for callers that cannot call cudaMalloc (for example, code in a
process whose device memory belongs to another allocator, or a latency-critical path
where an allocation would synchronise the device): its staging buffers and partial
slots live in a fixed array of the library's own device data. It runs the same kernels
in the same order as attn_ring_fwd_host, so its results must agree with that call's
within the parity tolerance (in fact bit for bit), on two calls in a row, the second
reusing the array the first left behind.

This file is collected last on purpose: it also passes when run alone in a fresh
process, where its first call does the per-device set-up.
"""

from __future__ import annotations

import ctypes

import pytest
import torch

from parity_util import compare
from workloads import randn_bf16

pytestmark = pytest.mark.gpu


def _noalloc(lib, q, k, v, o, lse, n_chunks, causal, scale, stream):
    B, Hq, N, d = q.shape
    return lib.attn_ring_fwd_host_noalloc(
        q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), B, Hq,
        k.shape[1], N, d, n_chunks, int(causal), float(scale), ctypes.c_void_p(stream),
        None, None)


@pytest.mark.parametrize("shape,n_chunks,causal", [
    ((1, 4, 2, 1000, 128), 4, True),     # chunks of 250: ragged key tiles, GQA
    ((2, 2, 2, 1024, 64), 2, False),
])
def test_noalloc_matches_the_allocating_call_twice_in_a_row(shape, n_chunks, causal):
    import online_softmax_exact_b200 as osx

    lib = osx.lib()
    B, Hq, Hkv, N, d = shape
    C = N // n_chunks
    scale = d ** -0.5
    stream = torch.cuda.current_stream()
    for call, seed in enumerate((91, 92)):
        q = randn_bf16((B, Hq, N, d), seed, 0).pin_memory()
        k = randn_bf16((B, Hkv, N, d), seed, 1).pin_memory()
        v = randn_bf16((B, Hkv, N, d), seed, 2).pin_memory()
        o = torch.full((n_chunks, B, Hq, C, d), float("nan")).pin_memory()
        lse = torch.full((n_chunks, B, Hq, C), float("nan")).pin_memory()
        st = _noalloc(lib, q, k, v, o, lse, n_chunks, causal, scale, stream.cuda_stream)
        assert st == osx.ATTN_OK, f"call {call}: {osx.attn_status_string(st)}"
        torch.cuda.synchronize()
        assert osx.attn_device_status() == osx.ATTN_OK
        o_ref, l_ref = osx.attn_ring_fwd_host(q, k, v, n_chunks=n_chunks, causal=causal,
                                              scale=scale)
        torch.cuda.synchronize()
        compare(o.numpy(), lse.numpy(), o_ref.numpy(), l_ref.numpy())
        assert torch.equal(o, o_ref) and torch.equal(lse, l_ref)


def test_noalloc_rejects_sizes_beyond_its_array():
    import online_softmax_exact_b200 as osx

    lib = osx.lib()
    limit = int(osx.ATTN_NOALLOC_SCRATCH_BYTES)
    # Q alone (bf16) would need more than the whole array: nothing is read or launched
    B, Hq, d = 1, 8, 128
    N = limit // (B * Hq * d * 2) + 128
    one = torch.empty(1, dtype=torch.bfloat16)
    st = lib.attn_ring_fwd_host_noalloc(one.data_ptr(), one.data_ptr(), one.data_ptr(),
                                        one.data_ptr(), one.data_ptr(), B, Hq, Hq, N, d, 1, 1,
                                        0.1, None, None, None)
    assert st == osx.ATTN_ERR_UNSUPPORTED

"""The cross-rank schedules on a one-rank NCCL group, with the default local compute
(the library's kernels on the rank's own GPU and stream), against the fp64 oracle.
With one rank the ring is one fold of the rank's own chunk (two folds of its halves
in the zigzag layout), the 1 x 1 grid one fragment, and Ulysses' all-to-all
exchanges copy within the rank; what this adds to the multi-rank tests (several
gloo ranks on the host, test_gpu_dist_kernels.py) is the NCCL path with device
tensors."""

from __future__ import annotations

import pytest
import torch

import oracle
from parity_util import compare, to_np
from workloads import randn_bf16

pytestmark = pytest.mark.gpu


@pytest.fixture
def nccl_one_rank():
    import torch.distributed as dist

    dist.init_process_group("nccl", store=dist.HashStore(), rank=0, world_size=1)
    try:
        yield
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("layout", ["contiguous", "zigzag"])
def test_one_rank_ring(nccl_one_rank, causal, layout):
    import online_softmax_exact_b200 as osx
    from online_softmax_exact_b200.ring_dist import ring_attention_dist

    q = randn_bf16((1, 4, 1000, 128), 23, 0)
    k = randn_bf16((1, 2, 1000, 128), 23, 1)
    v = randn_bf16((1, 2, 1000, 128), 23, 2)
    o, lse = ring_attention_dist(q.cuda(), k.cuda(), v.cuda(), causal=causal, layout=layout)
    torch.cuda.synchronize()
    assert osx.attn_device_status() == osx.ATTN_OK
    o_ref, l_ref = oracle.attention(q, k, v, causal=causal, scale=128 ** -0.5)
    compare(to_np(o), to_np(lse), o_ref, l_ref)


@pytest.mark.parametrize("overlap", [False, True])
def test_one_rank_ulysses_and_grid(nccl_one_rank, overlap):
    import online_softmax_exact_b200 as osx
    from online_softmax_exact_b200.grid2d_dist import grid2d_attention_dist
    from online_softmax_exact_b200.ulysses_dist import ulysses_attention_dist

    q = randn_bf16((2, 4, 700, 64), 27, 0)
    k = randn_bf16((2, 2, 700, 64), 27, 1)
    v = randn_bf16((2, 2, 700, 64), 27, 2)
    o_ref, l_ref = oracle.attention(q, k, v, causal=True, scale=64 ** -0.5)
    qg, kg, vg = q.cuda(), k.cuda(), v.cuda()
    o_u, l_u = ulysses_attention_dist(qg, kg, vg, causal=True)
    o_g, l_g = grid2d_attention_dist(qg, kg, vg, p_q=1, p_kv=1, causal=True, overlap=overlap)
    torch.cuda.synchronize()
    assert osx.attn_device_status() == osx.ATTN_OK
    compare(to_np(o_u), to_np(l_u), o_ref, l_ref)
    compare(to_np(o_g), to_np(l_g), o_ref, l_ref)

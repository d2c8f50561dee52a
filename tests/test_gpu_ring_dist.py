"""ring_attention_dist on a one-rank NCCL group (every box here has one GPU): the
default local compute runs through the library, and with one rank the ring is one
fold of the rank's own chunk, which must equal attn_fwd bit for bit. The multi-rank
schedule is checked on CPU ranks (test_ring_dist_host.py)."""

from __future__ import annotations

import pytest
import torch

from workloads import randn_bf16

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("causal", [False, True])
def test_one_rank_ring_equals_single_pass(causal):
    import torch.distributed as dist

    import online_softmax_exact_b200 as osx
    from online_softmax_exact_b200.ring_dist import ring_attention_dist

    dist.init_process_group("nccl", store=dist.HashStore(), rank=0, world_size=1)
    try:
        q = randn_bf16((1, 4, 1000, 128), 23, 0).cuda()
        k = randn_bf16((1, 2, 1000, 128), 23, 1).cuda()
        v = randn_bf16((1, 2, 1000, 128), 23, 2).cuda()
        o, lse = ring_attention_dist(q, k, v, causal=causal)
        o_ref, l_ref = osx.attn_fwd(q, k, v, causal=causal)
        torch.cuda.synchronize()
        assert osx.attn_device_status() == osx.ATTN_OK
        assert torch.equal(o, o_ref) and torch.equal(lse, l_ref)
    finally:
        dist.destroy_process_group()


def test_one_rank_ulysses_and_grid_equal_single_pass():
    """Ulysses' all-to-all exchanges and the 1 x 1 ATTENTION2D grid on one NCCL rank:
    the library's kernels behind them give attn_fwd's result bit for bit."""
    import torch.distributed as dist

    import online_softmax_exact_b200 as osx
    from online_softmax_exact_b200.grid2d_dist import grid2d_attention_dist
    from online_softmax_exact_b200.ulysses_dist import ulysses_attention_dist

    dist.init_process_group("nccl", store=dist.HashStore(), rank=0, world_size=1)
    try:
        q = randn_bf16((2, 4, 700, 64), 27, 0).cuda()
        k = randn_bf16((2, 2, 700, 64), 27, 1).cuda()
        v = randn_bf16((2, 2, 700, 64), 27, 2).cuda()
        o_ref, l_ref = osx.attn_fwd(q, k, v, causal=True)
        o_u, l_u = ulysses_attention_dist(q, k, v, causal=True)
        o_g, l_g = grid2d_attention_dist(q, k, v, p_q=1, p_kv=1, causal=True)
        torch.cuda.synchronize()
        assert osx.attn_device_status() == osx.ATTN_OK
        assert torch.equal(o_u, o_ref) and torch.equal(l_u, l_ref)
        assert torch.equal(o_g, o_ref) and torch.equal(l_g, l_ref)
    finally:
        dist.destroy_process_group()

"""ATTENTION2D across a grid of ranks: query chunks along one axis, key/value chunks
along the other.

ATTENTION2D (section 3) lays the attention of one head out as a P_q x P_kv grid of
(query chunk, key/value chunk) fragments: each processor computes its fragment with
fragment-local statistics, and the fragments of one query chunk are combined in
stages; section 2 shows the combination is commutative and associative, so no
approximation enters. Here rank r of a world of P_q * P_kv ranks holds query chunk
i = r // P_kv and key/value chunk j = r % P_kv, computes its normalised partial
(O_ij, LSE_ij) with ``attn_fwd_partial`` (global offsets, so the causal mask is the
whole sequence's), and the P_kv ranks of query chunk i gather each other's partials
and combine them with ``attn_merge``.
"""

from __future__ import annotations

import torch
import torch.distributed as dist

from . import attn_fwd_partial, attn_merge


def grid_coords(rank: int, p_q: int, p_kv: int) -> tuple[int, int]:
    """(query chunk, key/value chunk) of ``rank`` in a p_q x p_kv grid (row-major)."""
    if not 0 <= rank < p_q * p_kv:
        raise ValueError("rank outside the grid")
    return rank // p_kv, rank % p_kv


def row_groups(p_q: int, p_kv: int) -> list[list[int]]:
    """The ranks that share each query chunk (one list per query chunk)."""
    return [[i * p_kv + j for j in range(p_kv)] for i in range(p_q)]


def _default_partial(q, k, v, *, q_off, kv_off, causal, scale):
    C = q.shape[2]
    return attn_fwd_partial(q, k, v, q_start=0, q_len=C, kv_start=0, kv_len=k.shape[2],
                            causal=causal, scale=scale, q_off=q_off, kv_off=kv_off)


def _default_merge(o_parts, lse_parts):
    return attn_merge(o_parts, lse_parts)


def grid2d_attention_dist(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, p_q: int,
                          p_kv: int, causal: bool, scale: float | None = None,
                          row_group=None, merge_order=None, partial=None, merge=None):
    """This rank's fragment of the grid, then the combination along its row.

    q: [B, Hq, Cq, d], query chunk i of the sequence (rows i*Cq ..); k, v:
    [B, Hkv, Ckv, d], key/value chunk j (rows j*Ckv ..), with (i, j) =
    ``grid_coords(rank)``. ``row_group``: the process group of ``row_groups(p_q,
    p_kv)[i]`` (every rank must create all row groups, in the same order, as
    torch.distributed requires); None when p_kv == 1. ``merge_order``: the order of
    the key/value chunks in the combination (default 0..p_kv-1; any order gives the
    same result up to fp32 rounding). Returns (O [B, Hq, Cq, d], LSE [B, Hq, Cq]) of
    query chunk i, the same on every rank of the row.

    ``partial(q, k, v, *, q_off, kv_off, causal, scale) -> (O, LSE)`` and
    ``merge(o_parts, lse_parts) -> (O, LSE)`` replace the local compute.
    """
    rank = dist.get_rank()
    if dist.get_world_size() != p_q * p_kv:
        raise ValueError("the world must be the p_q x p_kv grid")
    i, j = grid_coords(rank, p_q, p_kv)
    B, Hq, Cq, d = q.shape
    Ckv = k.shape[2]
    if scale is None:
        scale = d ** -0.5
    partial = partial or _default_partial
    merge = merge or _default_merge
    order = list(range(p_kv)) if merge_order is None else list(merge_order)
    if sorted(order) != list(range(p_kv)):
        raise ValueError("merge_order must be a permutation of the key/value chunks")
    o, lse = partial(q, k, v, q_off=i * Cq, kv_off=j * Ckv, causal=causal, scale=scale)
    if p_kv == 1:
        return o, lse
    o_all = [torch.empty_like(o) for _ in range(p_kv)]
    l_all = [torch.empty_like(lse) for _ in range(p_kv)]
    dist.all_gather(o_all, o.contiguous(), group=row_group)
    dist.all_gather(l_all, lse.contiguous(), group=row_group)
    return merge([o_all[x] for x in order], [l_all[x] for x in order])

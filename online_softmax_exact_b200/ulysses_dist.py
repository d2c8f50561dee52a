"""Ulysses-style sequence parallelism: an all-to-all turns sequence shards into head
shards, each rank runs exact attention over the whole sequence for its heads, and a
second all-to-all turns the result back into sequence shards.

The Ulysses page describes partitioning the sequence across devices and, around the
attention, two all-to-all exchanges that give each device all positions of a subset
of heads, so that the attention itself is unchanged; the single-pass ``attn_fwd``
is that unchanged attention here.
"""

from __future__ import annotations

import torch
import torch.distributed as dist

from . import ATTN_OK, AttnError, attn_device_status, attn_fwd


def _default_attend(q, k, v, *, causal, scale):
    return attn_fwd(q, k, v, causal=causal, scale=scale)


def _seq_to_heads(x: torch.Tensor, world: int, group) -> torch.Tensor:
    """[B, H, C, d] (this rank's sequence chunk, all heads) -> [B, H/P, P*C, d] (all
    chunks, this rank's head group)."""
    B, H, C, d = x.shape
    h = H // world
    send = x.reshape(B, world, h, C, d).permute(1, 0, 2, 3, 4).contiguous()  # [P, B, h, C, d]
    recv = torch.empty_like(send)                                          # [P(src), B, h, C, d]
    dist.all_to_all_single(recv, send, group=group)
    return recv.permute(1, 2, 0, 3, 4).reshape(B, h, world * C, d).contiguous()


def _heads_to_seq(x: torch.Tensor, world: int, group) -> torch.Tensor:
    """[B, h, P*C, ...] (this rank's head group, all chunks) -> [B, P*h, C, ...] (all
    heads, this rank's chunk)."""
    B, h, N = x.shape[:3]
    rest = tuple(x.shape[3:])
    C = N // world
    send = x.reshape((B, h, world, C) + rest).transpose(0, 2).transpose(1, 2).contiguous()
    # send: [P(dst chunk), B, h, C, ...]
    recv = torch.empty_like(send)  # [P(src head group), B, h, C, ...]
    dist.all_to_all_single(recv, send, group=group)
    return recv.transpose(0, 1).reshape((B, world * h, C) + rest).contiguous()


def ulysses_attention_dist(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *,
                           causal: bool, scale: float | None = None, group=None,
                           attend=None, check_status: bool = True):
    """q: [B, Hq, C, d]; k, v: [B, Hkv, C, d] - chunk ``rank`` of the sequence on every
    rank of ``group`` (P ranks; Hq and Hkv divisible by P, and Hq/Hkv groups stay
    whole since head g of q reads head g // (Hq/Hkv) of k). Returns this rank's chunk
    of (O [B, Hq, C, d], LSE [B, Hq, C]) in fp32.

    ``attend(q, k, v, *, causal, scale) -> (O, LSE)`` replaces the local attention
    (default: the library's single pass; with ``check_status`` its device status is
    checked after it, raising ``AttnError`` on a device-side time-out).
    """
    world = dist.get_world_size(group)
    B, Hq, C, d = q.shape
    Hkv = k.shape[1]
    if Hq % world or Hkv % world:
        raise ValueError("the head counts must divide among the ranks")
    if scale is None:
        scale = d ** -0.5
    library = attend is None
    attend = attend or _default_attend
    qh = _seq_to_heads(q, world, group)
    kh = _seq_to_heads(k, world, group)
    vh = _seq_to_heads(v, world, group)
    o, lse = attend(qh, kh, vh, causal=causal, scale=scale)
    if library and check_status:
        st = attn_device_status()
        if st != ATTN_OK:
            raise AttnError(st, "ulysses_attention_dist")
    return _heads_to_seq(o, world, group), _heads_to_seq(lse, world, group)

"""Ring Attention across the ranks of a process group, one sequence chunk per rank.

"Ring Attention with Blockwise Parallel Transformers", section 3: each host keeps its
query block and passes its key/value block to the next host around a ring; at ring
step s the host of query block i holds key/value block (i - s) mod P and folds it
into its running result, while the next block is already on its way, so that the
transfer hides behind the blockwise compute when it is not longer than it.

Here a rank folds a block into its running (O, LSE) with ``attn_fwd_partial`` (first
block) and ``attn_fwd_partial_acc`` (later blocks) - the associative update of the
online softmax - and exchanges blocks with ``torch.distributed`` point-to-point
operations (NCCL between GPUs). The accumulation order is the ring order, the same
as :func:`schedules.ring_attention` with ``fused_merge=True`` on one GPU, so a rank's
result is the one that schedule gives for its chunk.
"""

from __future__ import annotations

import torch
import torch.distributed as dist

from . import attn_fwd_partial, attn_fwd_partial_acc


def ring_steps(rank: int, world: int, causal: bool) -> list[tuple[int, int, bool]]:
    """(step, key/value chunk held, whether it is folded) for every ring step of
    ``rank``: at step s the rank holds chunk (rank - s) mod world; under the causal
    mask a chunk after the rank's own is held and passed on but not folded."""
    out = []
    for s in range(world):
        kv = (rank - s) % world
        out.append((s, kv, not (causal and kv > rank)))
    return out


def _default_fold(o, lse, q, k, v, *, q_off, kv_off, causal, scale, first):
    fn = attn_fwd_partial if first else attn_fwd_partial_acc
    C = q.shape[2]
    fn(q, k, v, q_start=0, q_len=C, kv_start=0, kv_len=k.shape[2], causal=causal,
       scale=scale, q_off=q_off, kv_off=kv_off, o=o, lse=lse)


def ring_attention_dist(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, causal: bool,
                        scale: float | None = None, group=None, out=None, fold=None):
    """This rank's query chunk attends every rank's key/value chunk, in ring order.

    q: [B, Hq, C, d]; k, v: [B, Hkv, C, d] - chunk ``rank`` of the sequence (global
    rows rank*C .. rank*C + C - 1), bf16 on this rank's GPU. Returns (O [B, Hq, C, d],
    LSE [B, Hq, C]) in fp32 (or in ``out``). Every rank of ``group`` must call this
    with chunks of one shape; each step sends the held K/V chunk to rank + 1 and
    receives the next from rank - 1 while the held chunk is folded in.

    ``fold(o, lse, q, k, v, *, q_off, kv_off, causal, scale, first)`` replaces the
    local compute (default: the library's partial attention on the current stream).
    """
    rank = dist.get_rank(group)
    world = dist.get_world_size(group)
    B, Hq, C, d = q.shape
    if k.shape != v.shape or k.shape[0] != B or k.shape[2] != C or k.shape[3] != d:
        raise ValueError("k and v must be [B, Hkv, C, d] matching q's chunk")
    if scale is None:
        scale = d ** -0.5
    fold = fold or _default_fold
    if out is None:
        o = torch.empty((B, Hq, C, d), dtype=torch.float32, device=q.device)
        lse = torch.empty((B, Hq, C), dtype=torch.float32, device=q.device)
    else:
        o, lse = out
    # K and V travel together as one message; two buffers alternate between the
    # block being folded (and sent on) and the block being received
    cur = torch.empty((2,) + tuple(k.shape), dtype=k.dtype, device=k.device)
    nxt = torch.empty_like(cur)
    cur[0].copy_(k)
    cur[1].copy_(v)
    nxt_rank = dist.get_global_rank(group, (rank + 1) % world) if group is not None \
        else (rank + 1) % world
    prv_rank = dist.get_global_rank(group, (rank - 1) % world) if group is not None \
        else (rank - 1) % world
    first = True
    for s, kv, visible in ring_steps(rank, world, causal):
        works = []
        if s < world - 1:
            ops = [dist.P2POp(dist.isend, cur.view(torch.uint8), nxt_rank, group),
                   dist.P2POp(dist.irecv, nxt.view(torch.uint8), prv_rank, group)]
            works = dist.batch_isend_irecv(ops)
        if visible:
            fold(o, lse, q, cur[0], cur[1], q_off=rank * C, kv_off=kv * C, causal=causal,
                 scale=scale, first=first)
            first = False
        for w in works:
            w.wait()
        cur, nxt = nxt, cur
    return o, lse

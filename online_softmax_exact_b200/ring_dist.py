"""Ring Attention across the ranks of a process group, one sequence chunk per rank.

"Ring Attention with Blockwise Parallel Transformers", section 3: each host keeps its
query block and passes its key/value block to the next host around a ring; at ring
step s the host of query block i holds key/value block (i - s) mod P and folds it
into its running result, while the next block is already on its way, so that the
transfer hides behind the blockwise compute when it is not longer than it.

Here a rank folds a block into its running (O, LSE) with ``attn_fwd_partial`` (first
block) and ``attn_fwd_partial_acc`` (later blocks) - the associative update of the
online softmax - and exchanges blocks with ``torch.distributed`` point-to-point
operations (NCCL between GPUs).

Two layouts of the sequence over the ranks:

* ``"contiguous"``: rank r holds rows [r*C, (r+1)*C). The accumulation order is the
  ring order, the same as :func:`schedules.ring_attention` with ``fused_merge=True`` on
  one GPU. Under the causal mask rank r folds only blocks 0..r, so at step s the
  ranks r < s idle while the others fold a whole block: the ring takes P block-times
  for (P + 1) / 2 blocks of work per rank on average.
* ``"zigzag"``: the sequence is cut into 2P half-chunks and rank r holds half-chunks
  r and 2P-1-r (the section asks for the data to be spread evenly around the ring; this
  spreads the causal work evenly too). At every ring step each rank folds the same
  amount of visible work, two half-by-half blocks, so no rank waits for another.
  :func:`zigzag_rows` gives a rank's global rows; :func:`zigzag_shard` cuts a whole
  sequence into a rank's local tensor.
"""

from __future__ import annotations

import torch
import torch.distributed as dist

from . import ATTN_OK, AttnError, attn_device_status, attn_fwd_partial, attn_fwd_partial_acc


def ring_steps(rank: int, world: int, causal: bool) -> list[tuple[int, int, bool]]:
    """(step, key/value chunk held, whether it is folded) for every ring step of
    ``rank`` in the contiguous layout: at step s the rank holds chunk (rank - s) mod
    world; under the causal mask a chunk after the rank's own is held and passed on
    but not folded."""
    out = []
    for s in range(world):
        kv = (rank - s) % world
        out.append((s, kv, not (causal and kv > rank)))
    return out


def zigzag_halves(rank: int, world: int) -> tuple[int, int]:
    """The two half-chunk indices (of 2 * world) that ``rank`` holds in the zigzag
    layout, in local order."""
    return rank, 2 * world - 1 - rank


def zigzag_rows(rank: int, world: int, C: int) -> list[range]:
    """Global rows of ``rank``'s local chunk (C rows, C even) in the zigzag layout."""
    h = C // 2
    return [range(x * h, (x + 1) * h) for x in zigzag_halves(rank, world)]


def zigzag_shard(x: torch.Tensor, rank: int, world: int, dim: int = 2) -> torch.Tensor:
    """A rank's local tensor in the zigzag layout: its two half-chunks of the whole
    sequence ``x`` (split along ``dim`` into 2 * world equal pieces), concatenated."""
    pieces = torch.chunk(x, 2 * world, dim=dim)
    a, b = zigzag_halves(rank, world)
    return torch.cat([pieces[a], pieces[b]], dim=dim).contiguous()


def zigzag_steps(rank: int, world: int, causal: bool) -> list[tuple[int, int, list]]:
    """(step, rank whose block is held, [(local query half, held half, query half index,
    key/value half index)] folded at that step) in the zigzag layout. Under the causal
    mask a key/value half is folded into a query half when its index is not larger
    (the half on the diagonal is cut by the mask inside the fold)."""
    out = []
    mine = zigzag_halves(rank, world)
    for s in range(world):
        src = (rank - s) % world
        held = zigzag_halves(src, world)
        folds = []
        for a, qa in enumerate(mine):
            for b, kb in enumerate(held):
                if causal and kb > qa:
                    continue
                folds.append((a, b, qa, kb))
        out.append((s, src, folds))
    return out


def _default_fold(o, lse, q, k, v, *, q_off, kv_off, causal, scale, first):
    fn = attn_fwd_partial if first else attn_fwd_partial_acc
    C = q.shape[2]
    fn(q, k, v, q_start=0, q_len=C, kv_start=0, kv_len=k.shape[2], causal=causal,
       scale=scale, q_off=q_off, kv_off=kv_off, o=o, lse=lse)


def _peers(group, rank, world):
    nxt = (rank + 1) % world
    prv = (rank - 1) % world
    if group is not None:
        return dist.get_global_rank(group, nxt), dist.get_global_rank(group, prv)
    return nxt, prv


def ring_attention_dist(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, causal: bool,
                        scale: float | None = None, group=None, out=None, fold=None,
                        layout: str = "contiguous", check_status: bool = True):
    """This rank's query chunk attends every rank's key/value chunk, in ring order.

    q: [B, Hq, C, d]; k, v: [B, Hkv, C, d] - this rank's chunk of the sequence (global
    rows rank*C .. rank*C + C - 1 in the contiguous layout; :func:`zigzag_rows` in the
    zigzag layout, where C must be even), bf16 on this rank's device. Returns
    (O [B, Hq, C, d], LSE [B, Hq, C]) in fp32 (or in ``out``). Every rank of ``group``
    must call this with chunks of one shape; each step sends the held K/V block to
    rank + 1 and receives the next from rank - 1 while the held block is folded in.

    ``fold(o, lse, q, k, v, *, q_off, kv_off, causal, scale, first)`` replaces the
    local compute (default: the library's partial attention on the current stream):
    it folds keys k/v (global positions from kv_off) into the accumulator (o, lse) of
    queries q (positions from q_off); ``first`` says that the accumulator holds
    nothing yet. With the default fold and ``check_status``, the call ends by
    synchronising the current stream and raising ``AttnError`` if a kernel recorded a
    device-side time-out (its results would be unspecified).
    """
    if layout not in ("contiguous", "zigzag"):
        raise ValueError("layout must be 'contiguous' or 'zigzag'")
    rank = dist.get_rank(group)
    world = dist.get_world_size(group)
    B, Hq, C, d = q.shape
    if k.shape != v.shape or k.shape[0] != B or k.shape[2] != C or k.shape[3] != d:
        raise ValueError("k and v must be [B, Hkv, C, d] matching q's chunk")
    if layout == "zigzag" and C % 2:
        raise ValueError("the zigzag layout needs an even chunk length")
    if scale is None:
        scale = d ** -0.5
    library_fold = fold is None
    fold = fold or _default_fold
    if out is None:
        o = torch.empty((B, Hq, C, d), dtype=torch.float32, device=q.device)
        lse = torch.empty((B, Hq, C), dtype=torch.float32, device=q.device)
    else:
        o, lse = out
    nxt_rank, prv_rank = _peers(group, rank, world)
    if layout == "contiguous":
        _ring_contiguous(q, k, v, o, lse, rank, world, causal, scale, fold, nxt_rank,
                         prv_rank, group)
    else:
        _ring_zigzag(q, k, v, o, lse, rank, world, causal, scale, fold, nxt_rank,
                     prv_rank, group)
    if library_fold and check_status:
        _raise_on_device_failure("ring_attention_dist")
    return o, lse


def _raise_on_device_failure(where: str) -> None:
    st = attn_device_status()
    if st != ATTN_OK:
        raise AttnError(st, where)


def _exchange(cur, nxt, nxt_rank, prv_rank, group):
    ops = [dist.P2POp(dist.isend, cur.view(torch.uint8), nxt_rank, group),
           dist.P2POp(dist.irecv, nxt.view(torch.uint8), prv_rank, group)]
    return dist.batch_isend_irecv(ops)


def _ring_contiguous(q, k, v, o, lse, rank, world, causal, scale, fold, nxt_rank, prv_rank,
                     group):
    C = q.shape[2]
    # K and V travel together as one message; two buffers alternate between the
    # block being folded (and sent on) and the block being received
    cur = torch.empty((2,) + tuple(k.shape), dtype=k.dtype, device=k.device)
    nxt = torch.empty_like(cur)
    cur[0].copy_(k)
    cur[1].copy_(v)
    first = True
    for s, kv, visible in ring_steps(rank, world, causal):
        works = _exchange(cur, nxt, nxt_rank, prv_rank, group) if s < world - 1 else []
        if visible:
            fold(o, lse, q, cur[0], cur[1], q_off=rank * C, kv_off=kv * C, causal=causal,
                 scale=scale, first=first)
            first = False
        for w in works:
            w.wait()
        cur, nxt = nxt, cur


def _ring_zigzag(q, k, v, o, lse, rank, world, causal, scale, fold, nxt_rank, prv_rank,
                 group):
    B, Hq, C, d = q.shape
    h = C // 2
    # local halves as contiguous tensors: queries, and accumulators per query half
    q_half = [q[:, :, :h].contiguous(), q[:, :, h:].contiguous()]
    o_half = [torch.empty((B, Hq, h, d), dtype=o.dtype, device=o.device) for _ in range(2)]
    l_half = [torch.empty((B, Hq, h), dtype=lse.dtype, device=lse.device) for _ in range(2)]
    first = [True, True]
    # the travelling block: [K/V][half][B, Hkv, h, d], each half contiguous
    cur = torch.empty((2, 2) + (k.shape[0], k.shape[1], h, d), dtype=k.dtype, device=k.device)
    nxt = torch.empty_like(cur)
    for t, src in ((0, k), (1, v)):
        cur[t, 0].copy_(src[:, :, :h])
        cur[t, 1].copy_(src[:, :, h:])
    for s, _src, folds in zigzag_steps(rank, world, causal):
        works = _exchange(cur, nxt, nxt_rank, prv_rank, group) if s < world - 1 else []
        for a, b, qa, kb in folds:
            fold(o_half[a], l_half[a], q_half[a], cur[0, b], cur[1, b], q_off=qa * h,
                 kv_off=kb * h, causal=causal, scale=scale, first=first[a])
            first[a] = False
        for w in works:
            w.wait()
        cur, nxt = nxt, cur
    o[:, :, :h].copy_(o_half[0])
    o[:, :, h:].copy_(o_half[1])
    lse[:, :, :h].copy_(l_half[0])
    lse[:, :, h:].copy_(l_half[1])

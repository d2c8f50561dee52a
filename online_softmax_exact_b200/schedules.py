"""Chunk schedules of the sequence-parallel methods, emulated on one GPU over the C ABI.

Both schedules split the sequence into chunks, run ``attn_fwd_partial`` on (query
chunk, key/value chunk) pairs and combine each query chunk's partials with
``attn_merge``. Outputs are chunk-major: O ``[P, B, Hq, C, d]`` and LSE
``[P, B, Hq, C]`` for P chunks of C rows, i.e. the layout in which chunk i's result
lives on device i of the distributed method; ``chunks_to_sequence`` gives the
``[B, Hq, N, d]`` view when wanted.
"""

from __future__ import annotations

from dataclasses import dataclass

import torch

from . import attn_fwd_partial, attn_fwd_partial_acc, attn_fwd_partial_batch, attn_merge


def chunk_bounds(N: int, n_chunks: int) -> list[tuple[int, int]]:
    if n_chunks < 1 or N % n_chunks:
        raise ValueError("the sequence length must split into equal chunks")
    c = N // n_chunks
    return [(i * c, (i + 1) * c) for i in range(n_chunks)]


def ring_order(n_chunks: int, causal: bool) -> list[list[int]]:
    """Key/value chunks each query chunk visits, in ring order: at step s, query chunk
    i holds key/value chunk (i - s) mod P ("Ring Attention with Blockwise Parallel
    Transformers", section 3: blocks pass around the ring, one hop per step). Under the
    causal mask a key/value chunk entirely after the query chunk is hidden and skipped.
    """
    out = []
    for qi in range(n_chunks):
        visit = []
        for s in range(n_chunks):
            kv = (qi - s) % n_chunks
            if causal and kv > qi:
                continue
            visit.append(kv)
        out.append(visit)
    return out


@dataclass
class Workspace:
    """Partial-result buffers reused across calls (one per (query chunk, step))."""

    o: torch.Tensor    # [S, B, Hq, C, d]
    lse: torch.Tensor  # [S, B, Hq, C]

    @staticmethod
    def for_shape(slots: int, B: int, Hq: int, C: int, d: int, device) -> "Workspace":
        return Workspace(torch.empty((slots, B, Hq, C, d), dtype=torch.float32, device=device),
                         torch.empty((slots, B, Hq, C), dtype=torch.float32, device=device))


def _alloc_out(q, n_chunks, out):
    B, Hq, N, d = q.shape
    C = N // n_chunks
    if out is None:
        return (torch.empty((n_chunks, B, Hq, C, d), dtype=torch.float32, device=q.device),
                torch.empty((n_chunks, B, Hq, C), dtype=torch.float32, device=q.device))
    return out


class _NoTimer:
    def __call__(self, kind: str, stream=None):
        return self

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        return False


_NO_TIMER = _NoTimer()


def balance_streams(costs: list[float], n_streams: int) -> list[int]:
    """Assign query chunks to streams, heaviest first onto the least-loaded stream."""
    load = [0.0] * n_streams
    assign = [0] * len(costs)
    for i in sorted(range(len(costs)), key=lambda i: -costs[i]):
        s = min(range(n_streams), key=lambda j: load[j])
        assign[i] = s
        load[s] += costs[i]
    return assign


class _Streams:
    """Fork work from ``main`` onto side streams and join it back."""

    def __init__(self, main, n: int, device):
        self.main = main
        self.side = [main] if n <= 1 else [torch.cuda.Stream(device) for _ in range(n)]
        if n > 1:
            ev = torch.cuda.Event()
            ev.record(main)
            for s in self.side:
                s.wait_event(ev)

    def join(self, tensors):
        if len(self.side) == 1:
            return
        for s in self.side:
            ev = torch.cuda.Event()
            ev.record(s)
            self.main.wait_event(ev)
            for t in tensors:
                t.record_stream(s)


def _ring_batched(q, k, v, order, bounds, causal, scale, o_out, l_out, workspace, main,
                  timer, fused_merge):
    """The ring schedule with batched launches: without the fused merge, every partial
    of every query chunk in one launch, then one merge per query chunk; with it, one
    launch per ring step s holding the step-s pair of every query chunk (so each
    accumulator is updated once per launch, in ring order)."""
    P = len(order)
    if fused_merge:
        for s_step in range(max(len(x) for x in order)):
            pairs = []
            for qi, visit in enumerate(order):
                if s_step < len(visit):
                    qs, qe = bounds[qi]
                    ks, ke = bounds[visit[s_step]]
                    pairs.append(dict(q_start=qs, q_len=qe - qs, kv_start=ks, kv_len=ke - ks,
                                      o=o_out[qi], lse=l_out[qi]))
            with timer("partial", main):
                attn_fwd_partial_batch(q, k, v, pairs, causal=causal, scale=scale,
                                       accumulate=s_step > 0, stream=main)
        return
    pairs, slots, slot = [], {}, 0
    for qi, visit in enumerate(order):
        qs, qe = bounds[qi]
        for kv in visit:
            ks, ke = bounds[kv]
            if len(visit) == 1:
                o, lse = o_out[qi], l_out[qi]
            else:
                o, lse = workspace.o[slot], workspace.lse[slot]
                slots.setdefault(qi, []).append(slot)
                slot += 1
            pairs.append(dict(q_start=qs, q_len=qe - qs, kv_start=ks, kv_len=ke - ks,
                              o=o, lse=lse))
    with timer("partial", main):
        attn_fwd_partial_batch(q, k, v, pairs, causal=causal, scale=scale, stream=main)
    for qi in range(P):
        if qi in slots:
            idx = slots[qi]
            with timer("merge", main):
                attn_merge([workspace.o[i] for i in idx], [workspace.lse[i] for i in idx],
                           o=o_out[qi], lse=l_out[qi], stream=main)


def ring_slots(n_chunks: int, causal: bool, batched: bool, n_streams: int = 1) -> int:
    """Workspace slots (partial buffers) :func:`ring_attention` needs."""
    order = ring_order(n_chunks, causal)
    if batched:
        return sum(len(x) for x in order if len(x) > 1)
    return max(len(x) for x in order) * max(1, min(n_streams, n_chunks))


def ring_attention(q, k, v, *, n_chunks: int, causal: bool, scale: float | None = None,
                   out=None, workspace: Workspace | None = None, stream=None, timer=None,
                   n_streams: int = 1, fused_merge: bool = False, batched: bool = False):
    """Ring Attention's schedule on one GPU: query chunk i attends the key/value chunks
    of :func:`ring_order` one ring step at a time, then merges its partials.

    With ``n_streams`` > 1 the query chunks are spread over that many CUDA streams
    (balanced by their number of partials), so that one launch's tail overlaps the next
    launch; each chunk's partials and merge stay in order on its stream, and the result
    is joined back into ``stream``. ``timer(kind)``, if given, is entered around every
    launch ("partial" or "merge") with the launching stream as argument.
    With ``fused_merge`` each query chunk keeps one running (O, LSE) accumulator in the
    output: the first visited chunk writes it, every later ring step folds its partial
    into it (``attn_fwd_partial_acc``), as a ring device does; no partial buffers and
    no merge launches. With ``batched`` the chunk pairs go through
    ``attn_fwd_partial_batch`` instead, many pairs per launch (see :func:`_ring_batched`).
    Returns chunk-major (O [P,B,Hq,C,d], LSE [P,B,Hq,C]).
    """
    timer = timer or _NO_TIMER
    B, Hq, N, d = q.shape
    bounds = chunk_bounds(N, n_chunks)
    C = N // n_chunks
    order = ring_order(n_chunks, causal)
    o_out, l_out = _alloc_out(q, n_chunks, out)
    if batched:
        need = ring_slots(n_chunks, causal, True)
        if not fused_merge and (workspace is None or workspace.o.shape[0] < need
                                or workspace.o.shape[1:] != (B, Hq, C, d)):
            workspace = Workspace.for_shape(need, B, Hq, C, d, q.device)
        main = stream if stream is not None else torch.cuda.current_stream(q.device)
        _ring_batched(q, k, v, order, bounds, causal, scale, o_out, l_out, workspace, main,
                      timer, fused_merge)
        return o_out, l_out
    slots = max(len(x) for x in order)
    n_streams = max(1, min(n_streams, n_chunks))
    need = slots * n_streams
    if not fused_merge and (workspace is None or workspace.o.shape[0] < need
                            or workspace.o.shape[1:] != (B, Hq, C, d)):
        workspace = Workspace.for_shape(need, B, Hq, C, d, q.device)
    main = stream if stream is not None else torch.cuda.current_stream(q.device)
    st = _Streams(main, n_streams, q.device)
    assign = balance_streams([float(len(x)) for x in order], n_streams)
    for qi in sorted(range(n_chunks), key=lambda i: -len(order[i])):
        visit = order[qi]
        s_idx = assign[qi]
        s = st.side[s_idx]
        base = s_idx * slots
        qs, qe = bounds[qi]
        if fused_merge:
            for j, kv in enumerate(visit):
                ks, ke = bounds[kv]
                fn = attn_fwd_partial if j == 0 else attn_fwd_partial_acc
                with timer("partial", s):
                    fn(q, k, v, q_start=qs, q_len=qe - qs, kv_start=ks, kv_len=ke - ks,
                       causal=causal, scale=scale, o=o_out[qi], lse=l_out[qi], stream=s)
            continue
        if len(visit) == 1:
            # one part: the merge is the identity, so write the result in place
            ks, ke = bounds[visit[0]]
            with timer("partial", s):
                attn_fwd_partial(q, k, v, q_start=qs, q_len=qe - qs, kv_start=ks,
                                 kv_len=ke - ks, causal=causal, scale=scale, o=o_out[qi],
                                 lse=l_out[qi], stream=s)
            continue
        for j, kv in enumerate(visit):
            ks, ke = bounds[kv]
            with timer("partial", s):
                attn_fwd_partial(q, k, v, q_start=qs, q_len=qe - qs, kv_start=ks,
                                 kv_len=ke - ks, causal=causal, scale=scale,
                                 o=workspace.o[base + j], lse=workspace.lse[base + j], stream=s)
        n = len(visit)
        with timer("merge", s):
            attn_merge([workspace.o[base + i] for i in range(n)],
                       [workspace.lse[base + i] for i in range(n)],
                       o=o_out[qi], lse=l_out[qi], stream=s)
    st.join([q, k, v, o_out, l_out] + ([] if fused_merge else [workspace.o, workspace.lse]))
    return o_out, l_out


def _grid_batched(q, k, v, bounds, merge_orders, causal, scale, o_out, l_out, workspace,
                  main, timer, fused_merge):
    """The grid with batched launches: without the fused merge, every cell in one
    launch, then one merge per query chunk in its order; with it, one launch per merge
    step s holding cell (i, merge_orders[i][s]) of every query chunk i."""
    P = len(bounds)
    if fused_merge:
        for s_step in range(P):
            pairs = []
            for qi in range(P):
                qs, qe = bounds[qi]
                ks, ke = bounds[merge_orders[qi][s_step]]
                pairs.append(dict(q_start=qs, q_len=qe - qs, kv_start=ks, kv_len=ke - ks,
                                  o=o_out[qi], lse=l_out[qi]))
            with timer("partial", main):
                attn_fwd_partial_batch(q, k, v, pairs, causal=causal, scale=scale,
                                       accumulate=s_step > 0, stream=main)
        return
    pairs = []
    for qi in range(P):
        qs, qe = bounds[qi]
        for kv in range(P):
            ks, ke = bounds[kv]
            pairs.append(dict(q_start=qs, q_len=qe - qs, kv_start=ks, kv_len=ke - ks,
                              o=workspace.o[qi * P + kv], lse=workspace.lse[qi * P + kv]))
    with timer("partial", main):
        attn_fwd_partial_batch(q, k, v, pairs, causal=causal, scale=scale, stream=main)
    for qi in range(P):
        order = merge_orders[qi]
        with timer("merge", main):
            attn_merge([workspace.o[qi * P + x] for x in order],
                       [workspace.lse[qi * P + x] for x in order],
                       o=o_out[qi], lse=l_out[qi], stream=main)


def grid2d_attention(q, k, v, *, n_chunks: int, merge_orders: list[list[int]], causal: bool,
                     scale: float | None = None, out=None, workspace: Workspace | None = None,
                     stream=None, timer=None, n_streams: int = 1, fused_merge: bool = False,
                     batched: bool = False):
    """ATTENTION2D's query x key/value grid on one GPU: every (query chunk, key/value
    chunk) cell is a partial attention (fragment-local statistics, section 3); each
    query chunk's partials are merged in the order ``merge_orders[i]`` (any order gives
    the same result, section 2). With ``fused_merge`` the cells of a query chunk are
    folded into one running accumulator in that order instead. With ``batched`` the
    cells go through ``attn_fwd_partial_batch`` (all n_chunks^2 cells in one launch, at
    most 48; with ``fused_merge``, one launch per merge step). Returns chunk-major
    (O, LSE).
    """
    timer = timer or _NO_TIMER
    B, Hq, N, d = q.shape
    bounds = chunk_bounds(N, n_chunks)
    C = N // n_chunks
    o_out, l_out = _alloc_out(q, n_chunks, out)
    for qi in range(n_chunks):
        if sorted(merge_orders[qi]) != list(range(n_chunks)):
            raise ValueError("each merge order must be a permutation of the chunk indices")
    if batched:
        if n_chunks * n_chunks > 48 and not fused_merge:
            raise ValueError("a batched grid holds at most 48 cells per launch")
        need = n_chunks * n_chunks
        if not fused_merge and (workspace is None or workspace.o.shape[0] < need
                                or workspace.o.shape[1:] != (B, Hq, C, d)):
            workspace = Workspace.for_shape(need, B, Hq, C, d, q.device)
        main = stream if stream is not None else torch.cuda.current_stream(q.device)
        _grid_batched(q, k, v, bounds, merge_orders, causal, scale, o_out, l_out, workspace,
                      main, timer, fused_merge)
        return o_out, l_out
    n_streams = max(1, min(n_streams, n_chunks))
    need = n_chunks * n_streams
    if not fused_merge and (workspace is None or workspace.o.shape[0] < need
                            or workspace.o.shape[1:] != (B, Hq, C, d)):
        workspace = Workspace.for_shape(need, B, Hq, C, d, q.device)
    main = stream if stream is not None else torch.cuda.current_stream(q.device)
    st = _Streams(main, n_streams, q.device)
    for qi in range(n_chunks):
        s = st.side[qi % n_streams]
        base = (qi % n_streams) * n_chunks
        qs, qe = bounds[qi]
        order = merge_orders[qi]
        if sorted(order) != list(range(n_chunks)):
            raise ValueError("each merge order must be a permutation of the chunk indices")
        if fused_merge:
            for j, kv in enumerate(order):
                ks, ke = bounds[kv]
                fn = attn_fwd_partial if j == 0 else attn_fwd_partial_acc
                with timer("partial", s):
                    fn(q, k, v, q_start=qs, q_len=qe - qs, kv_start=ks, kv_len=ke - ks,
                       causal=causal, scale=scale, o=o_out[qi], lse=l_out[qi], stream=s)
            continue
        for kv in range(n_chunks):
            ks, ke = bounds[kv]
            with timer("partial", s):
                attn_fwd_partial(q, k, v, q_start=qs, q_len=qe - qs, kv_start=ks,
                                 kv_len=ke - ks, causal=causal, scale=scale,
                                 o=workspace.o[base + kv], lse=workspace.lse[base + kv],
                                 stream=s)
        with timer("merge", s):
            attn_merge([workspace.o[base + i] for i in order],
                       [workspace.lse[base + i] for i in order],
                       o=o_out[qi], lse=l_out[qi], stream=s)
    st.join([q, k, v, o_out, l_out] + ([] if fused_merge else [workspace.o, workspace.lse]))
    return o_out, l_out


def chunks_to_sequence(o_chunks: torch.Tensor, lse_chunks: torch.Tensor):
    """[P,B,Hq,C,d] / [P,B,Hq,C] -> [B,Hq,P*C,d] / [B,Hq,P*C] (a copy)."""
    P, B, Hq, C, d = o_chunks.shape
    o = o_chunks.permute(1, 2, 0, 3, 4).reshape(B, Hq, P * C, d)
    lse = lse_chunks.permute(1, 2, 0, 3).reshape(B, Hq, P * C)
    return o, lse

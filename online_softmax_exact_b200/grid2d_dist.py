"""ATTENTION2D across a grid of ranks: query chunks along one axis, key/value chunks
along the other.

ATTENTION2D (section 3) lays the attention of one head out as a P_q x P_kv grid of
(query chunk, key/value chunk) fragments: each processor computes its fragment with
fragment-local statistics, and the fragments of one query chunk are combined in
stages; section 2 shows the combination is commutative and associative, so no
approximation enters. Here rank r of a world of P_q * P_kv ranks holds query chunk
i = r // P_kv and key/value chunk j = r % P_kv and computes its normalised partial
(O_ij, LSE_ij) with ``attn_fwd_partial`` (global offsets, so the causal mask is the
whole sequence's).

The fragments of query chunk i are then reduce-scattered over the chunk's rows: the
chunk's Cq rows are cut into P_kv slices, the rank at column m of the row receives
slice m of every fragment (one all-to-all within the row) and combines them with
``attn_merge``. Each rank thus sends and merges 1/P_kv of the row's data, instead of
every rank receiving and merging every fragment whole.

The page describes two variants: ATTENTION2D-NO keeps communication and computation
apart, ATTENTION2D-O overlaps them (section 3; section 4 reports the lower latency of
-O). ``overlap=False`` is -NO: compute the whole fragment, then exchange, then merge.
``overlap=True`` is -O: the heads are cut into ``n_splits`` groups (whole key/value
head groups under GQA); as soon as a group's fragment is computed its exchange is
started asynchronously, and the next group is computed while it travels; each
group is merged once its exchange has completed.
"""

from __future__ import annotations

import torch
import torch.distributed as dist

from . import ATTN_OK, AttnError, attn_device_status, attn_fwd_partial, attn_merge


def grid_coords(rank: int, p_q: int, p_kv: int) -> tuple[int, int]:
    """(query chunk, key/value chunk) of ``rank`` in a p_q x p_kv grid (row-major)."""
    if not 0 <= rank < p_q * p_kv:
        raise ValueError("rank outside the grid")
    return rank // p_kv, rank % p_kv


def row_groups(p_q: int, p_kv: int) -> list[list[int]]:
    """The ranks that share each query chunk (one list per query chunk)."""
    return [[i * p_kv + j for j in range(p_kv)] for i in range(p_q)]


def row_slices(Cq: int, p_kv: int) -> list[tuple[int, int]]:
    """The [start, stop) rows of a query chunk that each column of the grid receives
    after the reduce-scatter: Cq rows in p_kv contiguous slices, the first Cq % p_kv
    of them one row longer."""
    base, extra = divmod(Cq, p_kv)
    out, a = [], 0
    for m in range(p_kv):
        b = a + base + (1 if m < extra else 0)
        out.append((a, b))
        a = b
    return out


def head_splits(Hq: int, Hkv: int, n_splits: int) -> list[tuple[int, int, int, int]]:
    """(q head start, stop, kv head start, stop) of each head group of the -O variant:
    key/value heads in n_splits contiguous groups (fewer when Hkv is smaller), each
    with its query heads (Hq / Hkv per key/value head)."""
    n = max(1, min(n_splits, Hkv))
    g = Hq // Hkv
    out = []
    for a, b in row_slices(Hkv, n):
        if b > a:
            out.append((a * g, b * g, a, b))
    return out


def _default_partial(q, k, v, *, q_off, kv_off, causal, scale):
    C = q.shape[2]
    return attn_fwd_partial(q, k, v, q_start=0, q_len=C, kv_start=0, kv_len=k.shape[2],
                            causal=causal, scale=scale, q_off=q_off, kv_off=kv_off)


def _default_merge(o_parts, lse_parts):
    return attn_merge(o_parts, lse_parts)


def _rows_major(o, lse):
    """[B, H, Cq, d], [B, H, Cq] -> [Cq, B, H, d], [Cq, B, H] (contiguous), so that
    row slices are contiguous along dimension 0."""
    return o.permute(2, 0, 1, 3).contiguous(), lse.permute(2, 0, 1).contiguous()


class _Exchange:
    """The all-to-all of one head group's fragment within the row: started at once,
    completed by :meth:`merged`."""

    def __init__(self, o, lse, slices, me, row_group, order, merge, async_op):
        p_kv = len(slices)
        o_r, l_r = _rows_major(o, lse)
        sizes = [b - a for a, b in slices]
        mine = sizes[me]
        self.recv_o = torch.empty((p_kv * mine,) + tuple(o_r.shape[1:]), dtype=o_r.dtype,
                                  device=o_r.device)
        self.recv_l = torch.empty((p_kv * mine,) + tuple(l_r.shape[1:]), dtype=l_r.dtype,
                                  device=l_r.device)
        self.mine, self.p_kv, self.order, self.merge = mine, p_kv, order, merge
        self._send = (o_r, l_r)  # kept alive until the exchange completes
        self.works = [
            dist.all_to_all_single(self.recv_o, o_r, output_split_sizes=[mine] * p_kv,
                                   input_split_sizes=sizes, group=row_group,
                                   async_op=async_op),
            dist.all_to_all_single(self.recv_l, l_r, output_split_sizes=[mine] * p_kv,
                                   input_split_sizes=sizes, group=row_group,
                                   async_op=async_op),
        ]

    def merged(self):
        for w in self.works:
            if w is not None:
                w.wait()
        m = self.mine
        o_parts = [self.recv_o[x * m:(x + 1) * m] for x in self.order]
        l_parts = [self.recv_l[x * m:(x + 1) * m] for x in self.order]
        o, lse = self.merge(o_parts, l_parts)             # [m, B, H, d], [m, B, H]
        return o.permute(1, 2, 0, 3).contiguous(), lse.permute(1, 2, 0).contiguous()


def grid2d_attention_dist(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, p_q: int,
                          p_kv: int, causal: bool, scale: float | None = None,
                          row_group=None, merge_order=None, partial=None, merge=None,
                          overlap: bool = False, n_splits: int = 2, check_status: bool = True):
    """This rank's fragment of the grid, then the reduce-scatter along its row.

    q: [B, Hq, Cq, d], query chunk i of the sequence (rows i*Cq ..); k, v:
    [B, Hkv, Ckv, d], key/value chunk j (rows j*Ckv ..), with (i, j) =
    ``grid_coords(rank)``. ``row_group``: the process group of ``row_groups(p_q,
    p_kv)[i]`` (every rank must create all row groups, in the same order, as
    torch.distributed requires); None when p_kv == 1. ``merge_order``: the order of
    the key/value chunks in the combination (default 0..p_kv-1; any order gives the
    same result up to fp32 rounding). ``overlap``: the -O variant with ``n_splits``
    head groups (see the module docstring).

    Returns (O [B, Hq, R, d], LSE [B, Hq, R]) in fp32 for the rows
    ``row_slices(Cq, p_kv)[j]`` of query chunk i (global rows i*Cq + start ..).

    ``partial(q, k, v, *, q_off, kv_off, causal, scale) -> (O, LSE)`` and
    ``merge(o_parts, lse_parts) -> (O, LSE)`` replace the local compute; ``merge``
    gets parts of shape [R, B, H, d] / [R, B, H]. With the library's own compute and
    ``check_status``, the call ends by synchronising the current stream and raising
    ``AttnError`` if a kernel recorded a device-side time-out.
    """
    rank = dist.get_rank()
    if dist.get_world_size() != p_q * p_kv:
        raise ValueError("the world must be the p_q x p_kv grid")
    i, j = grid_coords(rank, p_q, p_kv)
    B, Hq, Cq, d = q.shape
    Hkv, Ckv = k.shape[1], k.shape[2]
    if scale is None:
        scale = d ** -0.5
    library = partial is None and merge is None
    partial = partial or _default_partial
    merge = merge or _default_merge
    order = list(range(p_kv)) if merge_order is None else list(merge_order)
    if sorted(order) != list(range(p_kv)):
        raise ValueError("merge_order must be a permutation of the key/value chunks")
    if p_kv == 1:
        res = partial(q, k, v, q_off=i * Cq, kv_off=j * Ckv, causal=causal, scale=scale)
        _check(library and check_status)
        return res
    if Cq < p_kv:
        raise ValueError("a query chunk needs at least one row per column of the grid")
    slices = row_slices(Cq, p_kv)
    groups = head_splits(Hq, Hkv, n_splits) if overlap else [(0, Hq, 0, Hkv)]
    pending = []
    for hq0, hq1, hk0, hk1 in groups:
        qs = q if (hq0, hq1) == (0, Hq) else q[:, hq0:hq1].contiguous()
        ks = k if (hk0, hk1) == (0, Hkv) else k[:, hk0:hk1].contiguous()
        vs = v if (hk0, hk1) == (0, Hkv) else v[:, hk0:hk1].contiguous()
        o, lse = partial(qs, ks, vs, q_off=i * Cq, kv_off=j * Ckv, causal=causal, scale=scale)
        # -NO: a blocking exchange after the whole fragment; -O: started now, waited
        # for after the next head group has been computed
        pending.append(_Exchange(o, lse, slices, j, row_group, order, merge,
                                 async_op=overlap))
    parts = [x.merged() for x in pending]
    _check(library and check_status)
    if len(parts) == 1:
        return parts[0]
    return torch.cat([p[0] for p in parts], dim=1), torch.cat([p[1] for p in parts], dim=1)


def _check(enabled: bool) -> None:
    if enabled:
        st = attn_device_status()
        if st != ATTN_OK:
            raise AttnError(st, "grid2d_attention_dist")

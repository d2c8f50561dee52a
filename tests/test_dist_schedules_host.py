"""ATTENTION2D over a grid of ranks (grid2d_dist.py) and Ulysses head-parallel attention
(ulysses_dist.py) on CPU ranks over gloo, with the fp64 oracle as the local compute:
what is checked is the data movement - which fragment a rank computes and with which
global offsets, the reduce-scatter and combination along a grid row (in both the
-NO and the overlapped -O variant, whose head groups travel separately), the two
all-to-all exchanges and the head grouping under GQA. Every rank's result must equal
the oracle's attention over the whole sequence for its rows.
"""

from __future__ import annotations

import os
import socket
import sys
from pathlib import Path

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = Path(__file__).resolve().parents[1]
sys.path.insert(0, str(ROOT))
sys.path.insert(0, str(ROOT / "tests"))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(B, Hq, Hkv, N, d, seed):
    from workloads import randn_bf16

    return (randn_bf16((B, Hq, N, d), seed, 0), randn_bf16((B, Hkv, N, d), seed, 1),
            randn_bf16((B, Hkv, N, d), seed, 2))


def _oracle_partial(q, k, v, *, q_off, kv_off, causal, scale):
    import torch

    import oracle

    o, lse = oracle.attention(q.contiguous(), k.contiguous(), v.contiguous(), causal=causal,
                              scale=scale, q_off=q_off, kv_off=kv_off, threads=1)
    return torch.from_numpy(o), torch.from_numpy(lse)


def _oracle_merge(o_parts, lse_parts):
    import torch

    import oracle

    o, lse = oracle.merge([t.numpy() for t in o_parts], [t.numpy() for t in lse_parts])
    return torch.from_numpy(o), torch.from_numpy(lse)


def _oracle_attend(q, k, v, *, causal, scale):
    return _oracle_partial(q, k, v, q_off=0, kv_off=0, causal=causal, scale=scale)


def _grid_worker(rank, world, port, p_q, p_kv, shape, causal, out_dir, overlap=False,
                 n_splits=2):
    import torch.distributed as dist

    from online_softmax_exact_b200.grid2d_dist import (grid2d_attention_dist, grid_coords,
                                                       row_groups)

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        groups = [dist.new_group(g) for g in row_groups(p_q, p_kv)]
        i, j = grid_coords(rank, p_q, p_kv)
        B, Hq, Hkv, N, d = shape
        q, k, v = _inputs(B, Hq, Hkv, N, d, seed=29)
        cq, ckv = N // p_q, N // p_kv
        order = list(range(p_kv))[::-1] if i % 2 else None   # any order: same result
        o, lse = grid2d_attention_dist(
            q[:, :, i * cq:(i + 1) * cq], k[:, :, j * ckv:(j + 1) * ckv],
            v[:, :, j * ckv:(j + 1) * ckv], p_q=p_q, p_kv=p_kv, causal=causal,
            scale=d ** -0.5, row_group=groups[i], merge_order=order,
            partial=_oracle_partial, merge=_oracle_merge, overlap=overlap, n_splits=n_splits)
        np.save(Path(out_dir, f"o{rank}.npy"), o.numpy())
        np.save(Path(out_dir, f"l{rank}.npy"), lse.numpy())
    finally:
        dist.destroy_process_group()


def _ulysses_worker(rank, world, port, shape, causal, out_dir):
    import torch.distributed as dist

    from online_softmax_exact_b200.ulysses_dist import ulysses_attention_dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, Hq, Hkv, N, d = shape
        q, k, v = _inputs(B, Hq, Hkv, N, d, seed=31)
        C = N // world
        sl = slice(rank * C, (rank + 1) * C)
        o, lse = ulysses_attention_dist(q[:, :, sl].contiguous(), k[:, :, sl].contiguous(),
                                        v[:, :, sl].contiguous(), causal=causal,
                                        scale=d ** -0.5, attend=_oracle_attend)
        np.save(Path(out_dir, f"o{rank}.npy"), o.numpy())
        np.save(Path(out_dir, f"l{rank}.npy"), lse.numpy())
    finally:
        dist.destroy_process_group()


def _reference(shape, causal, seed):
    import oracle

    B, Hq, Hkv, N, d = shape
    q, k, v = _inputs(B, Hq, Hkv, N, d, seed=seed)
    return oracle.attention(q, k, v, causal=causal, scale=d ** -0.5)


def test_grid_layout():
    from online_softmax_exact_b200.grid2d_dist import grid_coords, row_groups

    assert [grid_coords(r, 2, 3) for r in range(6)] == [(0, 0), (0, 1), (0, 2), (1, 0),
                                                        (1, 1), (1, 2)]
    assert row_groups(2, 3) == [[0, 1, 2], [3, 4, 5]]
    with pytest.raises(ValueError):
        grid_coords(6, 2, 3)


def test_row_slices_and_head_splits():
    from online_softmax_exact_b200.grid2d_dist import head_splits, row_slices

    assert row_slices(10, 3) == [(0, 4), (4, 7), (7, 10)]
    assert row_slices(6, 3) == [(0, 2), (2, 4), (4, 6)]
    for cq, p in ((1, 1), (7, 7), (100, 3), (129, 4)):
        sl = row_slices(cq, p)
        assert sl[0][0] == 0 and sl[-1][1] == cq
        assert all(a < b for a, b in sl) and all(sl[m][1] == sl[m + 1][0] for m in range(p - 1))
    # key/value heads split in groups, their query heads along with them (GQA ratio 4)
    assert head_splits(16, 4, 2) == [(0, 8, 0, 2), (8, 16, 2, 4)]
    assert head_splits(8, 1, 2) == [(0, 8, 0, 1)]          # one kv head: cannot split
    assert head_splits(6, 3, 2) == [(0, 4, 0, 2), (4, 6, 2, 3)]


@pytest.mark.parametrize("p_q,p_kv,shape,causal,overlap", [
    (2, 2, (1, 2, 2, 256, 64), True, False),
    (3, 2, (1, 4, 2, 384, 64), False, False),    # GQA; 3 query chunks x 2 kv chunks
    (2, 3, (2, 2, 1, 192, 128), True, False),    # causal cut inside unequal fragments
    (2, 3, (1, 6, 3, 192, 64), True, True),      # -O: head groups of 2 and 1 kv heads
    (2, 2, (2, 8, 4, 256, 64), False, True),     # -O, GQA 2
    (2, 4, (1, 2, 1, 140, 64), True, True),      # rows 70 per chunk: slices 18,18,17,17
])
def test_grid2d_across_gloo_ranks(tmp_path, p_q, p_kv, shape, causal, overlap):
    from online_softmax_exact_b200.grid2d_dist import row_slices

    world = p_q * p_kv
    mp.start_processes(_grid_worker,
                       args=(world, _free_port(), p_q, p_kv, shape, causal, str(tmp_path),
                             overlap),
                       nprocs=world, join=True, start_method="spawn")
    o_ref, l_ref = _reference(shape, causal, 29)
    cq = shape[3] // p_q
    for r in range(world):
        i, j = r // p_kv, r % p_kv
        a, b = row_slices(cq, p_kv)[j]
        o = np.load(tmp_path / f"o{r}.npy")
        lse = np.load(tmp_path / f"l{r}.npy")
        rows = slice(i * cq + a, i * cq + b)
        np.testing.assert_allclose(o, o_ref[:, :, rows], rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, l_ref[:, :, rows], rtol=0, atol=1e-12)


@pytest.mark.parametrize("world,shape,causal", [
    (2, (1, 4, 2, 256, 64), True),
    (4, (2, 8, 4, 256, 64), False),        # GQA: groups of 2 query heads stay whole
])
def test_ulysses_across_gloo_ranks(tmp_path, world, shape, causal):
    mp.start_processes(_ulysses_worker, args=(world, _free_port(), shape, causal,
                                              str(tmp_path)),
                       nprocs=world, join=True, start_method="spawn")
    o_ref, l_ref = _reference(shape, causal, 31)
    C = shape[3] // world
    for r in range(world):
        o = np.load(tmp_path / f"o{r}.npy")
        lse = np.load(tmp_path / f"l{r}.npy")
        np.testing.assert_allclose(o, o_ref[:, :, r * C:(r + 1) * C], rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, l_ref[:, :, r * C:(r + 1) * C], rtol=0, atol=1e-12)

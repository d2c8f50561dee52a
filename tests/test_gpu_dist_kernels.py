"""The cross-rank schedules with the library's CUDA kernels as the local compute, on
several ranks, against the fp64 oracle.

Every call here has one GPU, so the ranks are processes that all use cuda:0 and talk
over gloo on the host: each rank moves its operands to the GPU, runs
attn_fwd_partial / attn_fwd_partial_acc / attn_merge / attn_fwd there, and brings the
result back for the next exchange. No kernel waits on another process (each launch
is an ordinary, self-contained attention or merge), so sharing one GPU between the
ranks is safe. Each rank's rows must match the oracle's attention over the whole
sequence within the bf16 tolerance.

  * Ring Attention ("Ring Attention with Blockwise Parallel Transformers", section 3),
    contiguous and zigzag layouts;
  * ATTENTION2D (section 3), -NO and -O variants, reduce-scatter along grid rows;
  * Ulysses (all-to-all from sequence shards to head shards and back).
"""

from __future__ import annotations

import os
import socket
import sys
from datetime import timedelta
from pathlib import Path

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = Path(__file__).resolve().parents[1]
sys.path.insert(0, str(ROOT))
sys.path.insert(0, str(ROOT / "tests"))

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(B, Hq, Hkv, N, d, seed):
    from workloads import randn_bf16

    return (randn_bf16((B, Hq, N, d), seed, 0), randn_bf16((B, Hkv, N, d), seed, 1),
            randn_bf16((B, Hkv, N, d), seed, 2))


# ---- local compute through the library on cuda:0, operands and results on the host
def _gpu_fold(o, lse, q, k, v, *, q_off, kv_off, causal, scale, first):
    import torch

    import online_softmax_exact_b200 as osx

    dev = torch.device("cuda", 0)
    qg, kg, vg = q.to(dev), k.contiguous().to(dev), v.contiguous().to(dev)
    C, L = qg.shape[2], kg.shape[2]
    if first:
        og, lg = osx.attn_fwd_partial(qg, kg, vg, q_start=0, q_len=C, kv_start=0, kv_len=L,
                                      causal=causal, scale=scale, q_off=q_off, kv_off=kv_off)
    else:
        og, lg = o.to(dev), lse.to(dev)
        osx.attn_fwd_partial_acc(qg, kg, vg, q_start=0, q_len=C, kv_start=0, kv_len=L,
                                 causal=causal, scale=scale, q_off=q_off, kv_off=kv_off,
                                 o=og, lse=lg)
    o.copy_(og.cpu())
    lse.copy_(lg.cpu())
    assert osx.attn_device_status() == osx.ATTN_OK


def _gpu_partial(q, k, v, *, q_off, kv_off, causal, scale):
    import torch

    import online_softmax_exact_b200 as osx

    dev = torch.device("cuda", 0)
    qg, kg, vg = (t.contiguous().to(dev) for t in (q, k, v))
    og, lg = osx.attn_fwd_partial(qg, kg, vg, q_start=0, q_len=qg.shape[2], kv_start=0,
                                  kv_len=kg.shape[2], causal=causal, scale=scale,
                                  q_off=q_off, kv_off=kv_off)
    assert osx.attn_device_status() == osx.ATTN_OK
    return og.cpu(), lg.cpu()


def _gpu_merge(o_parts, lse_parts):
    import torch

    import online_softmax_exact_b200 as osx

    dev = torch.device("cuda", 0)
    og, lg = osx.attn_merge([t.contiguous().to(dev) for t in o_parts],
                            [t.contiguous().to(dev) for t in lse_parts])
    assert osx.attn_device_status() == osx.ATTN_OK
    return og.cpu(), lg.cpu()


def _gpu_attend(q, k, v, *, causal, scale):
    import torch

    import online_softmax_exact_b200 as osx

    dev = torch.device("cuda", 0)
    og, lg = osx.attn_fwd(q.contiguous().to(dev), k.contiguous().to(dev),
                          v.contiguous().to(dev), causal=causal, scale=scale)
    assert osx.attn_device_status() == osx.ATTN_OK
    return og.cpu(), lg.cpu()


def _init(rank, world, port):
    import torch
    import torch.distributed as dist

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=timedelta(seconds=180))


def _save(out_dir, rank, o, lse):
    np.save(Path(out_dir, f"o{rank}.npy"), o.double().numpy())
    np.save(Path(out_dir, f"l{rank}.npy"), lse.double().numpy())


def _ring_worker(rank, world, port, shape, causal, layout, out_dir):
    import torch
    import torch.distributed as dist

    from online_softmax_exact_b200.ring_dist import ring_attention_dist, zigzag_shard

    _init(rank, world, port)
    try:
        B, Hq, Hkv, N, d = shape
        q, k, v = _inputs(B, Hq, Hkv, N, d, seed=43)
        C = N // world
        if layout == "zigzag":
            ql, kl, vl = (zigzag_shard(t, rank, world) for t in (q, k, v))
        else:
            ql, kl, vl = (t[:, :, rank * C:(rank + 1) * C].contiguous() for t in (q, k, v))
        o = torch.empty((B, Hq, C, d), dtype=torch.float32)
        lse = torch.empty((B, Hq, C), dtype=torch.float32)
        ring_attention_dist(ql, kl, vl, causal=causal, scale=d ** -0.5, out=(o, lse),
                            fold=_gpu_fold, layout=layout)
        _save(out_dir, rank, o, lse)
    finally:
        dist.destroy_process_group()


def _grid_worker(rank, world, port, p_q, p_kv, shape, causal, overlap, out_dir):
    import torch.distributed as dist

    from online_softmax_exact_b200.grid2d_dist import (grid2d_attention_dist, grid_coords,
                                                       row_groups)

    _init(rank, world, port)
    try:
        groups = [dist.new_group(g) for g in row_groups(p_q, p_kv)]
        i, j = grid_coords(rank, p_q, p_kv)
        B, Hq, Hkv, N, d = shape
        q, k, v = _inputs(B, Hq, Hkv, N, d, seed=47)
        cq, ckv = N // p_q, N // p_kv
        order = list(range(p_kv))[::-1] if i % 2 else None
        o, lse = grid2d_attention_dist(
            q[:, :, i * cq:(i + 1) * cq], k[:, :, j * ckv:(j + 1) * ckv],
            v[:, :, j * ckv:(j + 1) * ckv], p_q=p_q, p_kv=p_kv, causal=causal,
            scale=d ** -0.5, row_group=groups[i], merge_order=order, partial=_gpu_partial,
            merge=_gpu_merge, overlap=overlap)
        _save(out_dir, rank, o, lse)
    finally:
        dist.destroy_process_group()


def _ulysses_worker(rank, world, port, shape, causal, out_dir):
    import torch.distributed as dist

    from online_softmax_exact_b200.ulysses_dist import ulysses_attention_dist

    _init(rank, world, port)
    try:
        B, Hq, Hkv, N, d = shape
        q, k, v = _inputs(B, Hq, Hkv, N, d, seed=53)
        C = N // world
        sl = slice(rank * C, (rank + 1) * C)
        o, lse = ulysses_attention_dist(q[:, :, sl].contiguous(), k[:, :, sl].contiguous(),
                                        v[:, :, sl].contiguous(), causal=causal,
                                        scale=d ** -0.5, attend=_gpu_attend)
        _save(out_dir, rank, o, lse)
    finally:
        dist.destroy_process_group()


def _reference(shape, causal, seed):
    import oracle

    B, Hq, Hkv, N, d = shape
    q, k, v = _inputs(B, Hq, Hkv, N, d, seed=seed)
    return oracle.attention(q, k, v, causal=causal, scale=d ** -0.5)


def _check(out_dir, rank, rows, o_ref, l_ref):
    from parity_util import compare

    o = np.load(Path(out_dir, f"o{rank}.npy"))
    lse = np.load(Path(out_dir, f"l{rank}.npy"))
    compare(o, lse, o_ref[:, :, rows], l_ref[:, :, rows])


@pytest.mark.parametrize("world,shape,causal,layout", [
    (3, (1, 4, 2, 1500, 128), True, "contiguous"),   # chunks of 500: ragged tiles, GQA
    (2, (2, 2, 2, 1024, 64), False, "contiguous"),
    (2, (1, 4, 4, 1000, 128), True, "zigzag"),       # halves of 250
    (4, (1, 4, 2, 2048, 64), True, "zigzag"),
])
def test_ring_on_gpu_ranks(tmp_path, world, shape, causal, layout):
    from online_softmax_exact_b200.ring_dist import zigzag_rows

    mp.start_processes(_ring_worker, args=(world, _free_port(), shape, causal, layout,
                                           str(tmp_path)),
                       nprocs=world, join=True, start_method="spawn")
    o_ref, l_ref = _reference(shape, causal, 43)
    C = shape[3] // world
    for r in range(world):
        if layout == "zigzag":
            rows = np.concatenate([np.arange(x.start, x.stop)
                                   for x in zigzag_rows(r, world, C)])
        else:
            rows = np.arange(r * C, (r + 1) * C)
        _check(tmp_path, r, rows, o_ref, l_ref)


@pytest.mark.parametrize("p_q,p_kv,shape,causal,overlap", [
    (2, 2, (1, 4, 2, 1024, 128), True, False),
    (2, 2, (1, 8, 4, 1200, 64), False, True),    # -O: two head groups; chunks of 600
    (1, 3, (2, 6, 3, 768, 128), True, True),
])
def test_grid2d_on_gpu_ranks(tmp_path, p_q, p_kv, shape, causal, overlap):
    from online_softmax_exact_b200.grid2d_dist import row_slices

    world = p_q * p_kv
    mp.start_processes(_grid_worker, args=(world, _free_port(), p_q, p_kv, shape, causal,
                                           overlap, str(tmp_path)),
                       nprocs=world, join=True, start_method="spawn")
    o_ref, l_ref = _reference(shape, causal, 47)
    cq = shape[3] // p_q
    for r in range(world):
        i, j = r // p_kv, r % p_kv
        a, b = row_slices(cq, p_kv)[j]
        _check(tmp_path, r, np.arange(i * cq + a, i * cq + b), o_ref, l_ref)


@pytest.mark.parametrize("world,shape,causal", [
    (2, (1, 4, 2, 1024, 128), True),
    (4, (1, 8, 4, 768, 64), False),
])
def test_ulysses_on_gpu_ranks(tmp_path, world, shape, causal):
    mp.start_processes(_ulysses_worker, args=(world, _free_port(), shape, causal,
                                              str(tmp_path)),
                       nprocs=world, join=True, start_method="spawn")
    o_ref, l_ref = _reference(shape, causal, 53)
    C = shape[3] // world
    for r in range(world):
        _check(tmp_path, r, np.arange(r * C, (r + 1) * C), o_ref, l_ref)

"""The multi-rank Ring Attention schedule (ring_dist.py) on CPU ranks over gloo.

Each rank holds one chunk of the sequence; the ranks pass K/V chunks around the ring
with point-to-point messages. The local compute is replaced by the fp64 oracle (a
partial over the held chunk, folded into the running result with the oracle's merge),
so what is checked is the schedule itself: which chunk a rank holds at each step,
the global offsets, the causal skipping, and the send/receive pairing and buffer
swaps. Every rank's result must equal the oracle's attention over the whole
sequence for its rows.
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


def _oracle_fold(o, lse, q, k, v, *, q_off, kv_off, causal, scale, first):
    import torch

    import oracle

    o_p, l_p = oracle.attention(q, k.contiguous(), v.contiguous(), causal=causal,
                                scale=scale, q_off=q_off, kv_off=kv_off, threads=1)
    if not first:
        o_p, l_p = oracle.merge([o.numpy(), o_p], [lse.numpy(), l_p])
    o.copy_(torch.from_numpy(o_p))
    lse.copy_(torch.from_numpy(l_p))


def _worker(rank, world, port, shape, causal, out_dir, layout="contiguous"):
    import torch
    import torch.distributed as dist

    from online_softmax_exact_b200.ring_dist import ring_attention_dist, zigzag_shard

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, Hq, Hkv, N, d = shape
        q, k, v = _inputs(B, Hq, Hkv, N, d, seed=17)
        C = N // world
        if layout == "zigzag":
            ql, kl, vl = (zigzag_shard(t, rank, world) for t in (q, k, v))
        else:
            sl = slice(rank * C, (rank + 1) * C)
            ql, kl, vl = (t[:, :, sl].contiguous() for t in (q, k, v))
        o = torch.zeros((B, Hq, C, d), dtype=torch.float64)
        lse = torch.zeros((B, Hq, C), dtype=torch.float64)
        ring_attention_dist(ql, kl, vl, causal=causal, scale=d ** -0.5, out=(o, lse),
                            fold=_oracle_fold, layout=layout)
        np.save(Path(out_dir, f"o{rank}.npy"), o.numpy())
        np.save(Path(out_dir, f"l{rank}.npy"), lse.numpy())
    finally:
        dist.destroy_process_group()


def test_ring_steps_follow_the_ring_order():
    from online_softmax_exact_b200.ring_dist import ring_steps
    from online_softmax_exact_b200.schedules import ring_order

    for P in (1, 2, 5, 8):
        for causal in (False, True):
            order = ring_order(P, causal)
            for r in range(P):
                steps = ring_steps(r, P, causal)
                assert [s for s, _, _ in steps] == list(range(P))
                # every chunk passes through every rank exactly once
                assert sorted(kv for _, kv, _ in steps) == list(range(P))
                # the folded chunks, in fold order, are the single-GPU ring schedule's
                assert [kv for _, kv, f in steps if f] == order[r]
                # what a rank holds at step s+1 is what its predecessor held at step s
                prev = ring_steps((r - 1) % P, P, causal)
                for s in range(P - 1):
                    assert steps[s + 1][1] == prev[s][1]


@pytest.mark.parametrize("world,shape,causal", [
    (2, (1, 2, 2, 256, 64), True),
    (3, (1, 4, 2, 384, 64), True),     # GQA, odd ring
    (3, (2, 2, 1, 192, 128), False),
])
def test_ring_attention_across_gloo_ranks(tmp_path, world, shape, causal):
    import oracle

    mp.start_processes(_worker, args=(world, _free_port(), shape, causal, str(tmp_path)),
                       nprocs=world, join=True, start_method="spawn")
    B, Hq, Hkv, N, d = shape
    q, k, v = _inputs(B, Hq, Hkv, N, d, seed=17)
    o_ref, l_ref = oracle.attention(q, k, v, causal=causal, scale=d ** -0.5)
    C = N // world
    for r in range(world):
        o = np.load(tmp_path / f"o{r}.npy")
        lse = np.load(tmp_path / f"l{r}.npy")
        np.testing.assert_allclose(o, o_ref[:, :, r * C:(r + 1) * C], rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, l_ref[:, :, r * C:(r + 1) * C], rtol=0, atol=1e-12)


def test_zigzag_steps_balance_the_causal_work():
    """Zigzag layout: every key/value half reaches every query half exactly once, the
    causal mask's visible pairs are exactly those with kv half <= q half, and every
    rank folds the same visible work at every step (2 half-by-half blocks, a diagonal
    block counting one half)."""
    from online_softmax_exact_b200.ring_dist import zigzag_halves, zigzag_rows, zigzag_steps

    for P in (1, 2, 3, 4, 8):
        assert sorted(x for r in range(P) for x in zigzag_halves(r, P)) == list(range(2 * P))
        assert [list(x) for x in zigzag_rows(1, 4, 10)] == [list(range(5, 10)),
                                                            list(range(30, 35))]
        for causal in (False, True):
            for r in range(P):
                steps = zigzag_steps(r, P, causal)
                seen = {(qa, kb) for _, _, folds in steps for _, _, qa, kb in folds}
                mine = zigzag_halves(r, P)
                want = {(qa, kb) for qa in mine for kb in range(2 * P)
                        if not (causal and kb > qa)}
                assert seen == want
                assert sum(len(f) for _, _, f in steps) == len(want)   # no repeats
                if causal:
                    for _, _, folds in steps:
                        work = sum(0.5 if qa == kb else 1.0 for _, _, qa, kb in folds)
                        assert work == 2.0
                # what a rank holds at step s+1 is what its predecessor held at step s
                prev = zigzag_steps((r - 1) % P, P, causal)
                for s in range(P - 1):
                    assert steps[s + 1][1] == prev[s][1]


@pytest.mark.parametrize("world,shape,causal", [
    (2, (1, 2, 2, 256, 64), True),
    (4, (1, 4, 2, 512, 64), True),     # GQA
    (3, (2, 2, 1, 192, 128), False),
])
def test_zigzag_ring_across_gloo_ranks(tmp_path, world, shape, causal):
    import oracle
    from online_softmax_exact_b200.ring_dist import zigzag_rows

    mp.start_processes(_worker, args=(world, _free_port(), shape, causal, str(tmp_path),
                                      "zigzag"),
                       nprocs=world, join=True, start_method="spawn")
    B, Hq, Hkv, N, d = shape
    q, k, v = _inputs(B, Hq, Hkv, N, d, seed=17)
    o_ref, l_ref = oracle.attention(q, k, v, causal=causal, scale=d ** -0.5)
    C = N // world
    for r in range(world):
        rows = np.concatenate([np.arange(x.start, x.stop) for x in zigzag_rows(r, world, C)])
        o = np.load(tmp_path / f"o{r}.npy")
        lse = np.load(tmp_path / f"l{r}.npy")
        np.testing.assert_allclose(o, o_ref[:, :, rows], rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, l_ref[:, :, rows], rtol=0, atol=1e-12)

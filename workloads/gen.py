"""Seeded synthetic inputs (host, torch CPU generator).

Every tensor is drawn per (b, head) slice from its own generator, so that any
slice can be regenerated alone and the result does not depend on how many
slices are drawn at once. Values are drawn in fp32 from N(0, 1) and rounded to
bf16 once; the same host bf16 tensor feeds both the CUDA path and the oracle.
"""

from __future__ import annotations

import numpy as np
import torch

from .configs import Workload

_MIX = 1_000_003
_MASK = (1 << 63) - 1

# tensor ids used in seed derivation
_Q, _K, _V, _KSTRESS, _ROWS, _ORDER = 0, 1, 2, 3, 4, 5


def slice_seed(seed: int, tensor_id: int, b: int = 0, h: int = 0) -> int:
    s = seed
    for x in (tensor_id, b, h):
        s = (s * _MIX + x + 1) & _MASK
    return s


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def randn_bf16(shape, seed: int, tensor_id: int = 0) -> torch.Tensor:
    """bf16 tensor ``[B, H, N, d]`` of i.i.d. N(0,1) draws, generated per (b, h)."""
    B, H, N, d = shape
    out = torch.empty((B, H, N, d), dtype=torch.bfloat16)
    for b in range(B):
        for h in range(H):
            g = _gen(slice_seed(seed, tensor_id, b, h))
            out[b, h] = torch.randn((N, d), generator=g, dtype=torch.float32).to(torch.bfloat16)
    return out


def stress_rows(N: int, seed: int, b: int, h: int) -> torch.Tensor:
    """The floor(0.01*N) distinct K rows of (b, kv head h) that the rescale-stress
    workload multiplies by 16, from a seeded permutation."""
    n = (N * 1) // 100
    g = _gen(slice_seed(seed, _KSTRESS, b, h))
    return torch.randperm(N, generator=g)[:n]


def attention_inputs(w: Workload, N: int | None = None):
    """(q, k, v) bf16 CPU tensors for workload ``w`` (optionally at another N).

    The stress transform multiplies Q by 8 and the rows chosen by
    :func:`stress_rows` of K by 16; both factors are powers of two, so they are
    exact in bf16.
    """
    N = w.N if N is None else N
    q = randn_bf16((w.B, w.Hq, N, w.d), w.seed, _Q)
    k = randn_bf16((w.B, w.Hkv, N, w.d), w.seed, _K)
    v = randn_bf16((w.B, w.Hkv, N, w.d), w.seed, _V)
    if w.stress:
        q.mul_(8)
        for b in range(w.B):
            for h in range(w.Hkv):
                idx = stress_rows(N, w.seed, b, h)
                k[b, h, idx] = k[b, h, idx] * 16
    return q, k, v


def sample_rows(N: int, chunk: int, count: int, seed: int, tile: int = 128) -> np.ndarray:
    """Sorted distinct query rows for sampled checks at full size.

    Always includes rows 0, 1, N-1, the first and last row of every chunk, and the
    rows either side of the 128-row tile boundaries next to them; the rest are
    uniform draws from a seeded generator until ``count`` rows are reached.
    """
    fixed = {0, 1, N - 1}
    for c0 in range(0, N, max(chunk, 1)):
        for r in (c0, c0 + 1, c0 + chunk - 1, c0 + tile - 1, c0 + tile, c0 + chunk - tile,
                  c0 + chunk - tile - 1):
            if 0 <= r < N:
                fixed.add(r)
    rows = sorted(fixed)
    if len(rows) >= count:
        # keep the boundary rows spread over the sequence
        pick = np.linspace(0, len(rows) - 1, count).round().astype(np.int64)
        return np.unique(np.asarray(rows, dtype=np.int64)[pick])
    g = _gen(slice_seed(seed, _ROWS))
    extra = torch.randperm(N, generator=g).numpy()
    have = set(rows)
    for r in extra:
        if len(have) >= count:
            break
        have.add(int(r))
    return np.asarray(sorted(have), dtype=np.int64)


def grid_merge_orders(n_chunks: int, seed: int) -> list[list[int]]:
    """For each Q chunk of a 2-D grid, a seeded random order of its KV chunks."""
    out = []
    for qi in range(n_chunks):
        g = _gen(slice_seed(seed, _ORDER, qi))
        out.append([int(x) for x in torch.randperm(n_chunks, generator=g)])
    return out


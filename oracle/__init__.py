"""fp64 CPU oracle for exact blockwise attention forward and the (O, LSE) merge.

TEST INFRASTRUCTURE ONLY. Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg import this package. The CUDA library never imports,
links or calls it, and it imports nothing from the CUDA library: the two share no
code. Its inputs are the host bf16 tensors from :mod:`workloads`.

Contents
--------
``attention_rows`` / ``attention``
    The plain definition ("FlashAttention by hand", paragraph on the conventional
    three-step computation): logits, a materialised softmax row summing to one,
    weights times values; plus LSE = max + ln(sum of exp), natural log. Written in
    C (``attn_oracle.c``), fp64, OpenMP over rows.
``merge``
    Combination of partial results (O_i, LSE_i) computed over disjoint key sets:
    the log-sum-exp weighted convex combination. ATTENTION2D (section 3) combines
    fragment-local statistics in stages and relies on that combination being
    commutative and associative; this is the plainest formula with both
    properties, and it is the same rescale-to-a-common-maximum step the online
    softmax takes ("FlashAttention by hand", paragraphs on the running statistics
    and on rescaling).
``online_softmax_replay``
    The tiled algorithm in the order "FlashAttention by hand" describes it: keep an
    output accumulator, the running maximum and the running denominator; for each
    key/value tile compute its logits and tile maximum, fold them into the running
    statistics, rescale the accumulator and denominator when the maximum grows;
    divide once at the end. With ``normalise_each_step`` it keeps the output
    normalised after every tile instead (the per-step form the page says is
    mathematically equivalent). fp64, numpy, for small cases.

Parity pins for every function are in ``tests/test_oracle_pins.py``.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "attn_oracle.c"
_LIB_PATH = _HERE / "liboracle.so"
_lib = None


def build(force: bool = False) -> Path:
    """Compile ``attn_oracle.c`` into ``liboracle.so`` (gcc, -O2, OpenMP, strict IEEE)."""
    if force or not _LIB_PATH.exists() or _LIB_PATH.stat().st_mtime < _SRC.stat().st_mtime:
        tmp = _LIB_PATH.with_suffix(f".{os.getpid()}.tmp.so")
        cmd = ["gcc", "-std=c11", "-O2", "-fopenmp", "-fPIC", "-shared", "-Wall", "-Wextra",
               "-o", str(tmp), str(_SRC), "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(str(_LIB_PATH))
        lib.oracle_attention_rows.restype = ctypes.c_int
        lib.oracle_attention_rows.argtypes = [
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int64, ctypes.c_int64,
            ctypes.c_int, ctypes.c_int, ctypes.c_int64, ctypes.c_int64, ctypes.c_double,
            ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_int,
        ]
        lib.oracle_default_threads.restype = ctypes.c_int
        lib.oracle_default_threads.argtypes = []
        _lib = lib
    return _lib


def default_threads() -> int:
    return int(_load().oracle_default_threads())


def _bf16_bits(t) -> np.ndarray:
    """Dense uint16 numpy view of the bf16 bit patterns of a CPU tensor or array."""
    try:
        import torch

        if isinstance(t, torch.Tensor):
            assert t.dtype == torch.bfloat16 and t.device.type == "cpu"
            return t.contiguous().view(torch.int16).numpy().view(np.uint16)
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(t)
    assert a.dtype == np.uint16
    return a


def scale_as_used(scale: float) -> float:
    """The scale is handed to the GPU as a float; the oracle uses that float, widened."""
    return float(np.float32(scale))


def attention_rows(q, k, v, *, causal: bool, scale: float, rows=None, q_off: int = 0,
                   kv_off: int = 0, want_p: bool = False, threads: int = 0):
    """fp64 attention for the listed query rows of every (batch, head).

    q: bf16 ``[B, Hq, Nq, d]``; k, v: bf16 ``[B, Hkv, Nkv, d]`` (CPU tensors or uint16
    bit arrays). ``rows`` defaults to all rows. Returns ``(O, LSE)`` or
    ``(O, LSE, P)`` with O ``[B, Hq, R, d]``, LSE ``[B, Hq, R]``, P ``[B, Hq, R, Nkv]``.
    """
    qb, kb, vb = _bf16_bits(q), _bf16_bits(k), _bf16_bits(v)
    B, Hq, Nq, d = qb.shape
    Bk, Hkv, Nkv, dk = kb.shape
    assert vb.shape == kb.shape and Bk == B and dk == d
    if rows is None:
        rows = np.arange(Nq, dtype=np.int64)
    rows = np.ascontiguousarray(rows, dtype=np.int64)
    R = rows.shape[0]
    o = np.zeros((B, Hq, R, d), dtype=np.float64)
    lse = np.zeros((B, Hq, R), dtype=np.float64)
    p = np.zeros((B, Hq, R, Nkv), dtype=np.float64) if want_p else None
    rc = _load().oracle_attention_rows(
        qb.ctypes.data, kb.ctypes.data, vb.ctypes.data, B, Hq, Hkv, Nq, Nkv, d,
        1 if causal else 0, int(q_off), int(kv_off), scale_as_used(scale),
        rows.ctypes.data, R, o.ctypes.data, lse.ctypes.data,
        p.ctypes.data if p is not None else None, int(threads))
    if rc != 0:
        raise ValueError(f"oracle_attention_rows failed with code {rc}")
    return (o, lse, p) if want_p else (o, lse)


def attention(q, k, v, *, causal: bool, scale: float, q_off: int = 0, kv_off: int = 0,
              threads: int = 0):
    """fp64 attention over all query rows: ``(O [B,Hq,Nq,d], LSE [B,Hq,Nq])``."""
    return attention_rows(q, k, v, causal=causal, scale=scale, q_off=q_off, kv_off=kv_off,
                          threads=threads)


def merge(o_parts, lse_parts):
    """Combine partial results over disjoint key sets, in fp64.

    With M = max_i LSE_i and w_i = exp(LSE_i - M):
    O = sum_i w_i O_i / sum_i w_i and LSE = M + ln(sum_i w_i).
    Parts whose LSE is -inf carry no keys and get weight 0; if every part is
    -inf the result is O = 0, LSE = -inf.
    """
    lse_stack = np.stack([np.asarray(x, dtype=np.float64) for x in lse_parts])
    o_stack = np.stack([np.asarray(x, dtype=np.float64) for x in o_parts])
    M = lse_stack.max(axis=0)
    empty = np.isneginf(M)
    M_safe = np.where(empty, 0.0, M)
    w = np.exp(lse_stack - M_safe[None])          # exp(-inf) = 0 for empty parts
    wsum = w.sum(axis=0)
    wsum_safe = np.where(empty, 1.0, wsum)
    o = (w[..., None] * o_stack).sum(axis=0) / wsum_safe[..., None]
    o = np.where(empty[..., None], 0.0, o)
    lse = np.where(empty, -np.inf, M_safe + np.log(wsum_safe))
    return o, lse


def online_softmax_replay(q, k, v, *, causal: bool, scale: float, tile: int,
                          q_off: int = 0, kv_off: int = 0,
                          normalise_each_step: bool = False):
    """The tiled online-softmax algorithm, replayed in fp64 for every row.

    q: bf16 ``[B, Hq, Nq, d]``; k, v: bf16 ``[B, Hkv, Nkv, d]``. Keys are visited in
    tiles of ``tile``. Returns ``(O, LSE)`` like :func:`attention`.
    """
    import torch

    qd = q.to(torch.float64).numpy() if isinstance(q, torch.Tensor) else q
    kd = k.to(torch.float64).numpy() if isinstance(k, torch.Tensor) else k
    vd = v.to(torch.float64).numpy() if isinstance(v, torch.Tensor) else v
    B, Hq, Nq, d = qd.shape
    Hkv, Nkv = kd.shape[1], kd.shape[2]
    group = Hq // Hkv
    sc = scale_as_used(scale)
    O = np.zeros((B, Hq, Nq, d))
    LSE = np.zeros((B, Hq, Nq))
    qpos = q_off + np.arange(Nq)
    for b in range(B):
        for h in range(Hq):
            g = h // group
            acc = np.zeros((Nq, d))       # output accumulator
            m = np.full(Nq, -np.inf)      # running maximum of the logits
            l = np.zeros(Nq)              # running softmax denominator
            for j0 in range(0, Nkv, tile):
                j1 = min(j0 + tile, Nkv)
                s = sc * (qd[b, h] @ kd[b, g, j0:j1].T)          # this tile's logits
                if causal:
                    kpos = kv_off + np.arange(j0, j1)
                    s = np.where(kpos[None, :] <= qpos[:, None], s, -np.inf)
                m_tile = s.max(axis=1)                            # tile maximum
                m_new = np.maximum(m, m_tile)
                live = ~np.isneginf(m_new)
                m_ref = np.where(live, m_new, 0.0)
                alpha = np.where(live, np.exp(m - m_ref), 1.0)    # rescale factor
                p = np.exp(s - m_ref[:, None])                    # unnormalised weights
                l_new = alpha * l + p.sum(axis=1)
                if normalise_each_step:
                    # keep acc == (normalised output so far)
                    l_safe = np.where(l_new > 0, l_new, 1.0)
                    acc = ((alpha * l)[:, None] * acc + p @ vd[b, g, j0:j1]) / l_safe[:, None]
                else:
                    acc = alpha[:, None] * acc + p @ vd[b, g, j0:j1]
                l, m = l_new, m_new
            nonempty = l > 0
            l_safe = np.where(nonempty, l, 1.0)
            if normalise_each_step:
                O[b, h] = np.where(nonempty[:, None], acc, 0.0)
            else:
                O[b, h] = np.where(nonempty[:, None], acc / l_safe[:, None], 0.0)  # one divide
            LSE[b, h] = np.where(nonempty, m + np.log(l_safe), -np.inf)
    return O, LSE

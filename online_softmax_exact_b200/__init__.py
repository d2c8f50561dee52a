"""Exact blockwise self-attention forward and (O, LSE) merge for NVIDIA B200 (sm_100a).

A thin binding over the C ABI of ``libattn.so`` (``include/attn.h``): the functions
here check and marshal torch tensors and call the entry point of the same name.
All arithmetic runs in the library's CUDA kernels; torch provides device memory and
streams only. The library is loaded on first use; if it is missing or out of date
that first call raises (there is no fallback implementation).
"""

from __future__ import annotations

import ctypes

import torch

from ._abi import (
    ATTN_MAX_BATCH_PAIRS,
    AttnPair,
    ATTN_ERR_CUDA,
    ATTN_ERR_INJECTED,
    ATTN_ERR_INVALID_ARG,
    ATTN_ERR_TIMEOUT,
    ATTN_ERR_UNSUPPORTED,
    ATTN_MAX_MERGE_PARTS,
    ATTN_OK,
    AttnError,
    load,
)

_lib_handle = None


def lib() -> ctypes.CDLL:
    """The loaded libattn.so (loaded on first use)."""
    global _lib_handle
    if _lib_handle is None:
        _lib_handle = load()
    return _lib_handle

__all__ = [
    "ATTN_OK", "ATTN_ERR_INVALID_ARG", "ATTN_ERR_UNSUPPORTED", "ATTN_ERR_CUDA",
    "ATTN_ERR_TIMEOUT", "ATTN_ERR_INJECTED", "ATTN_MAX_MERGE_PARTS", "AttnError",
    "attn_fwd", "attn_fwd_partial", "attn_fwd_partial_acc", "attn_fwd_partial_batch",
    "attn_merge", "ATTN_MAX_BATCH_PAIRS", "attn_device_status", "attn_debug_inject",
    "attn_launch_count", "attn_status_string", "attn_version", "lib",
    "attn_debug_wait_timeout",
]


def _stream_handle(device: torch.device, stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _check(st: int, where: str) -> None:
    if st != ATTN_OK:
        raise AttnError(st, where)


def _need(t: torch.Tensor, dtype, name: str) -> None:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def attn_status_string(status: int) -> str:
    return lib().attn_status_string(int(status)).decode()


def attn_version() -> int:
    return int(lib().attn_version())


def attn_launch_count() -> int:
    return int(lib().attn_launch_count())


def attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, causal: bool,
             scale: float | None = None, o: torch.Tensor | None = None,
             lse: torch.Tensor | None = None, stream=None):
    """Single-pass exact attention. q bf16 [B,Hq,N,d]; k, v bf16 [B,Hkv,N,d].

    Returns (O fp32 [B,Hq,N,d], LSE fp32 [B,Hq,N]) - allocated here unless given.
    """
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, n)
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    if k.shape != (B, Hkv, N, d) or v.shape != k.shape:
        raise ValueError("k and v must be [B, Hkv, N, d] matching q")
    if scale is None:
        scale = d ** -0.5
    if o is None:
        o = torch.empty((B, Hq, N, d), dtype=torch.float32, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device)
    _need(o, torch.float32, "o")
    _need(lse, torch.float32, "lse")
    st = lib().attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                       B, Hq, Hkv, N, d, int(bool(causal)), float(scale),
                       _stream_handle(q.device, stream))
    _check(st, "attn_fwd")
    return o, lse


def _partial(entry: str, q, k, v, q_start, q_len, kv_start, kv_len, causal, scale, q_off,
             kv_off, o, lse, stream, alloc: bool):
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, n)
    B, Hq, Lq, d = q.shape
    Hkv, Lkv = k.shape[1], k.shape[2]
    if v.shape != k.shape or k.shape[0] != B or k.shape[3] != d:
        raise ValueError("k and v must be [B, Hkv, Lkv, d] matching q")
    if not (0 <= q_start and q_start + q_len <= Lq and 0 <= kv_start and kv_start + kv_len <= Lkv):
        raise ValueError("chunk outside its parent tensor")
    if scale is None:
        scale = d ** -0.5
    q_off = q_start if q_off is None else q_off
    kv_off = kv_start if kv_off is None else kv_off
    if o is None or lse is None:
        if not alloc:
            raise ValueError("the accumulator (o, lse) must be given")
        o = torch.empty((B, Hq, q_len, d), dtype=torch.float32, device=q.device) if o is None else o
        lse = torch.empty((B, Hq, q_len), dtype=torch.float32, device=q.device) if lse is None else lse
    _need(o, torch.float32, "o")
    _need(lse, torch.float32, "lse")
    if o.shape != (B, Hq, q_len, d) or lse.shape != (B, Hq, q_len):
        raise ValueError("o / lse must be [B, Hq, q_len, d] / [B, Hq, q_len]")
    es = q.element_size()
    st = getattr(lib(), entry)(
        q.data_ptr() + q_start * d * es, k.data_ptr() + kv_start * d * es,
        v.data_ptr() + kv_start * d * es, o.data_ptr(), lse.data_ptr(), B, Hq, Hkv,
        q_len, kv_len, Lq, Lkv, int(q_off), int(kv_off), d, int(bool(causal)), float(scale),
        _stream_handle(q.device, stream))
    _check(st, entry)
    return o, lse


def attn_fwd_partial(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, q_start: int,
                     q_len: int, kv_start: int, kv_len: int, causal: bool,
                     scale: float | None = None, q_off: int | None = None,
                     kv_off: int | None = None, o: torch.Tensor | None = None,
                     lse: torch.Tensor | None = None, stream=None):
    """Attention of query rows [q_start, q_start+q_len) against key/value rows
    [kv_start, kv_start+kv_len) of the parent tensors q [B,Hq,Lq,d], k/v [B,Hkv,Lkv,d].

    Global positions for the causal test default to the row indices in the parents
    (q_off = q_start, kv_off = kv_start). Returns the normalised partial
    (O fp32 [B,Hq,q_len,d], LSE fp32 [B,Hq,q_len]).
    """
    return _partial("attn_fwd_partial", q, k, v, q_start, q_len, kv_start, kv_len, causal,
                    scale, q_off, kv_off, o, lse, stream, alloc=True)


def attn_fwd_partial_acc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, q_start: int,
                         q_len: int, kv_start: int, kv_len: int, causal: bool,
                         o: torch.Tensor, lse: torch.Tensor, scale: float | None = None,
                         q_off: int | None = None, kv_off: int | None = None, stream=None):
    """Like :func:`attn_fwd_partial`, folding the chunk's result into the accumulator
    (o, lse) in place (log-sum-exp merge). Returns (o, lse)."""
    return _partial("attn_fwd_partial_acc", q, k, v, q_start, q_len, kv_start, kv_len,
                    causal, scale, q_off, kv_off, o, lse, stream, alloc=False)


def attn_fwd_partial_batch(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, pairs, *,
                           causal: bool, scale: float | None = None, accumulate: bool = False,
                           stream=None):
    """Several chunk pairs of the same parents in one launch. ``pairs`` is a sequence of
    dicts with keys q_start, q_len, kv_start, kv_len, o, lse and optionally q_off, kv_off
    (default: the row starts). With ``accumulate`` every (o, lse) is an in/out
    accumulator, as for :func:`attn_fwd_partial_acc`; otherwise it receives the pair's
    normalised partial."""
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, torch.bfloat16, n)
    B, Hq, Lq, d = q.shape
    Hkv, Lkv = k.shape[1], k.shape[2]
    if v.shape != k.shape or k.shape[0] != B or k.shape[3] != d:
        raise ValueError("k and v must be [B, Hkv, Lkv, d] matching q")
    if scale is None:
        scale = d ** -0.5
    n = len(pairs)
    arr = (AttnPair * max(n, 1))()
    for i, pr in enumerate(pairs):
        o, lse = pr["o"], pr["lse"]
        _need(o, torch.float32, "o")
        _need(lse, torch.float32, "lse")
        if o.shape != (B, Hq, pr["q_len"], d) or lse.shape != (B, Hq, pr["q_len"]):
            raise ValueError("o / lse must be [B, Hq, q_len, d] / [B, Hq, q_len]")
        arr[i] = AttnPair(pr["q_start"], pr["q_len"], pr["kv_start"], pr["kv_len"],
                          pr.get("q_off", pr["q_start"]), pr.get("kv_off", pr["kv_start"]),
                          o.data_ptr(), lse.data_ptr())
    st = lib().attn_fwd_partial_batch(q.data_ptr(), k.data_ptr(), v.data_ptr(), B, Hq, Hkv,
                                      Lq, Lkv, d, int(bool(causal)), float(scale), arr, n,
                                      int(bool(accumulate)), _stream_handle(q.device, stream))
    _check(st, "attn_fwd_partial_batch")


def attn_merge(o_parts, lse_parts, *, o: torch.Tensor | None = None,
               lse: torch.Tensor | None = None, stream=None):
    """Merge partial results over disjoint key sets. o_parts: fp32 tensors [..., d];
    lse_parts: fp32 tensors [...] with the same leading shape. Returns (O, LSE)."""
    n = len(o_parts)
    if n < 1 or n != len(lse_parts):
        raise ValueError("need matching, non-empty lists of parts")
    ref = o_parts[0]
    for t in o_parts:
        _need(t, torch.float32, "o_parts[i]")
        if t.shape != ref.shape:
            raise ValueError("all O parts must have one shape")
    for t in lse_parts:
        _need(t, torch.float32, "lse_parts[i]")
        if t.shape != ref.shape[:-1]:
            raise ValueError("LSE parts must match O parts without the last dim")
    d = ref.shape[-1]
    rows = ref.numel() // d
    if o is None:
        o = torch.empty_like(ref)
    if lse is None:
        lse = torch.empty(ref.shape[:-1], dtype=torch.float32, device=ref.device)
    _need(o, torch.float32, "o")
    _need(lse, torch.float32, "lse")
    optr = (ctypes.c_void_p * n)(*[t.data_ptr() for t in o_parts])
    lptr = (ctypes.c_void_p * n)(*[t.data_ptr() for t in lse_parts])
    st = lib().attn_merge(optr, lptr, n, o.data_ptr(), lse.data_ptr(), rows, d,
                         _stream_handle(ref.device, stream))
    _check(st, "attn_merge")
    return o, lse


def attn_device_status(stream=None, reset: bool = False) -> int:
    """Synchronise the stream; return ATTN_OK or ATTN_ERR_TIMEOUT (device-side record)."""
    dev = torch.device("cuda", torch.cuda.current_device())
    return int(lib().attn_device_status(_stream_handle(dev, stream), int(bool(reset))))


def attn_debug_inject(status: int, count: int) -> None:
    _check(lib().attn_debug_inject(int(status), int(count)), "attn_debug_inject")


def attn_debug_wait_timeout(limit_cycles: int, stream=None) -> None:
    """Launch the failure-path check kernel (a bounded wait that must run out)."""
    dev = torch.device("cuda", torch.cuda.current_device())
    _check(lib().attn_debug_wait_timeout(int(limit_cycles), _stream_handle(dev, stream)),
           "attn_debug_wait_timeout")

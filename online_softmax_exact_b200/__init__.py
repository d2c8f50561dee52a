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
    ATTN_NOALLOC_SCRATCH_BYTES,
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
    "attn_debug_wait_timeout", "attn_ring_fwd_host", "RingHostBuffers",
    "attn_ring_fwd_host_noalloc", "ATTN_NOALLOC_SCRATCH_BYTES", "attn_debug_exp2",
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


class RingHostBuffers:
    """Device buffers of :func:`attn_ring_fwd_host`: bf16 staging for q, k, v
    ([B, H, N, d]), the chunk-major fp32 result (O [P, B, Hq, C, d], LSE [P, B, Hq, C])
    and the partial slots (P of them when P > 1)."""

    def __init__(self, B: int, Hq: int, Hkv: int, N: int, d: int, n_chunks: int, device):
        if n_chunks < 1 or N % n_chunks:
            raise ValueError("the sequence length must split into equal chunks")
        C = N // n_chunks
        bf = dict(dtype=torch.bfloat16, device=device)
        f32 = dict(dtype=torch.float32, device=device)
        self.shape = (B, Hq, Hkv, N, d, n_chunks)
        self.q = torch.empty((B, Hq, N, d), **bf)
        self.k = torch.empty((B, Hkv, N, d), **bf)
        self.v = torch.empty((B, Hkv, N, d), **bf)
        self.o = torch.empty((n_chunks, B, Hq, C, d), **f32)
        self.lse = torch.empty((n_chunks, B, Hq, C), **f32)
        slots = n_chunks if n_chunks > 1 else 0
        self.ws_o = torch.empty((max(slots, 1), B, Hq, C, d), **f32)
        self.ws_lse = torch.empty((max(slots, 1), B, Hq, C), **f32)
        self.slots = slots

    def tensors(self):
        return [self.q, self.k, self.v, self.o, self.lse, self.ws_o, self.ws_lse]


_copy_streams: dict = {}

# Host tensors of attn_ring_fwd_host calls whose copies may still be queued: each entry
# holds an event recorded after the call's work and the tensors it reads or writes, so
# that a temporary (e.g. ``q.pin_memory()`` passed inline) is not freed, and its pinned
# block reused, before the copies have run. Entries go once their event has completed.
_inflight_host: list = []


def _keep_alive_until_done(stream, tensors) -> None:
    _inflight_host[:] = [(ev, ts) for ev, ts in _inflight_host if not ev.query()]
    ev = torch.cuda.Event()
    ev.record(stream)
    _inflight_host.append((ev, tuple(tensors)))


def _host_copy_streams(device: torch.device):
    if device.index not in _copy_streams:
        _copy_streams[device.index] = (torch.cuda.Stream(device), torch.cuda.Stream(device))
    return _copy_streams[device.index]


def attn_ring_fwd_host(q_h: torch.Tensor, k_h: torch.Tensor, v_h: torch.Tensor, *,
                       n_chunks: int, causal: bool, scale: float | None = None,
                       o_h: torch.Tensor | None = None, lse_h: torch.Tensor | None = None,
                       buffers: RingHostBuffers | None = None, device=None, stream=None,
                       h2d_stream=None, d2h_stream=None):
    """Ring Attention's schedule on one GPU from host tensors to host tensors, with the
    copies pipelined against the compute (see attn_ring_fwd_host in attn.h).
    q_h / k_h / v_h: CPU bf16 [B, H, N, d] (page-locked for overlap). Returns the
    chunk-major CPU fp32 (O [P, B, Hq, C, d], LSE [P, B, Hq, C]); the copies are
    asynchronous, so synchronise ``stream`` before reading them."""
    for t, n in ((q_h, "q_h"), (k_h, "k_h"), (v_h, "v_h")):
        if not isinstance(t, torch.Tensor) or t.is_cuda or t.dtype != torch.bfloat16 \
                or not t.is_contiguous():
            raise ValueError(f"{n} must be a contiguous CPU bf16 tensor")
    B, Hq, N, d = q_h.shape
    Hkv = k_h.shape[1]
    if v_h.shape != k_h.shape or k_h.shape[0] != B or k_h.shape[2] != N or k_h.shape[3] != d:
        raise ValueError("k_h and v_h must be [B, Hkv, N, d] matching q_h")
    if n_chunks < 1 or N % n_chunks:
        raise ValueError("the sequence length must split into equal chunks")
    C = N // n_chunks
    dev = torch.device(device) if device is not None else \
        torch.device("cuda", torch.cuda.current_device())
    if buffers is None:
        buffers = RingHostBuffers(B, Hq, Hkv, N, d, n_chunks, dev)
    elif buffers.shape != (B, Hq, Hkv, N, d, n_chunks):
        raise ValueError("buffers were made for another shape")
    if o_h is None:
        o_h = torch.empty((n_chunks, B, Hq, C, d), dtype=torch.float32).pin_memory()
    if lse_h is None:
        lse_h = torch.empty((n_chunks, B, Hq, C), dtype=torch.float32).pin_memory()
    for t, shape, n in ((o_h, (n_chunks, B, Hq, C, d), "o_h"),
                        (lse_h, (n_chunks, B, Hq, C), "lse_h")):
        if t.is_cuda or t.dtype != torch.float32 or not t.is_contiguous() \
                or tuple(t.shape) != shape:
            raise ValueError(f"{n} must be a contiguous CPU fp32 tensor of shape {shape}")
    if scale is None:
        scale = d ** -0.5
    s_main = stream if stream is not None else torch.cuda.current_stream(dev)
    if h2d_stream is None or d2h_stream is None:
        hs, ds = _host_copy_streams(dev)
        h2d_stream = h2d_stream or hs
        d2h_stream = d2h_stream or ds
    for t in buffers.tensors():  # also used on the copy streams
        t.record_stream(h2d_stream)
        t.record_stream(d2h_stream)
    b = buffers
    st = lib().attn_ring_fwd_host(
        q_h.data_ptr(), k_h.data_ptr(), v_h.data_ptr(), o_h.data_ptr(), lse_h.data_ptr(),
        b.q.data_ptr(), b.k.data_ptr(), b.v.data_ptr(), b.o.data_ptr(), b.lse.data_ptr(),
        b.ws_o.data_ptr() if b.slots else None, b.ws_lse.data_ptr() if b.slots else None,
        b.slots, B, Hq, Hkv, N, d, n_chunks, int(bool(causal)), float(scale),
        _stream_handle(dev, s_main), _stream_handle(dev, h2d_stream),
        _stream_handle(dev, d2h_stream))
    _check(st, "attn_ring_fwd_host")
    # later work on s_main waits for the last copy back (see attn.h)
    _keep_alive_until_done(s_main, (q_h, k_h, v_h, o_h, lse_h))
    return o_h, lse_h


def attn_ring_fwd_host_noalloc(q_h: torch.Tensor, k_h: torch.Tensor, v_h: torch.Tensor, *,
                               n_chunks: int, causal: bool, o_h: torch.Tensor,
                               lse_h: torch.Tensor, scale: float | None = None,
                               device=None, stream=None, h2d_stream=None, d2h_stream=None):
    """attn_ring_fwd_host without device allocations: for callers that cannot allocate
    device memory (the device buffers live in the library's fixed array of
    ATTN_NOALLOC_SCRATCH_BYTES per GPU; see attn_ring_fwd_host_noalloc in attn.h).
    The host outputs o_h / lse_h must be given (chunk-major, as attn_ring_fwd_host
    returns them). Calls whose work overlaps on the GPU race: keep them on one stream."""
    for t, n in ((q_h, "q_h"), (k_h, "k_h"), (v_h, "v_h")):
        if not isinstance(t, torch.Tensor) or t.is_cuda or t.dtype != torch.bfloat16 \
                or not t.is_contiguous():
            raise ValueError(f"{n} must be a contiguous CPU bf16 tensor")
    B, Hq, N, d = q_h.shape
    Hkv = k_h.shape[1]
    if n_chunks < 1 or N % n_chunks:
        raise ValueError("the sequence length must split into equal chunks")
    C = N // n_chunks
    for t, shape, n in ((o_h, (n_chunks, B, Hq, C, d), "o_h"),
                        (lse_h, (n_chunks, B, Hq, C), "lse_h")):
        if t.is_cuda or t.dtype != torch.float32 or not t.is_contiguous() \
                or tuple(t.shape) != shape:
            raise ValueError(f"{n} must be a contiguous CPU fp32 tensor of shape {shape}")
    if scale is None:
        scale = d ** -0.5
    dev = torch.device(device) if device is not None else \
        torch.device("cuda", torch.cuda.current_device())
    s_main = stream if stream is not None else torch.cuda.current_stream(dev)
    st = lib().attn_ring_fwd_host_noalloc(
        q_h.data_ptr(), k_h.data_ptr(), v_h.data_ptr(), o_h.data_ptr(), lse_h.data_ptr(),
        B, Hq, Hkv, N, d, n_chunks, int(bool(causal)), float(scale),
        _stream_handle(dev, s_main),
        _stream_handle(dev, h2d_stream) if h2d_stream is not None else None,
        _stream_handle(dev, d2h_stream) if d2h_stream is not None else None)
    _check(st, "attn_ring_fwd_host_noalloc")
    _keep_alive_until_done(s_main, (q_h, k_h, v_h, o_h, lse_h))
    return o_h, lse_h


def attn_device_status(stream=None, reset: bool = False) -> int:
    """Synchronise the stream; return ATTN_OK or ATTN_ERR_TIMEOUT (device-side record)."""
    dev = torch.device("cuda", torch.cuda.current_device())
    return int(lib().attn_device_status(_stream_handle(dev, stream), int(bool(reset))))


def attn_debug_inject(status: int, count: int) -> None:
    _check(lib().attn_debug_inject(int(status), int(count)), "attn_debug_inject")


def attn_debug_exp2(x: torch.Tensor, *, use_poly: bool, stream=None) -> torch.Tensor:
    """2^x of a CUDA fp32 tensor through the softmax's FMA-pipe polynomial (use_poly)
    or through the exp unit (ex2.approx); for tests of the polynomial."""
    _need(x, torch.float32, "x")
    y = torch.empty_like(x)
    _check(lib().attn_debug_exp2(x.data_ptr(), y.data_ptr(), x.numel(), int(bool(use_poly)),
                                 _stream_handle(x.device, stream)), "attn_debug_exp2")
    return y


def attn_debug_wait_timeout(limit_cycles: int, stream=None) -> None:
    """Launch the failure-path check kernel (a bounded wait that must run out)."""
    dev = torch.device("cuda", torch.cuda.current_device())
    _check(lib().attn_debug_wait_timeout(int(limit_cycles), _stream_handle(dev, stream)),
           "attn_debug_wait_timeout")

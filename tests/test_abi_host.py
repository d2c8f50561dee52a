"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every
entry point include/attn.h declares, and rejects bad arguments before touching a
device."""

from __future__ import annotations

import ctypes
import re
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parents[1]
HEADER = ROOT / "include" / "attn.h"


@pytest.fixture(scope="module")
def lib():
    from online_softmax_exact_b200 import build as b

    b.build()
    from online_softmax_exact_b200 import _abi

    return _abi.load()


def declared_functions() -> list[str]:
    text = HEADER.read_text()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(attn_[a-z0-9_]+)\s*\(",
                      text, flags=re.M)


def test_header_declares_the_abi():
    names = declared_functions()
    assert {"attn_fwd", "attn_fwd_partial", "attn_merge"} <= set(names)
    assert len(names) == len(set(names))


def test_every_declared_symbol_is_exported(lib):
    from online_softmax_exact_b200 import _abi

    for name in declared_functions():
        assert hasattr(lib, name), f"{name} not exported"
        assert name in _abi.SIGNATURES, f"{name} missing from the Python binding"
    assert set(_abi.SIGNATURES) == set(declared_functions())


def test_status_strings(lib):
    for code in range(6):
        s = lib.attn_status_string(code).decode()
        assert s.startswith("ATTN_")
    assert lib.attn_status_string(99).decode() == "unknown attn status"
    assert lib.attn_version() >> 16 == 1


A = 0x10000  # a 16-byte aligned fake address: never dereferenced by validation


def fwd(lib, q=A, k=2 * A, v=3 * A, o=4 * A, lse=8 * A, B=1, Hq=2, Hkv=2, N=64, d=64, causal=0,
        scale=0.125):
    return lib.attn_fwd(q, k, v, o, lse, B, Hq, Hkv, N, d, causal, scale, None)


def test_fwd_argument_checks(lib):
    from online_softmax_exact_b200._abi import (ATTN_ERR_INVALID_ARG, ATTN_ERR_UNSUPPORTED)

    big = 1 << 40
    assert fwd(lib, q=None) == ATTN_ERR_INVALID_ARG
    assert fwd(lib, o=None) == ATTN_ERR_INVALID_ARG
    assert fwd(lib, q=A + 8) == ATTN_ERR_INVALID_ARG          # misaligned
    assert fwd(lib, lse=8 * A + 2) == ATTN_ERR_INVALID_ARG    # misaligned
    assert fwd(lib, Hq=3, Hkv=2) == ATTN_ERR_INVALID_ARG
    assert fwd(lib, B=0) == ATTN_ERR_INVALID_ARG
    assert fwd(lib, N=0) == ATTN_ERR_INVALID_ARG
    assert fwd(lib, causal=2) == ATTN_ERR_INVALID_ARG
    assert fwd(lib, scale=-1.0) == ATTN_ERR_INVALID_ARG
    assert fwd(lib, scale=float("nan")) == ATTN_ERR_INVALID_ARG
    assert fwd(lib, scale=float("inf")) == ATTN_ERR_INVALID_ARG
    assert fwd(lib, d=96) == ATTN_ERR_UNSUPPORTED
    assert fwd(lib, d=256) == ATTN_ERR_UNSUPPORTED
    assert fwd(lib, o=A) == ATTN_ERR_INVALID_ARG               # output aliases q
    assert fwd(lib, o=A + 64 * 64) == ATTN_ERR_INVALID_ARG     # output overlaps q
    assert fwd(lib, lse=4 * A + 16) == ATTN_ERR_INVALID_ARG    # lse overlaps o
    assert fwd(lib, N=1 << 31, q=big, k=2 * big, v=3 * big, o=4 * big,
               lse=8 * big) == ATTN_ERR_UNSUPPORTED


def test_partial_argument_checks(lib):
    from online_softmax_exact_b200._abi import ATTN_ERR_INVALID_ARG

    def part(Nq=64, Nkv=64, q_ld=64, kv_ld=64, q_off=0, kv_off=0):
        return lib.attn_fwd_partial(A, 2 * A, 3 * A, 4 * A, 8 * A, 1, 2, 2, Nq, Nkv, q_ld, kv_ld,
                                    q_off, kv_off, 64, 1, 0.125, None)

    assert part(q_ld=32) == ATTN_ERR_INVALID_ARG
    assert part(kv_ld=10) == ATTN_ERR_INVALID_ARG
    assert part(q_off=-1) == ATTN_ERR_INVALID_ARG
    assert part(kv_off=-5) == ATTN_ERR_INVALID_ARG
    assert part(Nkv=0) == ATTN_ERR_INVALID_ARG


def test_merge_argument_checks(lib):
    from online_softmax_exact_b200._abi import (ATTN_ERR_INVALID_ARG, ATTN_ERR_UNSUPPORTED)

    P = ctypes.c_void_p

    def merge(n=2, parts_o=None, parts_l=None, o=16 * A, lse=32 * A, rows=100, d=64):
        po = parts_o if parts_o is not None else [A, 2 * A][:n] + [3 * A] * max(0, n - 2)
        pl = parts_l if parts_l is not None else [4 * A + 64 * i for i in range(n)]
        oa = (P * max(n, 1))(*po)
        la = (P * max(n, 1))(*pl)
        return lib.attn_merge(oa, la, n, o, lse, rows, d, None)

    assert merge(n=0) == ATTN_ERR_INVALID_ARG
    assert merge(rows=0) == ATTN_ERR_INVALID_ARG
    assert merge(d=32) == ATTN_ERR_UNSUPPORTED
    assert merge(n=65, parts_o=[A] * 65, parts_l=[4 * A] * 65) == ATTN_ERR_UNSUPPORTED
    assert merge(parts_o=[A, None]) == ATTN_ERR_INVALID_ARG
    assert merge(parts_o=[A + 4, 2 * A]) == ATTN_ERR_INVALID_ARG  # misaligned part
    assert merge(parts_o=[A + 16, 2 * A]) == ATTN_ERR_INVALID_ARG  # parts need 32 bytes
    assert merge(o=16 * A + 16) == ATTN_ERR_INVALID_ARG           # so does the output
    assert merge(o=A) == ATTN_ERR_INVALID_ARG                     # output aliases a part
    assert merge(lse=4 * A) == ATTN_ERR_INVALID_ARG               # lse aliases a part


def test_injection_and_no_device(lib):
    """With no GPU, a valid call reaches the device set-up and reports ATTN_ERR_CUDA;
    an injected failure is returned before that."""
    import torch

    from online_softmax_exact_b200._abi import ATTN_ERR_CUDA, ATTN_ERR_INJECTED, ATTN_ERR_INVALID_ARG

    if torch.cuda.is_available():
        pytest.skip("checks the no-device path")
    assert lib.attn_debug_inject(0, 1) == ATTN_ERR_INVALID_ARG   # success is not a failure code
    assert lib.attn_debug_inject(ATTN_ERR_INJECTED, 2) == 0
    n0 = lib.attn_launch_count()
    assert fwd(lib) == ATTN_ERR_INJECTED
    assert fwd(lib, q=None) != ATTN_ERR_INJECTED                   # checks come first
    assert fwd(lib) == ATTN_ERR_INJECTED
    assert fwd(lib) == ATTN_ERR_CUDA
    assert lib.attn_launch_count() == n0
    assert lib.attn_debug_inject(0, 0) == 0


def test_batch_argument_checks(lib):
    from online_softmax_exact_b200._abi import (ATTN_ERR_INVALID_ARG, ATTN_ERR_UNSUPPORTED,
                                                AttnPair)

    def batch(pairs, n=None, q_ld=1024, kv_ld=1024, d=64, accumulate=0):
        arr = (AttnPair * max(1, len(pairs)))(*pairs)
        return lib.attn_fwd_partial_batch(A, 2 * A, 3 * A, 1, 2, 2, q_ld, kv_ld, d, 1, 0.125,
                                          arr, len(pairs) if n is None else n, accumulate, None)

    big = 1 << 36
    ok_pair = AttnPair(0, 256, 0, 256, 0, 0, big, big + (1 << 24))
    assert batch([ok_pair], n=0) == ATTN_ERR_INVALID_ARG
    assert batch([ok_pair] * 49) == ATTN_ERR_UNSUPPORTED
    assert batch([ok_pair], d=96) == ATTN_ERR_UNSUPPORTED
    assert batch([ok_pair], accumulate=2) == ATTN_ERR_INVALID_ARG
    assert batch([AttnPair(900, 256, 0, 256, 0, 0, big, big + (1 << 24))]) == ATTN_ERR_INVALID_ARG
    assert batch([AttnPair(0, 256, 0, 0, 0, 0, big, big + (1 << 24))]) == ATTN_ERR_INVALID_ARG
    assert batch([AttnPair(0, 256, 0, 256, -1, 0, big, big + (1 << 24))]) == ATTN_ERR_INVALID_ARG
    assert batch([AttnPair(0, 256, 0, 256, 0, 0, None, big)]) == ATTN_ERR_INVALID_ARG
    assert batch([AttnPair(0, 256, 0, 256, 0, 0, A, big)]) == ATTN_ERR_INVALID_ARG  # o on q
    # two pairs writing the same output
    assert batch([ok_pair, AttnPair(256, 256, 0, 256, 0, 0, big, big + (1 << 25))]) == \
        ATTN_ERR_INVALID_ARG


def test_ring_host_argument_checks(lib):
    """attn_ring_fwd_host checks every argument before any CUDA call; with no device a
    valid call fails only at the first CUDA call, and an injected failure before it."""
    import torch

    from online_softmax_exact_b200._abi import (ATTN_ERR_CUDA, ATTN_ERR_INJECTED,
                                                ATTN_ERR_INVALID_ARG, ATTN_ERR_UNSUPPORTED)

    G = 1 << 32  # device buffers 4 GiB apart (B=1, H=2, N=1024, d=64 needs far less)
    H = 1 << 44  # fake host addresses, never dereferenced by the checks

    def ring(q_h=H, k_h=H + A, v_h=H + 2 * A, o_h=H + 3 * A, lse_h=H + 4 * A, q_d=G,
             k_d=2 * G, v_d=3 * G, o_d=4 * G, lse_d=5 * G, ws_o=6 * G, ws_lse=7 * G,
             ws_slots=4, B=1, Hq=2, Hkv=2, N=1024, d=64, n_chunks=4, causal=1, scale=0.125):
        return lib.attn_ring_fwd_host(q_h, k_h, v_h, o_h, lse_h, q_d, k_d, v_d, o_d, lse_d,
                                      ws_o, ws_lse, ws_slots, B, Hq, Hkv, N, d, n_chunks, causal,
                                      scale, None, None, None)

    assert ring(q_h=None) == ATTN_ERR_INVALID_ARG
    assert ring(lse_d=None) == ATTN_ERR_INVALID_ARG
    assert ring(n_chunks=3) == ATTN_ERR_INVALID_ARG            # 1024 rows do not split in 3
    assert ring(n_chunks=0) == ATTN_ERR_INVALID_ARG
    assert ring(n_chunks=64, N=64 * 16) == ATTN_ERR_UNSUPPORTED
    assert ring(d=96) == ATTN_ERR_UNSUPPORTED
    assert ring(causal=2) == ATTN_ERR_INVALID_ARG
    assert ring(scale=float("nan")) == ATTN_ERR_INVALID_ARG
    assert ring(o_d=4 * G + 16) == ATTN_ERR_INVALID_ARG         # merge output needs 32 bytes
    assert ring(ws_slots=3) == ATTN_ERR_INVALID_ARG             # the last chunk visits 4
    assert ring(ws_o=None) == ATTN_ERR_INVALID_ARG
    assert ring(ws_lse=5 * G) == ATTN_ERR_INVALID_ARG           # overlaps lse_d
    assert ring(k_d=G + 4096) == ATTN_ERR_INVALID_ARG           # overlaps q_d
    assert ring(Hq=3, Hkv=2) == ATTN_ERR_INVALID_ARG
    if torch.cuda.is_available():
        return
    # one chunk needs no partial buffers
    assert lib.attn_debug_inject(ATTN_ERR_INJECTED, 1) == 0
    assert ring(n_chunks=1, ws_o=None, ws_lse=None, ws_slots=0) == ATTN_ERR_INJECTED
    n0 = lib.attn_launch_count()
    assert ring() == ATTN_ERR_CUDA
    assert lib.attn_launch_count() == n0


def test_debug_exp2_argument_checks(lib):
    from online_softmax_exact_b200._abi import ATTN_ERR_INVALID_ARG

    assert lib.attn_debug_exp2(None, 2 * A, 16, 1, None) == ATTN_ERR_INVALID_ARG
    assert lib.attn_debug_exp2(A, None, 16, 1, None) == ATTN_ERR_INVALID_ARG
    assert lib.attn_debug_exp2(A, 2 * A, 0, 1, None) == ATTN_ERR_INVALID_ARG
    assert lib.attn_debug_exp2(A, 2 * A, 16, 2, None) == ATTN_ERR_INVALID_ARG
    assert lib.attn_debug_exp2(A, A + 32, 16, 1, None) == ATTN_ERR_INVALID_ARG   # overlap
    assert lib.attn_debug_exp2(A + 2, 2 * A, 16, 1, None) == ATTN_ERR_INVALID_ARG


def test_noalloc_argument_checks(lib):
    """The allocation-free ring call rejects bad arguments, and sizes its array cannot
    hold, before any CUDA call."""
    from online_softmax_exact_b200._abi import (ATTN_ERR_INVALID_ARG, ATTN_ERR_UNSUPPORTED,
                                                ATTN_NOALLOC_SCRATCH_BYTES)

    def call(B=1, Hq=2, Hkv=2, N=256, d=64, n_chunks=2, q=A):
        return lib.attn_ring_fwd_host_noalloc(q, 2 * A, 3 * A, 4 * A, 5 * A, B, Hq, Hkv, N, d,
                                              n_chunks, 1, 0.125, None, None, None)

    assert call(q=None) == ATTN_ERR_INVALID_ARG
    assert call(Hq=3, Hkv=2) == ATTN_ERR_INVALID_ARG
    assert call(N=255) == ATTN_ERR_INVALID_ARG           # 2 chunks do not divide 255
    assert call(d=96) == ATTN_ERR_UNSUPPORTED
    assert call(n_chunks=64, N=64 * 64) == ATTN_ERR_UNSUPPORTED
    # Q alone is larger than the array
    big_n = ATTN_NOALLOC_SCRATCH_BYTES // (2 * 64 * 2) + 256
    assert call(N=big_n, n_chunks=1) == ATTN_ERR_UNSUPPORTED
    # a size that fits Q, K, V but not the result and partial slots as well
    n_fit = ATTN_NOALLOC_SCRATCH_BYTES // (8 * 2 * 64 * 2) * 2
    assert call(N=n_fit, n_chunks=2) == ATTN_ERR_UNSUPPORTED

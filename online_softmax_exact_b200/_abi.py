"""ctypes view of libattn.so (the C ABI declared in include/attn.h).

Loading fails loudly: there is no fallback implementation of any entry point.
"""

from __future__ import annotations

import ctypes
from pathlib import Path

LIB_PATH = Path(__file__).resolve().parent / "libattn.so"

ATTN_OK = 0
ATTN_ERR_INVALID_ARG = 1
ATTN_ERR_UNSUPPORTED = 2
ATTN_ERR_CUDA = 3
ATTN_ERR_TIMEOUT = 4
ATTN_ERR_INJECTED = 5
ATTN_MAX_MERGE_PARTS = 64
ATTN_MAX_BATCH_PAIRS = 48
ATTN_NOALLOC_SCRATCH_BYTES = 64 * 1024 * 1024


class AttnPair(ctypes.Structure):
    """attn_pair_t of include/attn.h."""

    _fields_ = [("q_start", ctypes.c_int64), ("q_len", ctypes.c_int64),
                ("kv_start", ctypes.c_int64), ("kv_len", ctypes.c_int64),
                ("q_off", ctypes.c_int64), ("kv_off", ctypes.c_int64),
                ("o", ctypes.c_void_p), ("lse", ctypes.c_void_p)]

STATUS_NAMES = {
    ATTN_OK: "ATTN_OK",
    ATTN_ERR_INVALID_ARG: "ATTN_ERR_INVALID_ARG",
    ATTN_ERR_UNSUPPORTED: "ATTN_ERR_UNSUPPORTED",
    ATTN_ERR_CUDA: "ATTN_ERR_CUDA",
    ATTN_ERR_TIMEOUT: "ATTN_ERR_TIMEOUT",
    ATTN_ERR_INJECTED: "ATTN_ERR_INJECTED",
}

# name -> (restype, argtypes), in the order include/attn.h declares them
_c_void_p, _i32, _i64, _f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float
SIGNATURES = {
    "attn_status_string": (ctypes.c_char_p, [_i32]),
    "attn_version": (_i32, []),
    "attn_fwd": (_i32, [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p,
                        _i32, _i32, _i32, _i64, _i32, _i32, _f32, _c_void_p]),
    "attn_fwd_partial": (_i32, [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p,
                                _i32, _i32, _i32, _i64, _i64, _i64, _i64, _i64, _i64,
                                _i32, _i32, _f32, _c_void_p]),
    "attn_fwd_partial_acc": (_i32, [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p,
                                    _i32, _i32, _i32, _i64, _i64, _i64, _i64, _i64, _i64,
                                    _i32, _i32, _f32, _c_void_p]),
    "attn_fwd_partial_batch": (_i32, [_c_void_p, _c_void_p, _c_void_p, _i32, _i32, _i32, _i64,
                                      _i64, _i32, _i32, _f32, ctypes.POINTER(AttnPair), _i32,
                                      _i32, _c_void_p]),
    "attn_merge": (_i32, [ctypes.POINTER(_c_void_p), ctypes.POINTER(_c_void_p), _i32,
                          _c_void_p, _c_void_p, _i64, _i32, _c_void_p]),
    "attn_ring_fwd_host": (_i32, [_c_void_p] * 12 + [_i32, _i32, _i32, _i32, _i64, _i32, _i32,
                                                     _i32, _f32, _c_void_p, _c_void_p,
                                                     _c_void_p]),
    "attn_ring_fwd_host_noalloc": (_i32, [_c_void_p] * 5 + [_i32, _i32, _i32, _i64, _i32, _i32,
                                                            _i32, _f32, _c_void_p, _c_void_p,
                                                            _c_void_p]),
    "attn_device_status": (_i32, [_c_void_p, _i32]),
    "attn_debug_inject": (_i32, [_i32, _i32]),
    "attn_debug_wait_timeout": (_i32, [_i64, _c_void_p]),
    "attn_debug_exp2": (_i32, [_c_void_p, _c_void_p, _i64, _i32, _c_void_p]),
    "attn_launch_count": (ctypes.c_uint64, []),
}


class AttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")


_lib = None


def load() -> ctypes.CDLL:
    """Load libattn.so from the package directory (built by ``build.py``)."""
    global _lib
    if _lib is None:
        if not LIB_PATH.exists():
            raise ImportError(
                f"{LIB_PATH} is missing: build it with `python -m online_softmax_exact_b200.build`"
                " (there is no fallback implementation)")
        lib = ctypes.CDLL(str(LIB_PATH))
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib

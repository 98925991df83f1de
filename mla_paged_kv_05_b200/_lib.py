"""ctypes loader for libmla_decode.so (argument marshalling only).

The library must exist in this package directory (built by
``python -m mla_paged_kv_05_b200.build`` or ``__graft_entry__.build()``).
There is no fallback: if it is missing, every call raises.
"""

from __future__ import annotations

import ctypes
import os
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmla_decode.so")

MLA_OK = 0
MLA_ERR_INVALID_ARG = -1
MLA_ERR_UNSUPPORTED = -2
MLA_ERR_WORKSPACE_TOO_SMALL = -3
MLA_ERR_CUDA = -4
MLA_ERR_DEVICE_FLAG = -5

STATUS_NAMES = {
    MLA_OK: "MLA_OK",
    MLA_ERR_INVALID_ARG: "MLA_ERR_INVALID_ARG",
    MLA_ERR_UNSUPPORTED: "MLA_ERR_UNSUPPORTED",
    MLA_ERR_WORKSPACE_TOO_SMALL: "MLA_ERR_WORKSPACE_TOO_SMALL",
    MLA_ERR_CUDA: "MLA_ERR_CUDA",
    MLA_ERR_DEVICE_FLAG: "MLA_ERR_DEVICE_FLAG",
}

MLA_KV_BF16 = 0
MLA_KV_FP8_E4M3 = 1

PHASE_ATTEND = 1
PHASE_COMBINE = 2

NOALLOC_SCRATCH_BYTES = 48 << 20   # MLA_NOALLOC_SCRATCH_BYTES

FLAG_TIMEOUT = 1
FLAG_BAD_SEQLEN = 2
FLAG_BAD_PAGE = 4
FLAG_BAD_PREFIX = 8
FLAG_PLAN_MISMATCH = 16

# every symbol include/mla_decode.h declares, with its ctypes signature
_c_int, _c_void_p, _c_size_t, _c_float = ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_float
SIGNATURES = {
    "mla_decode_plan": (_c_int, [_c_void_p, _c_void_p, ctypes.c_int64, _c_int, _c_int, _c_int, _c_int, _c_int,
                                 _c_int, _c_void_p, ctypes.POINTER(_c_size_t), ctypes.POINTER(_c_int), _c_void_p]),
    "mla_decode_run": (_c_int, [_c_void_p, _c_void_p, ctypes.c_int64, _c_int, _c_void_p, _c_void_p, _c_void_p,
                                _c_void_p, _c_int, _c_int, _c_int, _c_int, _c_float, _c_void_p, _c_size_t,
                                _c_void_p]),
    "mla_decode_run_phases": (_c_int, [_c_void_p, _c_void_p, ctypes.c_int64, _c_int, _c_void_p, _c_void_p,
                                       _c_void_p, _c_void_p, _c_int, _c_int, _c_int, _c_int, _c_float, _c_void_p,
                                       _c_size_t, _c_int, _c_void_p]),
    "mla_decode_noalloc": (_c_int, [_c_void_p, _c_void_p, ctypes.c_int64, _c_int, _c_void_p, _c_void_p, _c_void_p,
                                    _c_void_p, _c_int, _c_int, _c_int, _c_int, _c_float, _c_void_p]),
    "mla_cache_append": (_c_int, [_c_void_p, _c_void_p, ctypes.c_int64, _c_int, _c_void_p, _c_void_p, _c_int,
                                  _c_int, _c_int, _c_void_p, _c_void_p]),
    "mla_absorb_q": (_c_int, [_c_void_p, _c_void_p, _c_void_p, _c_int, _c_int, _c_void_p, _c_void_p]),
    "mla_project_out": (_c_int, [_c_void_p, _c_void_p, _c_void_p, _c_int, _c_int, _c_void_p, _c_void_p]),
    "mla_decode_cascade": (_c_int, [_c_void_p, _c_void_p, ctypes.c_int64, _c_int, _c_void_p, _c_void_p, _c_int,
                                    _c_void_p, _c_void_p, _c_int, _c_int, _c_int, _c_int, _c_float, _c_void_p,
                                    ctypes.POINTER(_c_size_t), _c_void_p]),
    "mla_get_last_error": (ctypes.c_char_p, []),
    "mla_read_device_flag": (_c_int, [_c_void_p, ctypes.POINTER(_c_int), _c_void_p]),
    "mla_set_wait_timeout_ns": (_c_int, [ctypes.c_uint64]),
    "mla_version": (ctypes.c_char_p, []),
}

_lock = threading.Lock()
_lib = None


class MlaError(RuntimeError):
    def __init__(self, status: int, message: str):
        self.status = status
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")


def load() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build it with `python -m mla_paged_kv_05_b200.build` "
                    "(there is no non-CUDA fallback)")
            lib = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def check(status: int) -> None:
    if status != MLA_OK:
        msg = load().mla_get_last_error().decode(errors="replace")
        raise MlaError(status, msg)

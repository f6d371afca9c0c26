"""ctypes view of libdsc.so (the C ABI declared in include/dsc.h).

Loading fails loudly when the library has not been built: there is no
fallback implementation of any entry point.
"""

from __future__ import annotations

import ctypes as C
import os
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libdsc.so")

DSC_OK, DSC_ERR_INVALID_ARG, DSC_ERR_UNSUPPORTED, DSC_ERR_MISALIGNED, DSC_ERR_CUDA, DSC_ERR_TIMEOUT = range(6)
DSC_F32, DSC_BF16 = 0, 1


class DscError(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn}: {msg} (status {status})")
        self.status = status


class DscProblem(C.Structure):
    _fields_ = [("B", C.c_int64), ("T", C.c_int64), ("D", C.c_int64), ("W", C.c_int64),
                ("H", C.c_int64), ("R", C.c_int64), ("dtype", C.c_int32), ("residual", C.c_int32)]


_P = C.POINTER(DscProblem)
_v = C.c_void_p
_SIGS = {
    "dsc_fwd_headwise": (C.c_int, [_P, _v, _v, _v, _v]),
    "dsc_bwd_headwise": (C.c_int, [_P, _v, _v, _v, _v, _v, _v]),
    "dsc_fwd_lowrank_workspace_bytes": (C.c_size_t, [_P]),
    "dsc_bwd_lowrank_workspace_bytes": (C.c_size_t, [_P]),
    "dsc_lowrank_kernels": (C.c_int, [_P, C.c_int]),
    "dsc_decode_headwise": (C.c_int, [_P, _v, _v, _v, _v, _v]),
    "dsc_decode_static": (C.c_int, [_P, _v, _v, _v, _v, _v]),
    "dsc_decode_lowrank_workspace_bytes": (C.c_size_t, [_P]),
    "dsc_decode_lowrank": (C.c_int, [_P, _v, _v, _v, _v, _v, _v, C.c_size_t, _v]),
    "dsc_decode_state": (C.c_int, [_P, _v, _v, _v]),
    "dsc_fwd_lowrank": (C.c_int, [_P, _v, _v, _v, _v, _v, C.c_size_t, _v]),
    "dsc_bwd_lowrank": (C.c_int, [_P, _v, _v, _v, _v, _v, _v, _v, _v, C.c_size_t, _v]),
    "dsc_fwd_static": (C.c_int, [_P, _v, _v, _v, _v]),
    "dsc_bwd_static_workspace_bytes": (C.c_size_t, [_P]),
    "dsc_bwd_static": (C.c_int, [_P, _v, _v, _v, _v, _v, _v, C.c_size_t, _v]),
    "dsc_bwd_static_noalloc": (C.c_int, [_P, _v, _v, _v, _v, _v, _v]),
    "dsc_fwd_headwise_varlen": (C.c_int, [_P, _v, C.c_int64, _v, _v, _v, _v]),
    "dsc_bwd_headwise_varlen": (C.c_int, [_P, _v, C.c_int64, _v, _v, _v, _v, _v, _v]),
    "dsc_fwd_lowrank_varlen": (C.c_int, [_P, _v, C.c_int64, _v, _v, _v, _v, _v, C.c_size_t, _v]),
    "dsc_bwd_lowrank_varlen_workspace_bytes": (C.c_size_t, [_P, C.c_int64]),
    "dsc_bwd_lowrank_varlen": (C.c_int, [_P, _v, C.c_int64, _v, _v, _v, _v, _v, _v, _v, _v, C.c_size_t, _v]),
    "dsc_fwd_static_varlen": (C.c_int, [_P, _v, C.c_int64, _v, _v, _v, _v]),
    "dsc_bwd_static_varlen": (C.c_int, [_P, _v, C.c_int64, _v, _v, _v, _v, _v, _v, C.c_size_t, _v]),
    "dsc_fwd_headwise_chunk": (C.c_int, [_P, _v, _v, _v, _v, C.c_int, _v]),
    "dsc_bwd_headwise_chunk": (C.c_int, [_P, _v, _v, _v, _v, _v, _v, _v, _v, C.c_int, _v]),
    "dsc_fwd_lowrank_chunk": (C.c_int, [_P, _v, _v, _v, _v, _v, _v, C.c_size_t, C.c_int, _v]),
    "dsc_bwd_lowrank_chunk_workspace_bytes": (C.c_size_t, [_P]),
    "dsc_bwd_lowrank_chunk": (C.c_int, [_P, _v, _v, _v, _v, _v, _v, _v, _v, _v, _v, _v, C.c_size_t, C.c_int, _v]),
    "dsc_fwd_static_chunk": (C.c_int, [_P, _v, _v, _v, _v, C.c_int, _v]),
    "dsc_bwd_static_chunk": (C.c_int, [_P, _v, _v, _v, _v, _v, _v, _v, _v, C.c_size_t, C.c_int, _v]),
    "dsc_fwd_lowrank_proj_workspace_bytes": (C.c_size_t, [_P, C.c_int64]),
    "dsc_fwd_lowrank_proj": (C.c_int, [_P, C.c_int64, _v, _v, _v, _v, _v, _v, _v, C.c_size_t, _v]),
    "dsc_bwd_lowrank_proj_workspace_bytes": (C.c_size_t, [_P, C.c_int64]),
    "dsc_bwd_lowrank_proj": (C.c_int, [_P, C.c_int64, _v, _v, _v, _v, _v, _v, _v, _v, _v, _v, _v, C.c_size_t, _v]),
    "dsc_check": (C.c_int, [_v]),
    "dsc_selftest_timeout": (C.c_int, [_v]),
    "dsc_status_string": (C.c_char_p, [C.c_int]),
    "dsc_version": (C.c_int, []),
    "dsc_launch_count": (C.c_uint64, []),
}

_lock = threading.Lock()
_lib = None


def lib():
    """The loaded library (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(f"{LIB_PATH} is missing: build it with `python -m input_dependent_short_b200.build`")
            L = C.CDLL(LIB_PATH)
            for name, (res, args) in _SIGS.items():
                f = getattr(L, name)
                f.restype = res
                f.argtypes = args
            _lib = L
    return _lib


def status_string(s: int) -> str:
    return lib().dsc_status_string(s).decode()


def call(name: str, *args) -> int:
    """Call an entry point and raise DscError unless it returns DSC_OK."""
    s = getattr(lib(), name)(*args)
    if s != DSC_OK:
        raise DscError(name, s, status_string(s))
    return s

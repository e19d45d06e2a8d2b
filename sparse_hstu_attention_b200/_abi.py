"""ctypes view of include/hstu_sla.h (argument marshalling only)."""
from __future__ import annotations

import ctypes
import os
import re

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libhstu_sla.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "hstu_sla.h")

OK = 0
ERR_INVALID_ARG = -1
ERR_UNSUPPORTED = -2
ERR_CUDA = -3
ERR_BAD_INPUT = -4
ERR_WORKSPACE = -5
ERR_TIMEOUT = -6

WS_FWD = 0
WS_BWD = 1


class FwdParams(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int32), ("H", ctypes.c_int32), ("d", ctypes.c_int32),
        ("total_tokens", ctypes.c_int64), ("max_seq_len", ctypes.c_int32),
        ("seq_offsets", ctypes.c_void_p), ("num_targets", ctypes.c_void_p),
        ("contextual_len", ctypes.c_int32), ("K1", ctypes.c_int32), ("K2", ctypes.c_int32),
        ("alpha", ctypes.c_float), ("N", ctypes.c_float),
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("q_row_stride", ctypes.c_int64), ("k_row_stride", ctypes.c_int64),
        ("v_row_stride", ctypes.c_int64),
        ("out", ctypes.c_void_p), ("out_row_stride", ctypes.c_int64),
        ("event_begin", ctypes.c_void_p), ("event_end", ctypes.c_void_p),
    ]


class BwdParams(ctypes.Structure):
    _fields_ = [
        ("fwd", FwdParams),
        ("dout", ctypes.c_void_p), ("dout_row_stride", ctypes.c_int64),
        ("dq", ctypes.c_void_p), ("dk", ctypes.c_void_p), ("dv", ctypes.c_void_p),
        ("dq_row_stride", ctypes.c_int64), ("dk_row_stride", ctypes.c_int64),
        ("dv_row_stride", ctypes.c_int64),
    ]


_lib = None


class LibraryMissing(RuntimeError):
    pass


def load():
    """Load libhstu_sla.so; raise if it has not been built (there is no fallback)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise LibraryMissing(
            f"{LIB_PATH} is missing: build it with `python -m sparse_hstu_attention_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    vp, sz = ctypes.c_void_p, ctypes.c_size_t
    lib.hstu_sla_workspace_bytes.argtypes = [ctypes.c_int, ctypes.c_int64, ctypes.c_int32,
                                             ctypes.c_int32, ctypes.c_int32]
    lib.hstu_sla_workspace_bytes.restype = sz
    lib.hstu_sla_fwd.argtypes = [ctypes.POINTER(FwdParams), vp, sz, vp]
    lib.hstu_sla_fwd.restype = ctypes.c_int
    lib.hstu_sla_bwd.argtypes = [ctypes.POINTER(BwdParams), vp, sz, vp]
    lib.hstu_sla_bwd.restype = ctypes.c_int
    lib.hstu_sla_fwd_noalloc.argtypes = [ctypes.POINTER(FwdParams), vp]
    lib.hstu_sla_fwd_noalloc.restype = ctypes.c_int
    lib.hstu_sla_count_pairs.argtypes = [ctypes.POINTER(FwdParams), vp, vp, vp, sz, vp]
    lib.hstu_sla_count_pairs.restype = ctypes.c_int
    lib.hstu_sla_get_error.argtypes = [vp, vp]
    lib.hstu_sla_get_error.restype = ctypes.c_int
    lib.hstu_sla_strerror.argtypes = [ctypes.c_int]
    lib.hstu_sla_strerror.restype = ctypes.c_char_p
    lib.hstu_sla_version.argtypes = []
    lib.hstu_sla_version.restype = ctypes.c_int
    _lib = lib
    return lib


def declared_functions():
    """Names of the functions include/hstu_sla.h declares."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(hstu_\w+)\s*\(", text)))


def strerror(code: int) -> str:
    return load().hstu_sla_strerror(code).decode()

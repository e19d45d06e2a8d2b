"""ctypes view of include/hstu_sla.h (argument marshalling only)."""
from __future__ import annotations

import ctypes
import os
import re

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libhstu_sla.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "hstu_sla.h")
INCLUDE_DIR = os.path.join(os.path.dirname(PKG), "include")
HEADERS = [HEADER, os.path.join(INCLUDE_DIR, "hstu_stu.h")]

OK = 0
ERR_INVALID_ARG = -1
ERR_UNSUPPORTED = -2
ERR_CUDA = -3
ERR_BAD_INPUT = -4
ERR_WORKSPACE = -5
ERR_TIMEOUT = -6

WS_FWD = 0
WS_BWD = 1
MAX_GROUPS = 4   # HSTU_SLA_MAX_GROUPS
WS_FWD_FP8 = 2   # hstu_stu_workspace_bytes only: the layer forward with fp8 = 1
WS_FWD_REMAT = 3  # hstu_stu_workspace_bytes only: the layer forward with remat = 1
WS_BWD_REMAT = 4  # hstu_stu_workspace_bytes only: the layer backward with remat = 1


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
        ("candidates_only", ctypes.c_int32),
        ("timestamps", ctypes.c_void_p), ("rab_pos", ctypes.c_void_p),
        ("rab_time", ctypes.c_void_p), ("rab_pos_buckets", ctypes.c_int32),
        ("rab_time_buckets", ctypes.c_int32),
    ]


class BwdParams(ctypes.Structure):
    _fields_ = [
        ("fwd", FwdParams),
        ("dout", ctypes.c_void_p), ("dout_row_stride", ctypes.c_int64),
        ("dq", ctypes.c_void_p), ("dk", ctypes.c_void_p), ("dv", ctypes.c_void_p),
        ("dq_row_stride", ctypes.c_int64), ("dk_row_stride", ctypes.c_int64),
        ("dv_row_stride", ctypes.c_int64),
        ("d_rab_pos", ctypes.c_void_p), ("d_rab_time", ctypes.c_void_p),
        ("prepared", ctypes.c_int32),
    ]


class StuLayerParams(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int32), ("H", ctypes.c_int32), ("d", ctypes.c_int32),
        ("total_tokens", ctypes.c_int64), ("max_seq_len", ctypes.c_int32),
        ("seq_offsets", ctypes.c_void_p), ("num_targets", ctypes.c_void_p),
        ("contextual_len", ctypes.c_int32), ("K1", ctypes.c_int32), ("K2", ctypes.c_int32),
        ("alpha", ctypes.c_float), ("N", ctypes.c_float), ("ln_eps", ctypes.c_float),
        ("ln1_w", ctypes.c_void_p), ("ln1_b", ctypes.c_void_p), ("w1", ctypes.c_void_p),
        ("b1", ctypes.c_void_p), ("ln2_w", ctypes.c_void_p), ("ln2_b", ctypes.c_void_p),
        ("w2", ctypes.c_void_p), ("b2", ctypes.c_void_p),
        ("x", ctypes.c_void_p), ("out", ctypes.c_void_p),
        ("xn", ctypes.c_void_p), ("pre", ctypes.c_void_p), ("uvqk", ctypes.c_void_p),
        ("av", ctypes.c_void_p), ("y", ctypes.c_void_p), ("stats", ctypes.c_void_p),
        ("fp8", ctypes.c_int32), ("w1q", ctypes.c_void_p), ("w1s", ctypes.c_void_p),
        ("w2q", ctypes.c_void_p), ("w2s", ctypes.c_void_p),
        ("remat", ctypes.c_int32), ("u", ctypes.c_void_p),
    ]


class StuLayerBwdParams(ctypes.Structure):
    _fields_ = [
        ("fwd", StuLayerParams),
        ("dout", ctypes.c_void_p), ("dx", ctypes.c_void_p),
        ("dy", ctypes.c_void_p), ("dav", ctypes.c_void_p), ("dpre", ctypes.c_void_p),
        ("dxn", ctypes.c_void_p),
        ("d_ln1_w", ctypes.c_void_p), ("d_ln1_b", ctypes.c_void_p), ("d_w1", ctypes.c_void_p),
        ("d_b1", ctypes.c_void_p), ("d_ln2_w", ctypes.c_void_p), ("d_ln2_b", ctypes.c_void_p),
        ("d_w2", ctypes.c_void_p), ("d_b2", ctypes.c_void_p),
    ]


GEMM_STORE, GEMM_BIAS_SILU, GEMM_BIAS_RESID, GEMM_RED_F32 = 0, 1, 2, 3


class GemmParams(ctypes.Structure):
    _fields_ = [
        ("M", ctypes.c_int32), ("N", ctypes.c_int32), ("K", ctypes.c_int32),
        ("a", ctypes.c_void_p), ("lda", ctypes.c_int64), ("a_mn_major", ctypes.c_int32),
        ("b", ctypes.c_void_p), ("ldb", ctypes.c_int64), ("b_mn_major", ctypes.c_int32),
        ("epilogue", ctypes.c_int32), ("splits", ctypes.c_int32),
        ("bias", ctypes.c_void_p), ("resid", ctypes.c_void_p), ("ldr", ctypes.c_int64),
        ("out", ctypes.c_void_p), ("ldo", ctypes.c_int64),
        ("out2", ctypes.c_void_p), ("ldo2", ctypes.c_int64),
        ("outf", ctypes.c_void_p), ("ldf", ctypes.c_int64),
        ("fp8", ctypes.c_int32), ("a_scale", ctypes.c_void_p), ("b_scale", ctypes.c_void_p),
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
    lib.hstu_sla_noalloc_get_error.argtypes = [vp]
    lib.hstu_sla_noalloc_get_error.restype = ctypes.c_int
    lib.hstu_sla_count_pairs.argtypes = [ctypes.POINTER(FwdParams), vp, vp, vp, sz, vp]
    lib.hstu_sla_count_pairs.restype = ctypes.c_int
    lib.hstu_sla_grouped_workspace_bytes.argtypes = [ctypes.c_int, ctypes.c_int32, vp, vp, vp,
                                                     vp]
    lib.hstu_sla_grouped_workspace_bytes.restype = sz
    lib.hstu_sla_fwd_grouped.argtypes = [ctypes.POINTER(FwdParams), ctypes.c_int32, vp, sz, vp]
    lib.hstu_sla_fwd_grouped.restype = ctypes.c_int
    lib.hstu_sla_bwd_prepare.argtypes = [ctypes.POINTER(BwdParams), vp, sz, vp]
    lib.hstu_sla_bwd_prepare.restype = ctypes.c_int
    lib.hstu_sla_bwd_grouped.argtypes = [ctypes.POINTER(BwdParams), ctypes.c_int32, vp, sz, vp]
    lib.hstu_sla_bwd_grouped.restype = ctypes.c_int
    lib.hstu_sla_test_wait_timeout.argtypes = [ctypes.POINTER(BwdParams), ctypes.c_int32,
                                               ctypes.c_int64, vp, sz, vp]
    lib.hstu_sla_test_wait_timeout.restype = ctypes.c_int
    lib.hstu_sla_get_error.argtypes = [vp, vp]
    lib.hstu_sla_get_error.restype = ctypes.c_int
    lib.hstu_sla_strerror.argtypes = [ctypes.c_int]
    lib.hstu_sla_strerror.restype = ctypes.c_char_p
    lib.hstu_sla_version.argtypes = []
    lib.hstu_sla_version.restype = ctypes.c_int
    i32, i64 = ctypes.c_int32, ctypes.c_int64
    lib.hstu_stu_workspace_bytes.argtypes = [ctypes.c_int, i64, i32, i32, i32]
    lib.hstu_stu_workspace_bytes.restype = sz
    lib.hstu_stu_layer_fwd.argtypes = [ctypes.POINTER(StuLayerParams), vp, sz, vp]
    lib.hstu_stu_layer_fwd.restype = ctypes.c_int
    lib.hstu_stu_layer_bwd.argtypes = [ctypes.POINTER(StuLayerBwdParams), vp, sz, vp]
    lib.hstu_stu_layer_bwd.restype = ctypes.c_int
    lib.hstu_stu_get_error.argtypes = [vp, vp]
    lib.hstu_stu_get_error.restype = ctypes.c_int
    lib.hstu_jagged_truncate_offsets.argtypes = [vp, vp, i32, i32, i32, vp, vp]
    lib.hstu_jagged_truncate_offsets.restype = ctypes.c_int
    lib.hstu_jagged_truncate_lengths.argtypes = [vp, vp, i32, i32, i32, vp]
    lib.hstu_jagged_truncate_lengths.restype = ctypes.c_int64
    lib.hstu_jagged_truncate.argtypes = [vp, i64, vp, vp, vp, i32, i32, i32, i32, vp, i64, i64,
                                         i32, vp]
    lib.hstu_jagged_truncate.restype = ctypes.c_int
    lib.hstu_gemm.argtypes = [ctypes.POINTER(GemmParams), vp, vp]
    lib.hstu_gemm.restype = ctypes.c_int
    lib.hstu_quant_weight_e4m3.argtypes = [vp, i64, i32, i32, vp, i64, vp, vp]
    lib.hstu_quant_weight_e4m3.restype = ctypes.c_int
    _lib = lib
    return lib


def declared_functions():
    """Names of the functions include/hstu_sla.h and include/hstu_stu.h declare."""
    names = set()
    for h in HEADERS:
        text = re.sub(r"/\*.*?\*/", "", open(h).read(), flags=re.S)
        names.update(re.findall(r"\b(hstu_\w+)\s*\(", text))
    return sorted(names)


def strerror(code: int) -> str:
    return load().hstu_sla_strerror(code).decode()

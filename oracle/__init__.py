"""CPU oracle for SLA HSTU attention -- TEST INFRASTRUCTURE ONLY.

Only the tests, the package's ``smoke()`` check and the benchmark's
CPU-baseline leg may import this package.  The product (the CUDA library and
its binding) never imports it and shares no code with it.

The arithmetic lives in ``hstu_sla_oracle.c`` (plain fp64 loops over every
key of every sequence, gated by the SLA mask predicate); this module only
compiles it with gcc and marshals numpy arrays.  ``stu.py`` holds the STU-layer
oracle (LayerNorm, linear, SiLU, gated norm, truncation) in plain numpy.

Parity pins (tests/test_oracle_pins.py) tie it to the cited definitions: a dense
brute-force masked attention built from the mask's definition, the full-causal
special case, the closed-form per-row pair counts, the K1 = 0 and K2 = 0
cases, the M-FALCON mask figure, finite differences and invariants.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hstu_sla_oracle.c")
_LIB = os.path.join(_HERE, "liboracle_hstu_sla.so")

INCLUSIVE_WINDOW = 1
UNCLAMPED_TARGETS = 2

_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle (gcc, OpenMP, no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-std=c99", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
               "-shared", "-fPIC", _SRC, "-o", _LIB + ".tmp", "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


class _Cfg(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("d", ctypes.c_int),
                ("offsets", ctypes.c_void_p), ("num_targets", ctypes.c_void_p),
                ("contextual_len", ctypes.c_int64), ("K1", ctypes.c_int64),
                ("K2", ctypes.c_int64), ("alpha", ctypes.c_double), ("N", ctypes.c_double),
                ("flags", ctypes.c_int), ("ts", ctypes.c_void_p),
                ("rab_pos", ctypes.c_void_p), ("n_pos", ctypes.c_int64),
                ("rab_time", ctypes.c_void_p), ("n_time", ctypes.c_int64)]


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            i64, vp = ctypes.c_int64, ctypes.c_void_p
            lib.oracle_sla_visible.argtypes = [i64] * 7 + [ctypes.c_int]
            lib.oracle_sla_visible.restype = ctypes.c_int
            lib.oracle_sla_row_counts.argtypes = [vp, vp]
            lib.oracle_sla_key_counts.argtypes = [vp, vp]
            lib.oracle_sla_fwd_rows.argtypes = [vp, vp, vp, vp, vp, i64, vp]
            lib.oracle_sla_bwd_dq_rows.argtypes = [vp, vp, vp, vp, vp, vp, i64, vp]
            lib.oracle_sla_bwd_dkv_keys.argtypes = [vp, vp, vp, vp, vp, vp, i64, vp, vp]
            lib.oracle_sla_bwd_drab.argtypes = [vp, vp, vp, vp, vp, vp, vp]
            lib.oracle_rab_bucket.argtypes = [i64, i64]
            lib.oracle_rab_bucket.restype = i64
            for f in ("oracle_sla_row_counts", "oracle_sla_key_counts", "oracle_sla_fwd_rows",
                      "oracle_sla_bwd_dq_rows", "oracle_sla_bwd_dkv_keys", "oracle_sla_bwd_drab"):
                getattr(lib, f).restype = None
            _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


class Problem:
    """One jagged SLA attention problem: offsets, targets, window sizes, scales."""

    def __init__(self, seq_offsets, num_targets, H, d, contextual_len, K1, K2,
                 alpha, N, flags=0, timestamps=None, rab_pos=None, rab_time=None):
        """rab_pos [H][n_pos], rab_time [H][n_time] and timestamps [T]: the
        optional relative attention bias (rab_time needs timestamps)."""
        self.offsets = np.ascontiguousarray(np.asarray(seq_offsets, dtype=np.int64))
        B = len(self.offsets) - 1
        nt = np.zeros(B, np.int64) if num_targets is None else num_targets
        self.num_targets = np.ascontiguousarray(np.asarray(nt, dtype=np.int64))
        keep = lambda a, dt: None if a is None else np.ascontiguousarray(np.asarray(a, dtype=dt))
        self.ts = keep(timestamps, np.int64)
        self.rab_pos = keep(rab_pos, np.float64)
        self.rab_time = keep(rab_time, np.float64)
        ptr = lambda a: None if a is None else a.ctypes.data
        self._cfg = _Cfg(B, H, d, self.offsets.ctypes.data, self.num_targets.ctypes.data,
                         contextual_len, K1, K2, float(alpha), float(N), flags,
                         ptr(self.ts), ptr(self.rab_pos),
                         0 if self.rab_pos is None else self.rab_pos.shape[1],
                         ptr(self.rab_time),
                         0 if self.rab_time is None else self.rab_time.shape[1])
        self.B, self.H, self.d = B, H, d
        self.T = int(self.offsets[-1])

    @classmethod
    def from_batch(cls, batch, flags=0, **override):
        w = batch.workload
        kw = dict(H=w.H, d=w.d, contextual_len=w.contextual_len, K1=w.K1, K2=w.K2,
                  alpha=w.alpha, N=w.N)
        kw.update(override)
        return cls(batch.seq_offsets, batch.num_targets, flags=flags, **kw)

    def _idx(self, idx):
        if idx is None:
            idx = np.arange(self.T, dtype=np.int64)
        return np.ascontiguousarray(np.asarray(idx, dtype=np.int64))

    def row_counts(self) -> np.ndarray:
        out = np.zeros(self.T, np.int64)
        _load().oracle_sla_row_counts(ctypes.byref(self._cfg), out.ctypes.data)
        return out

    def key_counts(self) -> np.ndarray:
        out = np.zeros(self.T, np.int64)
        _load().oracle_sla_key_counts(ctypes.byref(self._cfg), out.ctypes.data)
        return out

    def fwd(self, q, k, v, rows=None) -> np.ndarray:
        q, k, v = _f64(q), _f64(k), _f64(v)
        rows = self._idx(rows)
        out = np.zeros((len(rows), self.H, self.d), np.float64)
        _load().oracle_sla_fwd_rows(ctypes.byref(self._cfg), q.ctypes.data, k.ctypes.data,
                                    v.ctypes.data, rows.ctypes.data, len(rows),
                                    out.ctypes.data)
        return out

    def bwd_dq(self, q, k, v, dout, rows=None) -> np.ndarray:
        q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
        rows = self._idx(rows)
        dq = np.zeros((len(rows), self.H, self.d), np.float64)
        _load().oracle_sla_bwd_dq_rows(ctypes.byref(self._cfg), q.ctypes.data, k.ctypes.data,
                                       v.ctypes.data, dout.ctypes.data, rows.ctypes.data,
                                       len(rows), dq.ctypes.data)
        return dq

    def bwd_dkv(self, q, k, v, dout, keys=None):
        q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
        keys = self._idx(keys)
        dk = np.zeros((len(keys), self.H, self.d), np.float64)
        dv = np.zeros_like(dk)
        _load().oracle_sla_bwd_dkv_keys(ctypes.byref(self._cfg), q.ctypes.data, k.ctypes.data,
                                        v.ctypes.data, dout.ctypes.data, keys.ctypes.data,
                                        len(keys), dk.ctypes.data, dv.ctypes.data)
        return dk, dv

    def bwd(self, q, k, v, dout):
        dq = self.bwd_dq(q, k, v, dout)
        dk, dv = self.bwd_dkv(q, k, v, dout)
        return dq, dk, dv

    def bwd_rab(self, q, k, v, dout):
        """Gradients of the bias tables (None for an absent table)."""
        q, k, v, dout = _f64(q), _f64(k), _f64(v), _f64(dout)
        dp = None if self.rab_pos is None else np.zeros_like(self.rab_pos)
        dt = None if self.rab_time is None else np.zeros_like(self.rab_time)
        _load().oracle_sla_bwd_drab(ctypes.byref(self._cfg), q.ctypes.data, k.ctypes.data,
                                    v.ctypes.data, dout.ctypes.data,
                                    None if dp is None else dp.ctypes.data,
                                    None if dt is None else dt.ctypes.data)
        return dp, dt


def rab_bucket(n: int, nb: int) -> int:
    """The oracle's bucket of a non-negative distance n (tables of nb rows)."""
    return int(_load().oracle_rab_bucket(int(n), int(nb)))


def visible(L, nt, contextual_len, K1, K2, i, j, flags=0) -> int:
    """The mask predicate M(i, j) of one sequence (0-based positions)."""
    return _load().oracle_sla_visible(L, nt, contextual_len, K1, K2, i, j, flags)


def mask_matrix(L, nt, contextual_len, K1, K2, flags=0) -> np.ndarray:
    """The L x L mask, evaluated point by point through the predicate."""
    lib = _load()
    return np.array([[lib.oracle_sla_visible(L, nt, contextual_len, K1, K2, i, j, flags)
                      for j in range(L)] for i in range(L)], dtype=np.int64)

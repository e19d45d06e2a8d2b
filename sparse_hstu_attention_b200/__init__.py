"""SLA HSTU attention on B200 (sm_100a).

A thin binding over the C ABI of ``libhstu_sla.so`` (include/hstu_sla.h):
every step of the attention runs in the library's CUDA kernels; this module
only checks tensor shapes, allocates outputs / workspace with PyTorch and
marshals pointers.  There is no CPU or PyTorch fallback: if the library is
missing, the calls raise.

    out = hstu_sla_fwd(q, k, v, seq_offsets, num_targets, contextual_len=32,
                       K1=1024, K2=128, alpha=128 ** -0.5, N=16384.0)
    dq, dk, dv = hstu_sla_bwd(dout, q, k, v, seq_offsets, num_targets, ...)

q, k, v, dout: CUDA bf16 tensors [T, H, d] whose last two dims are dense
(row stride free, so views into a fused [T, 4*H*d] projection work);
seq_offsets: CUDA int32 [B+1]; num_targets: CUDA int32 [B] or None.

Options of the same calls: candidates_only=True (M-FALCON candidate scoring,
forward); timestamps / rab_pos / rab_time (relative attention bias; the
backward then also returns the tables' gradients).  Several problems (e.g.
Mixture-of-Transducers channels) run in one launch through
hstu_sla_fwd_grouped / hstu_sla_bwd_grouped.  The STU layer, the truncated
stack and the FP8 projections are in the ``stu`` module.
"""
from __future__ import annotations

import ctypes
from typing import Optional

import numpy as np
import torch

from . import _abi
from ._abi import LibraryMissing  # noqa: F401

__all__ = ["hstu_sla_fwd", "hstu_sla_bwd_prepare", "hstu_sla_fwd_noalloc", "hstu_sla_noalloc_get_error", "hstu_sla_bwd", "hstu_sla_workspace_bytes",
           "hstu_sla_count_pairs", "hstu_sla_fwd_grouped", "hstu_sla_bwd_grouped",
           "hstu_sla_grouped_workspace_bytes", "hstu_sla_get_error", "hstu_sla_strerror",
           "SLAError", "SLAAttention", "sla_attention"]


class SLAError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {hstu_sla_strerror(code)} (status {code})")


def hstu_sla_strerror(code: int) -> str:
    return _abi.strerror(code)


def _check(code: int, where: str):
    if code != _abi.OK:
        raise SLAError(code, where)


def _stream_ptr(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return int(s.cuda_stream)


def _row_stride(t: torch.Tensor, name: str, H: int, d: int) -> int:
    if t.dtype != torch.bfloat16 or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA bfloat16 tensor")
    if t.dim() != 3 or t.shape[1] != H or t.shape[2] != d:
        raise ValueError(f"{name} must be [T, {H}, {d}], got {tuple(t.shape)}")
    if t.stride(2) != 1 or t.stride(1) != d:
        raise ValueError(f"{name}: heads and head_dim must be dense (stride (*, {d}, 1))")
    return t.stride(0)


def hstu_sla_workspace_bytes(which: int, total_tokens: int, B: int, H: int, d: int) -> int:
    return int(_abi.load().hstu_sla_workspace_bytes(which, total_tokens, B, H, d))


def _set_rab(p, H, timestamps, rab_pos, rab_time):
    """Relative attention bias fields: timestamps CUDA int32 [T]; rab_pos /
    rab_time CUDA float32 [H, buckets] (1..32 buckets), either may be None."""
    for name, t in (("rab_pos", rab_pos), ("rab_time", rab_time)):
        if t is not None and (t.dtype != torch.float32 or not t.is_cuda or t.dim() != 2 or
                              t.shape[0] != H or not t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous CUDA float32 [{H}, buckets] tensor")
    if timestamps is not None and (timestamps.dtype != torch.int32 or not timestamps.is_cuda):
        raise TypeError("timestamps must be a CUDA int32 tensor [T]")
    p.timestamps = timestamps.data_ptr() if timestamps is not None else None
    if rab_pos is not None:
        p.rab_pos, p.rab_pos_buckets = rab_pos.data_ptr(), rab_pos.shape[1]
    if rab_time is not None:
        p.rab_time, p.rab_time_buckets = rab_time.data_ptr(), rab_time.shape[1]


def _fwd_params(q, k, v, seq_offsets, num_targets, contextual_len, K1, K2, alpha, N,
                max_seq_len, events=None, candidates_only=False) -> _abi.FwdParams:
    T, H, d = q.shape
    if seq_offsets.dtype != torch.int32 or not seq_offsets.is_cuda:
        raise TypeError("seq_offsets must be a CUDA int32 tensor [B+1]")
    if num_targets is not None and (num_targets.dtype != torch.int32 or not num_targets.is_cuda):
        raise TypeError("num_targets must be a CUDA int32 tensor [B] or None")
    B = seq_offsets.numel() - 1
    p = _abi.FwdParams()
    p.B, p.H, p.d = B, H, d
    p.total_tokens = T
    p.max_seq_len = T if max_seq_len is None else int(max_seq_len)
    p.seq_offsets = seq_offsets.data_ptr()
    p.num_targets = num_targets.data_ptr() if num_targets is not None else None
    p.contextual_len, p.K1, p.K2 = int(contextual_len), int(K1), int(K2)
    p.alpha, p.N = float(alpha), float(N)
    p.q, p.k, p.v = q.data_ptr(), k.data_ptr(), v.data_ptr()
    p.q_row_stride = _row_stride(q, "q", H, d)
    p.k_row_stride = _row_stride(k, "k", H, d)
    p.v_row_stride = _row_stride(v, "v", H, d)
    if k.shape[0] != T or v.shape[0] != T:
        raise ValueError("q, k, v must have the same number of tokens")
    if events is not None:
        p.event_begin = events[0].cuda_event
        p.event_end = events[1].cuda_event
    p.candidates_only = int(bool(candidates_only))
    return p


def _workspace(which, T, B, H, d, device, workspace):
    need = hstu_sla_workspace_bytes(which, T, B, H, d)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=device)
    if workspace.numel() < need:
        raise ValueError(f"workspace too small: {workspace.numel()} < {need} bytes")
    return workspace


def hstu_sla_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, seq_offsets: torch.Tensor,
                 num_targets: Optional[torch.Tensor], *, contextual_len: int, K1: int, K2: int,
                 alpha: float, N: float, max_seq_len: Optional[int] = None,
                 out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                 stream=None, events=None, candidates_only: bool = False,
                 timestamps=None, rab_pos=None, rab_time=None) -> torch.Tensor:
    """SLA HSTU attention forward; returns out [T, H, d] (bf16).  `events`: an
    optional pair of torch.cuda.Event recorded around the attention kernel.
    candidates_only: M-FALCON scoring, only the query tiles that hold
    candidates are computed (other rows of `out` are left as they were).
    timestamps / rab_pos / rab_time: the optional relative attention bias
    (include/hstu_sla.h)."""
    lib = _abi.load()
    p = _fwd_params(q, k, v, seq_offsets, num_targets, contextual_len, K1, K2, alpha, N,
                    max_seq_len, events, candidates_only)
    _set_rab(p, q.shape[1], timestamps, rab_pos, rab_time)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device)
    p.out = out.data_ptr()
    p.out_row_stride = _row_stride(out, "out", p.H, p.d)
    ws = _workspace(_abi.WS_FWD, p.total_tokens, p.B, p.H, p.d, q.device, workspace)
    _check(lib.hstu_sla_fwd(ctypes.byref(p), ws.data_ptr(), ws.numel(), _stream_ptr(stream)),
           "hstu_sla_fwd")
    return out


def hstu_sla_fwd_noalloc(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                         seq_offsets: torch.Tensor, num_targets: Optional[torch.Tensor], *,
                         contextual_len: int, K1: int, K2: int, alpha: float, N: float,
                         max_seq_len: Optional[int] = None, out: Optional[torch.Tensor] = None,
                         stream=None, check: bool = True) -> torch.Tensor:
    """The forward through the C entry point that allocates no workspace (for
    callers whose runtime forbids device allocation in the launch path).  The
    library keeps one 2 MiB scratch array per device; overlapping calls race.
    check: synchronise and raise if the device recorded an input error or a
    timed-out wait (out is then unwritten); check=False leaves that to
    hstu_sla_noalloc_get_error."""
    lib = _abi.load()
    p = _fwd_params(q, k, v, seq_offsets, num_targets, contextual_len, K1, K2, alpha, N,
                    max_seq_len)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device)
    p.out = out.data_ptr()
    p.out_row_stride = _row_stride(out, "out", p.H, p.d)
    _check(lib.hstu_sla_fwd_noalloc(ctypes.byref(p), _stream_ptr(stream)), "hstu_sla_fwd_noalloc")
    if check:
        _check(lib.hstu_sla_noalloc_get_error(_stream_ptr(stream)), "hstu_sla_fwd_noalloc (device)")
    return out


def hstu_sla_noalloc_get_error(stream=None) -> int:
    """Synchronise and return the device-side status of the last
    hstu_sla_fwd_noalloc call on the current device."""
    return int(_abi.load().hstu_sla_noalloc_get_error(_stream_ptr(stream)))


def hstu_sla_bwd(dout: torch.Tensor, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                 seq_offsets: torch.Tensor, num_targets: Optional[torch.Tensor], *,
                 contextual_len: int, K1: int, K2: int, alpha: float, N: float,
                 max_seq_len: Optional[int] = None, dq: Optional[torch.Tensor] = None,
                 dk: Optional[torch.Tensor] = None, dv: Optional[torch.Tensor] = None,
                 workspace: Optional[torch.Tensor] = None, stream=None, events=None,
                 timestamps=None, rab_pos=None, rab_time=None, prepared: bool = False):
    """SLA HSTU attention backward; returns (dq, dk, dv) [T, H, d] (bf16), and
    with a relative attention bias (dq, dk, dv, (d_rab_pos, d_rab_time)),
    fp32, None for an absent table.  prepared: hstu_sla_bwd_prepare already
    ran on `workspace` for this batch, ordered before this call."""
    lib = _abi.load()
    p = _abi.BwdParams()
    p.prepared = int(bool(prepared))
    p.fwd = _fwd_params(q, k, v, seq_offsets, num_targets, contextual_len, K1, K2, alpha, N,
                        max_seq_len, events)
    _set_rab(p.fwd, q.shape[1], timestamps, rab_pos, rab_time)
    d_rab = (torch.empty_like(rab_pos) if rab_pos is not None else None,
             torch.empty_like(rab_time) if rab_time is not None else None)
    p.d_rab_pos = d_rab[0].data_ptr() if d_rab[0] is not None else None
    p.d_rab_time = d_rab[1].data_ptr() if d_rab[1] is not None else None
    H, d = p.fwd.H, p.fwd.d
    dq = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device) if dq is None else dq
    dk = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device) if dk is None else dk
    dv = torch.empty(q.shape, dtype=torch.bfloat16, device=q.device) if dv is None else dv
    p.dout, p.dout_row_stride = dout.data_ptr(), _row_stride(dout, "dout", H, d)
    p.dq, p.dq_row_stride = dq.data_ptr(), _row_stride(dq, "dq", H, d)
    p.dk, p.dk_row_stride = dk.data_ptr(), _row_stride(dk, "dk", H, d)
    p.dv, p.dv_row_stride = dv.data_ptr(), _row_stride(dv, "dv", H, d)
    ws = _workspace(_abi.WS_BWD, p.fwd.total_tokens, p.fwd.B, H, d, q.device, workspace)
    _check(lib.hstu_sla_bwd(ctypes.byref(p), ws.data_ptr(), ws.numel(), _stream_ptr(stream)),
           "hstu_sla_bwd")
    if rab_pos is not None or rab_time is not None:
        return dq, dk, dv, d_rab
    return dq, dk, dv


def hstu_sla_bwd_prepare(q: torch.Tensor, seq_offsets: torch.Tensor,
                         num_targets: Optional[torch.Tensor], *, contextual_len: int, K1: int,
                         K2: int, alpha: float, N: float, workspace: torch.Tensor,
                         max_seq_len: Optional[int] = None, stream=None) -> None:
    """The backward's preparation (work lists; the clear of the dQ
    accumulator for head_dim 128) into `workspace`, on `stream`: it reads only
    the batch geometry, so it can run early (e.g. beside the forward).  The
    backward then takes prepared=True and the same workspace."""
    lib = _abi.load()
    p = _abi.BwdParams()
    p.fwd = _fwd_params(q, q, q, seq_offsets, num_targets, contextual_len, K1, K2, alpha, N,
                        max_seq_len)
    H, d = p.fwd.H, p.fwd.d
    rs = _row_stride(q, "q", H, d)
    p.dout = p.dq = p.dk = p.dv = q.data_ptr()  # validated, never read or written
    p.dout_row_stride = p.dq_row_stride = p.dk_row_stride = p.dv_row_stride = rs
    ws = _workspace(_abi.WS_BWD, p.fwd.total_tokens, p.fwd.B, H, d, q.device, workspace)
    _check(lib.hstu_sla_bwd_prepare(ctypes.byref(p), ws.data_ptr(), ws.numel(),
                                    _stream_ptr(stream)), "hstu_sla_bwd_prepare")


def hstu_sla_grouped_workspace_bytes(which: int, problems) -> int:
    """Workspace of a grouped call; problems: (total_tokens, B, H, d) per group."""
    G = len(problems)
    arr = [np.asarray([p[i] for p in problems], dtype=dt)
           for i, dt in enumerate((np.int64, np.int32, np.int32, np.int32))]
    ptrs = [a.ctypes.data for a in arr]
    return int(_abi.load().hstu_sla_grouped_workspace_bytes(which, G, *ptrs))


def _group_params(g: dict, events=None) -> _abi.FwdParams:
    p = _fwd_params(g["q"], g["k"], g["v"], g["seq_offsets"], g.get("num_targets"),
                    g["contextual_len"], g["K1"], g["K2"], g["alpha"], g["N"],
                    g.get("max_seq_len"), events, g.get("candidates_only", False))
    _set_rab(p, g["q"].shape[1], g.get("timestamps"), g.get("rab_pos"), g.get("rab_time"))
    return p


def _grouped_ws(which, params, device, workspace):
    need = hstu_sla_grouped_workspace_bytes(
        which, [(p.total_tokens, p.B, p.H, p.d) for p in params])
    if need == 0:
        raise ValueError("invalid grouped problem sizes")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=device)
    if workspace.numel() < need:
        raise ValueError(f"workspace too small: {workspace.numel()} < {need} bytes")
    return workspace


def hstu_sla_fwd_grouped(groups, *, workspace=None, stream=None, events=None):
    """Several independent SLA forwards (e.g. the channels of a Mixture of
    Transducers) in one launch.  groups: list of dicts with the keyword
    arguments of hstu_sla_fwd plus q, k, v, seq_offsets (num_targets,
    max_seq_len, out, candidates_only, and the relative attention bias's
    timestamps, rab_pos, rab_time optional, per group).  Returns the
    outputs."""
    lib = _abi.load()
    G = len(groups)
    arr = (_abi.FwdParams * G)()
    outs = []
    for i, g in enumerate(groups):
        p = _group_params(g, events if i == 0 else None)
        out = g.get("out")
        if out is None:
            out = torch.empty(g["q"].shape, dtype=torch.bfloat16, device=g["q"].device)
        p.out = out.data_ptr()
        p.out_row_stride = _row_stride(out, "out", p.H, p.d)
        arr[i] = p
        outs.append(out)
    ws = _grouped_ws(_abi.WS_FWD, list(arr), groups[0]["q"].device, workspace)
    _check(lib.hstu_sla_fwd_grouped(arr, G, ws.data_ptr(), ws.numel(), _stream_ptr(stream)),
           "hstu_sla_fwd_grouped")
    return outs


def hstu_sla_bwd_grouped(groups, *, workspace=None, stream=None, events=None):
    """Several independent SLA backwards in one launch (head_dim 128).  groups:
    as for hstu_sla_fwd_grouped plus dout (and optionally preallocated dq, dk,
    dv).  Returns (dq, dk, dv) per group, and
    (dq, dk, dv, (d_rab_pos, d_rab_time)) for a group with a relative
    attention bias."""
    lib = _abi.load()
    G = len(groups)
    arr = (_abi.BwdParams * G)()
    grads = []
    for i, g in enumerate(groups):
        b = _abi.BwdParams()
        b.fwd = _group_params(g, events if i == 0 else None)
        q, H, d = g["q"], b.fwd.H, b.fwd.d
        dq, dk, dv = (g.get(n) if g.get(n) is not None else
                      torch.empty(q.shape, dtype=torch.bfloat16, device=q.device)
                      for n in ("dq", "dk", "dv"))
        b.dout, b.dout_row_stride = g["dout"].data_ptr(), _row_stride(g["dout"], "dout", H, d)
        b.dq, b.dq_row_stride = dq.data_ptr(), _row_stride(dq, "dq", H, d)
        b.dk, b.dk_row_stride = dk.data_ptr(), _row_stride(dk, "dk", H, d)
        b.dv, b.dv_row_stride = dv.data_ptr(), _row_stride(dv, "dv", H, d)
        rp, rt = g.get("rab_pos"), g.get("rab_time")
        d_rab = (torch.empty_like(rp) if rp is not None else None,
                 torch.empty_like(rt) if rt is not None else None)
        b.d_rab_pos = d_rab[0].data_ptr() if d_rab[0] is not None else None
        b.d_rab_time = d_rab[1].data_ptr() if d_rab[1] is not None else None
        arr[i] = b
        grads.append((dq, dk, dv, d_rab) if rp is not None or rt is not None else (dq, dk, dv))
    ws = _grouped_ws(_abi.WS_BWD, [b.fwd for b in arr], groups[0]["q"].device, workspace)
    _check(lib.hstu_sla_bwd_grouped(arr, G, ws.data_ptr(), ws.numel(), _stream_ptr(stream)),
           "hstu_sla_bwd_grouped")
    return grads


def hstu_sla_count_pairs(q, k, v, seq_offsets, num_targets, *, contextual_len, K1, K2,
                         max_seq_len=None, stream=None):
    """Per-token visible-key counts (forward enumeration) and per-token
    seeing-row counts (backward enumeration), int64 [T] each."""
    lib = _abi.load()
    p = _fwd_params(q, k, v, seq_offsets, num_targets, contextual_len, K1, K2, 1.0, 1.0,
                    max_seq_len)
    T = p.total_tokens
    rows = torch.empty(T, dtype=torch.int64, device=q.device)
    keys = torch.empty(T, dtype=torch.int64, device=q.device)
    ws = _workspace(_abi.WS_FWD, T, p.B, p.H, p.d, q.device, None)
    _check(lib.hstu_sla_count_pairs(ctypes.byref(p), rows.data_ptr(), keys.data_ptr(),
                                    ws.data_ptr(), ws.numel(), _stream_ptr(stream)),
           "hstu_sla_count_pairs")
    status = lib.hstu_sla_get_error(ws.data_ptr(), _stream_ptr(stream))
    _check(status, "hstu_sla_count_pairs (device)")
    return rows, keys


def hstu_sla_get_error(workspace: torch.Tensor, stream=None) -> int:
    """Synchronise and return the device-side status stored in `workspace`."""
    return int(_abi.load().hstu_sla_get_error(workspace.data_ptr(), _stream_ptr(stream)))


class SLAAttention(torch.autograd.Function):
    """Autograd wrapper: forward and backward both run in the CUDA library."""

    @staticmethod
    def forward(ctx, q, k, v, seq_offsets, num_targets, contextual_len, K1, K2, alpha, N,
                max_seq_len):
        out = hstu_sla_fwd(q, k, v, seq_offsets, num_targets, contextual_len=contextual_len,
                           K1=K1, K2=K2, alpha=alpha, N=N, max_seq_len=max_seq_len)
        ctx.save_for_backward(q, k, v, seq_offsets,
                              num_targets if num_targets is not None else seq_offsets[:0])
        ctx.has_targets = num_targets is not None
        ctx.cfg = (contextual_len, K1, K2, alpha, N, max_seq_len)
        return out

    @staticmethod
    def backward(ctx, dout):
        q, k, v, offs, nts = ctx.saved_tensors
        c, K1, K2, alpha, N, msl = ctx.cfg
        if dout.stride(2) != 1 or dout.stride(1) != dout.shape[2]:
            dout = dout.contiguous()
        dq, dk, dv = hstu_sla_bwd(dout, q, k, v, offs, nts if ctx.has_targets else None,
                                  contextual_len=c, K1=K1, K2=K2, alpha=alpha, N=N,
                                  max_seq_len=msl)
        return dq, dk, dv, None, None, None, None, None, None, None, None


def sla_attention(q, k, v, seq_offsets, num_targets=None, *, contextual_len=0, K1, K2, alpha,
                  N, max_seq_len=None):
    return SLAAttention.apply(q, k, v, seq_offsets, num_targets, contextual_len, K1, K2, alpha,
                              N, max_seq_len)

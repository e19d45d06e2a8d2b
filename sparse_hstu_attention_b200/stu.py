"""STU layers and the truncated STU stack over the C ABI (include/hstu_stu.h).

Argument marshalling only: every step (LayerNorm, the UVQK and output GEMMs,
SiLU, the SLA attention, the gated norm, truncation and all their backward
passes) runs in the library's CUDA kernels.  PyTorch allocates the buffers.

One layer ("Bending the Scaling Law Curve in Large-Scale Recommendation
Systems", section 3, Eq. 1-5, and Listing 1 of section 4.2.2):

    x^ = LN1(x);  U, V, Q, K = split(SiLU(x^ W1 + b1))
    A = SLA(Q, K, V);  y = LN2(A) * U;  out = y W2 + b2 + x

The stack (section 4.3, attention truncation) runs `trunc_after` layers on
the full sequences, keeps per sequence the contextual prefix, the last `tail`
history tokens and the candidates, and runs the remaining layers on those.
"""
from __future__ import annotations

import ctypes
import dataclasses
from typing import List, Optional

import numpy as np
import torch

from . import _abi


class STUError(RuntimeError):
    pass


def _check(code: int, where: str):
    if code != _abi.OK:
        raise STUError(f"{where}: {_abi.strerror(code)} (status {code})")


def _stream(stream) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return int(s.cuda_stream)


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


@dataclasses.dataclass(frozen=True)
class StuConfig:
    """Attention settings of one layer (N may differ before / after truncation)."""
    H: int
    d: int
    contextual_len: int
    K1: int
    K2: int
    alpha: float
    N: float
    ln_eps: float = 1e-5

    @property
    def d_model(self) -> int:
        return self.H * self.d


@dataclasses.dataclass
class StuWeights:
    """One layer's parameters on the device: LayerNorm affine maps and biases
    fp32, projection matrices bf16 in the x W convention ([in][out])."""
    ln1_w: torch.Tensor
    ln1_b: torch.Tensor
    w1: torch.Tensor   # [d_model, 4 d_model]
    b1: torch.Tensor
    ln2_w: torch.Tensor
    ln2_b: torch.Tensor
    w2: torch.Tensor   # [d_model, d_model]
    b2: torch.Tensor

    @staticmethod
    def from_host(t: dict, device) -> "StuWeights":
        """Move a dict of CPU tensors (names as the fields) to the device:
        projections as bf16, everything else as fp32."""
        def mv(name):
            dt = torch.bfloat16 if name in ("w1", "w2") else torch.float32
            return t[name].to(device=device, dtype=dt).contiguous()
        return StuWeights(*(mv(f.name) for f in dataclasses.fields(StuWeights)))

    def tensors(self):
        """The field tensors themselves, in field order (no copies: their
        device pointers go to the library)."""
        return tuple(getattr(self, f.name) for f in dataclasses.fields(self))


@dataclasses.dataclass
class Fp8Weights:
    """E4M3 copies of a layer's projections for the FP8 forward: W1 and W2
    transposed to [out][in] bytes, with one fp32 scale per output column
    (wq[n][k] * scale[n] ~ W[k][n])."""
    w1q: torch.Tensor  # uint8 [4 d_model, d_model]
    w1s: torch.Tensor  # [4 d_model]
    w2q: torch.Tensor  # uint8 [d_model, d_model]
    w2s: torch.Tensor  # [d_model]


def quantize_weight_e4m3(w: torch.Tensor, stream=None):
    """(wq, scale) for a bf16 [K, N] weight: wq uint8 [N, K] holding E4M3
    bytes, scale [N] = max_k |w[k, n]| / 448 (1 for a zero column)."""
    if w.dtype != torch.bfloat16 or not w.is_cuda or w.dim() != 2 or w.stride(1) != 1:
        raise ValueError("w must be a CUDA bf16 matrix with contiguous rows")
    K, N = w.shape
    wq = torch.empty((N, K), dtype=torch.uint8, device=w.device)
    sc = torch.empty(N, dtype=torch.float32, device=w.device)
    _check(_abi.load().hstu_quant_weight_e4m3(w.data_ptr(), w.stride(0), K, N, wq.data_ptr(), K,
                                              sc.data_ptr(), _stream(stream)),
           "hstu_quant_weight_e4m3")
    return wq, sc


def quantize_weights(w: StuWeights, stream=None) -> Fp8Weights:
    """The E4M3 projections of one layer (redo after every weight update)."""
    return Fp8Weights(*quantize_weight_e4m3(w.w1, stream), *quantize_weight_e4m3(w.w2, stream))


@dataclasses.dataclass
class LayerState:
    """What one layer's forward saves for its backward.  Without remat: x^,
    pre, U|V|Q|K, A, y and both norms' statistics.  With remat (the save set
    of Listing 1 in ULTRA-HSTU section 4.2.2): only u (the U block), A and
    the statistics; xn, pre, uvqk, y are None and the backward recomputes
    them."""
    x: torch.Tensor
    seq_offsets: torch.Tensor
    num_targets: Optional[torch.Tensor]
    max_seq_len: int
    xn: Optional[torch.Tensor]
    pre: Optional[torch.Tensor]
    uvqk: Optional[torch.Tensor]
    av: torch.Tensor
    y: Optional[torch.Tensor]
    stats: torch.Tensor
    u: Optional[torch.Tensor] = None
    remat: bool = False

    def saved_bytes(self) -> int:
        """Bytes this state holds beyond the layer input x."""
        ts = (self.xn, self.pre, self.uvqk, self.av, self.y, self.stats, self.u)
        return sum(t.numel() * t.element_size() for t in ts if t is not None)


def _layer_params(cfg: StuConfig, w: StuWeights, st: LayerState, out,
                  fp8: Optional[Fp8Weights] = None) -> _abi.StuLayerParams:
    p = _abi.StuLayerParams()
    T = st.x.shape[0]
    p.B, p.H, p.d = st.seq_offsets.numel() - 1, cfg.H, cfg.d
    p.total_tokens, p.max_seq_len = T, st.max_seq_len
    p.seq_offsets, p.num_targets = st.seq_offsets.data_ptr(), _ptr(st.num_targets)
    p.contextual_len, p.K1, p.K2 = cfg.contextual_len, cfg.K1, cfg.K2
    p.alpha, p.N, p.ln_eps = cfg.alpha, cfg.N, cfg.ln_eps
    (p.ln1_w, p.ln1_b, p.w1, p.b1, p.ln2_w, p.ln2_b, p.w2, p.b2) = (t.data_ptr()
                                                                     for t in w.tensors())
    p.x, p.out = st.x.data_ptr(), _ptr(out)
    p.xn, p.pre, p.uvqk = _ptr(st.xn), _ptr(st.pre), _ptr(st.uvqk)
    p.av, p.y, p.stats = st.av.data_ptr(), _ptr(st.y), st.stats.data_ptr()
    p.remat, p.u = int(st.remat), _ptr(st.u)
    if fp8 is not None:
        p.fp8 = 1
        p.w1q, p.w1s, p.w2q, p.w2s = (fp8.w1q.data_ptr(), fp8.w1s.data_ptr(), fp8.w2q.data_ptr(),
                                      fp8.w2s.data_ptr())
    return p


def _check_x(x: torch.Tensor, cfg: StuConfig):
    if x.dtype != torch.bfloat16 or not x.is_cuda or x.dim() != 2 or x.shape[1] != cfg.d_model:
        raise ValueError(f"x must be CUDA bf16 [T, {cfg.d_model}]")
    if not x.is_contiguous():
        raise ValueError("x must be contiguous")


def workspace_bytes(which: int, T: int, B: int, cfg: StuConfig) -> int:
    return int(_abi.load().hstu_stu_workspace_bytes(which, T, B, cfg.H, cfg.d))


def layer_fwd(x: torch.Tensor, seq_offsets: torch.Tensor, num_targets: Optional[torch.Tensor],
              w: StuWeights, cfg: StuConfig, max_seq_len: int, workspace=None, stream=None,
              fp8: Optional[Fp8Weights] = None, remat: bool = False):
    """One STU layer forward; returns (out, state for the backward).  With
    fp8 (from quantize_weights) the two projections run in E4M3.  remat:
    keep only Listing 1's save set (u, A, statistics) for the backward."""
    _check_x(x, cfg)
    T, dm, dev = x.shape[0], cfg.d_model, x.device
    bf = dict(dtype=torch.bfloat16, device=dev)
    stats = torch.empty((4, T), dtype=torch.float32, device=dev)
    if remat:
        st = LayerState(x, seq_offsets, num_targets, int(max_seq_len), None, None, None,
                        torch.empty((T, dm), **bf), None, stats, torch.empty((T, dm), **bf), True)
    else:
        st = LayerState(x, seq_offsets, num_targets, int(max_seq_len),
                        torch.empty((T, dm), **bf), torch.empty((T, 4 * dm), **bf),
                        torch.empty((T, 4 * dm), **bf), torch.empty((T, dm), **bf),
                        torch.empty((T, dm), **bf), stats)
    out = torch.empty((T, dm), **bf)
    p = _layer_params(cfg, w, st, out, fp8)
    kind = _abi.WS_FWD_REMAT if remat else (_abi.WS_FWD if fp8 is None else _abi.WS_FWD_FP8)
    need = workspace_bytes(kind, T, p.B, cfg)
    ws = torch.empty(need, dtype=torch.uint8, device=dev) if workspace is None else workspace
    _check(_abi.load().hstu_stu_layer_fwd(ctypes.byref(p), ws.data_ptr(), ws.numel(),
                                          _stream(stream)), "hstu_stu_layer_fwd")
    return out, st


def layer_bwd(dout: torch.Tensor, st: LayerState, w: StuWeights, cfg: StuConfig, workspace=None,
              stream=None):
    """One STU layer backward; returns (dx, gradients as a StuWeights of fp32)."""
    T, dm, dev = st.x.shape[0], cfg.d_model, st.x.device
    if dout.shape != (T, dm) or dout.dtype != torch.bfloat16 or not dout.is_contiguous():
        raise ValueError(f"dout must be contiguous bf16 [{T}, {dm}]")
    bf = dict(dtype=torch.bfloat16, device=dev)
    f32 = dict(dtype=torch.float32, device=dev)
    q = _abi.StuLayerBwdParams()
    q.fwd = _layer_params(cfg, w, st, None)
    dx = torch.empty((T, dm), **bf)
    scratch = [torch.empty((T, dm), **bf), torch.empty((T, dm), **bf),
               torch.empty((T, 4 * dm), **bf), torch.empty((T, dm), **bf)]
    g = StuWeights(torch.empty(dm, **f32), torch.empty(dm, **f32), torch.empty((dm, 4 * dm), **f32),
                   torch.empty(4 * dm, **f32), torch.empty(dm, **f32), torch.empty(dm, **f32),
                   torch.empty((dm, dm), **f32), torch.empty(dm, **f32))
    q.dout, q.dx = dout.data_ptr(), dx.data_ptr()
    q.dy, q.dav, q.dpre, q.dxn = (t.data_ptr() for t in scratch)
    (q.d_ln1_w, q.d_ln1_b, q.d_w1, q.d_b1, q.d_ln2_w, q.d_ln2_b, q.d_w2,
     q.d_b2) = (t.data_ptr() for t in g.tensors())
    need = workspace_bytes(_abi.WS_BWD_REMAT if st.remat else _abi.WS_BWD, T, q.fwd.B, cfg)
    ws = torch.empty(need, dtype=torch.uint8, device=dev) if workspace is None else workspace
    _check(_abi.load().hstu_stu_layer_bwd(ctypes.byref(q), ws.data_ptr(), ws.numel(),
                                          _stream(stream)), "hstu_stu_layer_bwd")
    return dx, g


def truncated_lengths(lengths, num_targets, contextual_len: int, tail: int) -> np.ndarray:
    """Per-sequence lengths after truncation, from the library's host helper
    (the rule the truncation kernels apply), to size the truncated buffers."""
    L = np.ascontiguousarray(lengths, dtype=np.int32)
    nt = None if num_targets is None else np.ascontiguousarray(num_targets, dtype=np.int32)
    out = np.empty_like(L)
    total = _abi.load().hstu_jagged_truncate_lengths(
        L.ctypes.data, None if nt is None else nt.ctypes.data, len(L), int(contextual_len),
        int(tail), out.ctypes.data)
    if total < 0:
        _check(int(total), "hstu_jagged_truncate_lengths")
    return out.astype(np.int64)


def truncate_offsets(seq_offsets, num_targets, contextual_len: int, tail: int, stream=None):
    B = seq_offsets.numel() - 1
    new = torch.empty_like(seq_offsets)
    _check(_abi.load().hstu_jagged_truncate_offsets(seq_offsets.data_ptr(), _ptr(num_targets), B,
                                                    contextual_len, tail, new.data_ptr(),
                                                    _stream(stream)),
           "hstu_jagged_truncate_offsets")
    return new


def jagged_truncate(x, seq_offsets, new_offsets, num_targets, contextual_len: int, tail: int,
                    T_out: int, scatter: bool = False, stream=None):
    """Gather the kept rows of x (scatter=False) or put rows back into the full
    layout with zeros for the dropped ones (scatter=True)."""
    W = x.shape[1]
    dst = torch.empty((T_out, W), dtype=x.dtype, device=x.device)
    _check(_abi.load().hstu_jagged_truncate(x.data_ptr(), x.stride(0), seq_offsets.data_ptr(),
                                            new_offsets.data_ptr(), _ptr(num_targets),
                                            seq_offsets.numel() - 1, contextual_len, tail, W,
                                            dst.data_ptr(), dst.stride(0), T_out, int(scatter),
                                            _stream(stream)),
           "hstu_jagged_truncate")
    return dst


def gemm(a, b, *, M, N, K, a_mn_major, b_mn_major, epilogue, splits=1, bias=None, resid=None,
         out=None, out2=None, outf=None, a_scale=None, b_scale=None, stream=None):
    """The layer GEMM D[m][n] = sum_k A[m][k] B[n][k] (test hook).  With
    a_scale / b_scale, a and b are E4M3 bytes and D is scaled by
    a_scale[m] * b_scale[n]."""
    p = _abi.GemmParams()
    p.M, p.N, p.K = M, N, K
    p.a, p.lda, p.a_mn_major = a.data_ptr(), a.stride(0), int(a_mn_major)
    p.b, p.ldb, p.b_mn_major = b.data_ptr(), b.stride(0), int(b_mn_major)
    p.epilogue, p.splits = epilogue, splits
    p.bias = _ptr(bias)
    p.resid, p.ldr = _ptr(resid), (resid.stride(0) if resid is not None else 0)
    p.out, p.ldo = _ptr(out), (out.stride(0) if out is not None else 0)
    p.out2, p.ldo2 = _ptr(out2), (out2.stride(0) if out2 is not None else 0)
    p.outf, p.ldf = _ptr(outf), (outf.stride(0) if outf is not None else 0)
    if a_scale is not None or b_scale is not None:
        p.fp8, p.a_scale, p.b_scale = 1, _ptr(a_scale), _ptr(b_scale)
    ws = torch.empty(256, dtype=torch.uint8, device=a.device)
    lib = _abi.load()
    _check(lib.hstu_gemm(ctypes.byref(p), ws.data_ptr(), _stream(stream)), "hstu_gemm")
    _check(lib.hstu_sla_get_error(ws.data_ptr(), _stream(stream)), "hstu_gemm (device)")


class StuStack:
    """`len(weights)` STU layers, truncation after the first `trunc_after`.

    cfg_full / cfg_trunc: attention settings before / after truncation (their
    N differ: the longest sequence of each stage).  fp8=True runs the forward
    projections in E4M3; call requantize() after every weight update.
    remat=True keeps only Listing 1's save set per layer and recomputes the
    rest in the backward."""

    def __init__(self, weights: List[StuWeights], cfg_full: StuConfig, cfg_trunc: StuConfig,
                 trunc_after: int, tail: int, fp8: bool = False, remat: bool = False):
        self.weights, self.cfg_full, self.cfg_trunc = weights, cfg_full, cfg_trunc
        self.trunc_after, self.tail = trunc_after, tail
        self.remat = remat
        self.fp8 = None
        if fp8:
            self.requantize()

    def requantize(self, stream=None):
        """E4M3 copies of every layer's projections (the FP8 forward's weights)."""
        self.fp8 = [quantize_weights(w, stream) for w in self.weights]

    def forward(self, x, seq_offsets, num_targets, lengths, host_num_targets, stream=None):
        """x: [T, d_model] bf16; lengths / host_num_targets: host copies of the
        batch geometry (sizes of the truncated buffers).  Returns (out, ctx)."""
        c = self.cfg_full.contextual_len
        states, h = [], x
        offs, msl = seq_offsets, int(np.max(lengths))
        new_offs, T_new = None, None
        for i, w in enumerate(self.weights):
            if i == self.trunc_after:
                tl = truncated_lengths(lengths, host_num_targets, c, self.tail)
                T_new, msl = int(tl.sum()), int(tl.max())
                new_offs = truncate_offsets(seq_offsets, num_targets, c, self.tail, stream)
                h = jagged_truncate(h, seq_offsets, new_offs, num_targets, c, self.tail, T_new,
                                    stream=stream)
                offs = new_offs
            cfg = self.cfg_full if i < self.trunc_after else self.cfg_trunc
            h, st = layer_fwd(h, offs, num_targets, w, cfg, msl, stream=stream,
                              fp8=None if self.fp8 is None else self.fp8[i], remat=self.remat)
            states.append(st)
        return h, (states, seq_offsets, new_offs, num_targets, x.shape[0])

    def backward(self, dout, ctx, stream=None):
        """Returns (dx, [per-layer gradients as StuWeights of fp32])."""
        states, offs, new_offs, nts, T_full = ctx
        c = self.cfg_full.contextual_len
        grads = [None] * len(self.weights)
        g = dout
        for i in reversed(range(len(self.weights))):
            cfg = self.cfg_full if i < self.trunc_after else self.cfg_trunc
            g, grads[i] = layer_bwd(g.contiguous(), states[i], self.weights[i], cfg, stream=stream)
            if i == self.trunc_after:
                g = jagged_truncate(g, offs, new_offs, nts, c, self.tail, T_full, scatter=True,
                                    stream=stream)
        return g, grads

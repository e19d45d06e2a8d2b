"""STU-layer and STU-stack oracle -- TEST INFRASTRUCTURE ONLY.

Plain numpy in fp64 (matrix products through numpy's matmul, the attention
through this package's C loops), step by step as the cited papers define them; no
fusion, no blocking.  Only the tests and the benchmark's CPU-baseline leg may
import it; the CUDA library shares nothing with it.

Definitions followed:
  * STU layer: "Bending the Scaling Law Curve in Large-Scale Recommendation
    Systems", section 3, Eq. 1-2 (the four blocks = phi1(f1(Norm(x))), f1 a
    linear map, phi1 = SiLU), Eq. 3 (the pointwise SiLU attention), Eq. 4-5
    (Norm(A) * U, the output map f2 and the residual).  The block order
    U, V, Q, K is the one the forward of Listing 1 (section 4.2.2) unpacks;
    the residual enters as the output map's bias there (out = y W2 + x), and
    the backward below is that listing's backward with everything recomputed
    kept instead.
  * LayerNorm: biased variance, eps inside the square root, affine weight and
    bias (the reading used throughout: eps = 1e-5).
  * Truncation: section 4.3 ("attention truncation": keep the most recent
    history segment) and TorchEasyRec's "Mid-stack Attention Truncation"
    bullet (contextual prefix and candidates always kept): after a given layer
    keep per sequence the contextual prefix, the last `tail` history tokens
    and all candidates; when the history past the prefix is no longer than
    `tail`, keep the whole sequence.

Parity pins: tests/test_oracle_stu_pins.py (finite differences of the layer
and the stack, LayerNorm moments, the residual identity, the block order of
the split through zeroed weight blocks, the truncation index set built from
its definition).
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional

import numpy as np

from . import Problem
from . import fp8 as _fp8


def silu(x):
    return x / (1.0 + np.exp(-x))


def silu_grad(x):
    s = 1.0 / (1.0 + np.exp(-x))
    return s * (1.0 + x * (1.0 - s))


def layer_norm(x, w, b, eps):
    """Returns (normalised * w + b, x_hat, rstd)."""
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    rstd = 1.0 / np.sqrt(var + eps)
    xh = (x - mu) * rstd
    return xh * w + b, xh, rstd


def layer_norm_bwd(g, xh, rstd):
    """dL/dx of x_hat given g = dL/dx_hat (per row)."""
    return rstd * (g - g.mean(axis=-1, keepdims=True) - xh * (g * xh).mean(axis=-1, keepdims=True))


@dataclasses.dataclass
class Weights:
    """One layer's parameters as fp64 arrays (W in the x W convention)."""
    ln1_w: np.ndarray
    ln1_b: np.ndarray
    w1: np.ndarray   # [dm, 4 dm]
    b1: np.ndarray
    ln2_w: np.ndarray
    ln2_b: np.ndarray
    w2: np.ndarray   # [dm, dm]
    b2: np.ndarray

    @staticmethod
    def of(**kw) -> "Weights":
        return Weights(**{k: np.asarray(v, dtype=np.float64) for k, v in kw.items()})


@dataclasses.dataclass
class AttnCfg:
    H: int
    d: int
    contextual_len: int
    K1: int
    K2: int
    alpha: float
    N: float
    eps: float = 1e-5


def _problem(offsets, num_targets, cfg: AttnCfg) -> Problem:
    return Problem(offsets, num_targets, cfg.H, cfg.d, cfg.contextual_len, cfg.K1, cfg.K2,
                   cfg.alpha, cfg.N)


def layer_fwd(x, w: Weights, offsets, num_targets, cfg: AttnCfg, fp8: bool = False):
    """One STU layer; returns (out, cache).  fp8: both projections take E4M3
    operands (oracle.fp8: the bf16 value of x^ and of y quantized per row,
    W1 and W2 per column); the cache, and so the backward, keeps the
    unquantized values."""
    x = np.asarray(x, dtype=np.float64)
    T, dm = x.shape
    xn, xh1, r1 = layer_norm(x, w.ln1_w, w.ln1_b, cfg.eps)
    pre = (_fp8.fp8_matmul(_fp8.bf16_round(xn), w.w1) if fp8 else xn @ w.w1) + w.b1
    uvqk = silu(pre)
    u, v, q, k = (uvqk[:, i * dm:(i + 1) * dm] for i in range(4))
    prob = _problem(offsets, num_targets, cfg)
    shp = (T, cfg.H, cfg.d)
    av = prob.fwd(q.reshape(shp), k.reshape(shp), v.reshape(shp)).reshape(T, dm)
    z, xh2, r2 = layer_norm(av, w.ln2_w, w.ln2_b, cfg.eps)
    y = z * u
    out = (_fp8.fp8_matmul(_fp8.bf16_round(y), w.w2) if fp8 else y @ w.w2) + w.b2 + x
    cache = dict(x=x, xn=xn, xh1=xh1, r1=r1, pre=pre, u=u, v=v, q=q, k=k, av=av, z=z, xh2=xh2,
                 r2=r2, y=y, prob=prob, shp=shp)
    return out, cache


def layer_bwd(dout, w: Weights, cache):
    """Gradients of sum(out * dout): returns (dx, Weights of gradients)."""
    dout = np.asarray(dout, dtype=np.float64)
    c = cache
    dW2 = c["y"].T @ dout
    db2 = dout.sum(axis=0)
    dy = dout @ w.w2.T
    dz = dy * c["u"]
    du = dy * c["z"]
    dln2_w = (dz * c["xh2"]).sum(axis=0)
    dln2_b = dz.sum(axis=0)
    dav = layer_norm_bwd(dz * w.ln2_w, c["xh2"], c["r2"])
    shp, T = c["shp"], dout.shape[0]
    dq, dk, dv = c["prob"].bwd(c["q"].reshape(shp), c["k"].reshape(shp), c["v"].reshape(shp),
                               dav.reshape(shp))
    duvqk = np.concatenate([du, dv.reshape(T, -1), dq.reshape(T, -1), dk.reshape(T, -1)], axis=1)
    dpre = duvqk * silu_grad(c["pre"])
    dW1 = c["xn"].T @ dpre
    db1 = dpre.sum(axis=0)
    dxn = dpre @ w.w1.T
    dln1_w = (dxn * c["xh1"]).sum(axis=0)
    dln1_b = dxn.sum(axis=0)
    dx = dout + layer_norm_bwd(dxn * w.ln1_w, c["xh1"], c["r1"])
    return dx, Weights(dln1_w, dln1_b, dW1, db1, dln2_w, dln2_b, dW2, db2)


def kept_positions(L: int, nt: int, contextual_len: int, tail: int) -> List[int]:
    """Positions (within one sequence) that survive truncation."""
    Lh = L - nt
    if Lh - contextual_len <= tail:
        return list(range(L))
    return (list(range(contextual_len)) + list(range(Lh - tail, Lh)) + list(range(Lh, L)))


def truncation_index(offsets, num_targets, contextual_len: int, tail: int):
    """Global source rows of the truncated layout, and its offsets."""
    offsets = np.asarray(offsets, dtype=np.int64)
    B = len(offsets) - 1
    nts = np.zeros(B, np.int64) if num_targets is None else np.asarray(num_targets, np.int64)
    idx, new = [], [0]
    for b in range(B):
        L = int(offsets[b + 1] - offsets[b])
        keep = kept_positions(L, int(nts[b]), contextual_len, tail)
        idx.extend(int(offsets[b]) + p for p in keep)
        new.append(new[-1] + len(keep))
    return np.asarray(idx, dtype=np.int64), np.asarray(new, dtype=np.int64)


def stack_fwd(x, weights: List[Weights], offsets, num_targets, cfg_full: AttnCfg,
              cfg_trunc: AttnCfg, trunc_after: int, tail: int, fp8: bool = False):
    """The truncated STU stack; returns (out, cache).  fp8 as in layer_fwd."""
    h = np.asarray(x, dtype=np.float64)
    caches, offs, idx, new_offs = [], offsets, None, None
    for i, w in enumerate(weights):
        if i == trunc_after:
            idx, new_offs = truncation_index(offsets, num_targets, cfg_full.contextual_len, tail)
            h = h[idx]
            offs = new_offs
        cfg = cfg_full if i < trunc_after else cfg_trunc
        h, c = layer_fwd(h, w, offs, num_targets, cfg, fp8)
        caches.append(c)
    return h, dict(caches=caches, idx=idx, T=np.asarray(x).shape[0], trunc_after=trunc_after)


def stack_bwd(dout, weights: List[Weights], cache):
    """Returns (dx, [per-layer gradient Weights])."""
    g = np.asarray(dout, dtype=np.float64)
    grads: List[Optional[Weights]] = [None] * len(weights)
    for i in reversed(range(len(weights))):
        g, grads[i] = layer_bwd(g, weights[i], cache["caches"][i])
        if i == cache["trunc_after"]:
            full = np.zeros((cache["T"], g.shape[1]), np.float64)
            full[cache["idx"]] = g
            g = full
    return g, grads

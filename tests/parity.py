"""Helpers shared by the GPU parity tests: run the CUDA library through its
binding and the oracle on the same seeded inputs, compare."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import sparse_hstu_attention_b200 as sla
from workloads import Batch

TOL = 2e-2  # max|gpu - ref| <= TOL * max|ref|, per tensor


def to_gpu(batch: Batch, strided: bool = False):
    """Device copies of the batch.  strided=True places q, k, v as views of a
    fused [T, 4*H*d] buffer in U, V, Q, K order (the STU projection layout)."""
    dev = torch.device("cuda")
    offs = torch.tensor(batch.seq_offsets, dtype=torch.int32, device=dev)
    nts = torch.tensor(batch.num_targets, dtype=torch.int32, device=dev)
    T, H, d = batch.q.shape
    if strided:
        fused = torch.zeros((T, 4, H, d), dtype=torch.bfloat16, device=dev)
        fused[:, 1] = batch.v.to(dev)
        fused[:, 2] = batch.q.to(dev)
        fused[:, 3] = batch.k.to(dev)
        q, k, v = fused[:, 2], fused[:, 3], fused[:, 1]
    else:
        q, k, v = (t.to(dev) for t in (batch.q, batch.k, batch.v))
    dout = batch.dout.to(dev) if batch.dout is not None else None
    return dict(q=q, k=k, v=v, dout=dout, offs=offs, nts=nts)


def kwargs_of(batch: Batch, **override):
    w = batch.workload
    kw = dict(contextual_len=w.contextual_len, K1=w.K1, K2=w.K2, alpha=w.alpha, N=w.N,
              max_seq_len=int(batch.lengths.max()) if len(batch.lengths) else 0)
    kw.update(override)
    return kw


def gpu_fwd(batch: Batch, g=None, **override):
    g = g or to_gpu(batch)
    out = sla.hstu_sla_fwd(g["q"], g["k"], g["v"], g["offs"], g["nts"], **kwargs_of(batch, **override))
    torch.cuda.synchronize()
    return out


def gpu_bwd(batch: Batch, g=None, **override):
    g = g or to_gpu(batch)
    dq, dk, dv = sla.hstu_sla_bwd(g["dout"], g["q"], g["k"], g["v"], g["offs"], g["nts"],
                                  **kwargs_of(batch, **override))
    torch.cuda.synchronize()
    return dq, dk, dv


def oracle_problem(batch: Batch, **override):
    w = batch.workload
    kw = dict(H=w.H, d=w.d, contextual_len=w.contextual_len, K1=w.K1, K2=w.K2, alpha=w.alpha,
              N=w.N)
    kw.update({k: v for k, v in override.items() if k in kw})
    return oracle.Problem(batch.seq_offsets, batch.num_targets, **kw)


def assert_close(name, got, ref, tol=TOL):
    got = got.float().cpu().numpy().astype(np.float64) if isinstance(got, torch.Tensor) else got
    scale = float(np.abs(ref).max()) if ref.size else 0.0
    err = float(np.abs(got - ref).max()) if ref.size else 0.0
    assert np.all(np.isfinite(got)), f"{name}: non-finite values"
    assert err <= tol * max(scale, 1e-30), f"{name}: max|err| {err:.3e} > {tol} * {scale:.3e}"
    return err, scale


def sample_tokens(batch: Batch, n_random: int, seed: int = 0):
    """Random tokens plus the edges: first/last token of each sequence, the first
    and last candidate, and positions around 64/128-token tile boundaries."""
    rng = np.random.default_rng(seed)
    offs = batch.seq_offsets
    picks = set(rng.integers(0, batch.T, size=n_random).tolist()) if batch.T else set()
    for b in range(len(offs) - 1):
        s0, s1 = int(offs[b]), int(offs[b + 1])
        if s1 == s0:
            continue
        L, nt = s1 - s0, int(batch.num_targets[b])
        for p in (0, 1, L - 1, L - nt, L - nt - 1, 63, 64, 127, 128, 129):
            if 0 <= p < L:
                picks.add(s0 + p)
    return np.array(sorted(picks), dtype=np.int64)

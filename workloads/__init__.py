"""Seeded synthetic jagged batches for SLA HSTU attention.

This module only draws inputs: sequence lengths, candidate counts and the
bf16 tensors q, k, v, dout.  It holds none of the attention arithmetic; the
oracle (test infrastructure) and the CUDA library both consume what it
returns, so the two are fed bit-identical inputs.

Shapes follow the workloads the ULTRA-HSTU pages describe: user histories of
3K-16K events ("Bending the Scaling Law Curve in Large-Scale Recommendation
Systems", section 5.1.1; 16K production sequences, section 1), a contextual
prefix at the start and candidate targets at the end (section 3, "Input";
TorchEasyRec "ULTRA HSTU" docs), 4 heads of 128 (TorchEasyRec example config,
embedding_dim 512 / num_heads 4 / attention_dim 128).  The industrial logs and
KuaiRand those papers measure on are not available; these draws stand in for
them.

Recipe (fixed): lengths from ``numpy.random.default_rng(1000 + index)``;
tensors from ``torch.Generator('cpu').manual_seed(1000 + index)`` drawn as
fp32 N(0, 1) in the order q, k, v, dout, then rounded to bf16.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    index: int                 # 1-based; seeds derive from it
    name: str
    B: int
    H: int
    d: int
    K1: int
    K2: int
    contextual_len: int
    num_targets: int
    alpha: float
    N: float
    fwd_only: bool = False
    description: str = ""

    @property
    def seed(self) -> int:
        return 1000 + self.index


WORKLOADS = {
    "tiny": Workload(1, "tiny", B=4, H=2, d=32, K1=32, K2=16, contextual_len=4,
                     num_targets=8, alpha=1.0 / math.sqrt(32), N=256.0,
                     description="4 seqs, L~U{32..256}, 2x32 heads"),
    "mid": Workload(2, "mid", B=32, H=4, d=128, K1=256, K2=64, contextual_len=16,
                    num_targets=16, alpha=1.0 / math.sqrt(128), N=4096.0,
                    description="32 seqs, L~U{1024..4096}, 4x128 heads"),
    "hist16k": Workload(3, "hist16k", B=8, H=4, d=128, K1=1024, K2=128,
                        contextual_len=32, num_targets=64,
                        alpha=1.0 / math.sqrt(128), N=16384.0,
                        description="8 seqs: 4x16384 + 4x16384*U(0.25,1), total<=98304"),
    "infer": Workload(4, "infer", B=64, H=4, d=128, K1=512, K2=128,
                      contextual_len=32, num_targets=512,
                      alpha=1.0 / math.sqrt(128), N=8704.0, fwd_only=True,
                      description="64 seqs of 8192 history + 512 candidates"),
    "stu": Workload(5, "stu", B=16, H=4, d=128, K1=1024, K2=128,
                    contextual_len=32, num_targets=64,
                    alpha=1.0 / math.sqrt(128), N=16384.0,
                    description="6-layer STU stack, L~U{4096..16384}"),
}

HIST16K_TOKEN_BUDGET = 96 * 1024

# Mixture of Transducers: one transducer per user-signal channel, each with its
# own sequences and SLA settings ("Bending the Scaling Law Curve...", section
# 4.3 and appendix A; TorchEasyRec "ULTRA HSTU" docs, MoT: per-channel STU
# stack and SLA / truncation configuration).  The sources give no channel mix;
# this one pairs a long dense channel (16K-class histories, as hist16k), a
# medium one and a short one with full causal attention.  The three
# channels' attentions run as one grouped launch.
MOT_CHANNELS = {
    "mot_long": Workload(6, "mot_long", B=8, H=4, d=128, K1=1024, K2=128, contextual_len=32,
                         num_targets=64, alpha=1.0 / math.sqrt(128), N=16384.0,
                         description="8 seqs, L~U{8192..16384}"),
    "mot_mid": Workload(7, "mot_mid", B=32, H=4, d=128, K1=256, K2=64, contextual_len=16,
                        num_targets=16, alpha=1.0 / math.sqrt(128), N=4096.0,
                        description="32 seqs, L~U{1024..4096}"),
    "mot_short": Workload(8, "mot_short", B=128, H=4, d=128, K1=1024, K2=0, contextual_len=0,
                          num_targets=8, alpha=1.0 / math.sqrt(128), N=1024.0,
                          description="128 seqs, L~U{128..1024}, full causal"),
}


def draw_lengths(w: Workload, seed: Optional[int] = None) -> np.ndarray:
    """Total per-sequence lengths (contextual prefix and candidates included);
    `seed` overrides the workload's own (another batch of the same recipe)."""
    rng = np.random.default_rng(w.seed if seed is None else seed)
    if w.name == "tiny":
        return rng.integers(32, 256, size=w.B, endpoint=True).astype(np.int64)
    if w.name == "mid":
        return rng.integers(1024, 4096, size=w.B, endpoint=True).astype(np.int64)
    if w.name == "hist16k":
        pinned = np.full(4, 16384, dtype=np.int64)
        while True:  # redraw the free half until the batch fits the token budget
            free = np.floor(16384 * rng.uniform(0.25, 1.0, size=4)).astype(np.int64)
            if pinned.sum() + free.sum() <= HIST16K_TOKEN_BUDGET:
                return np.concatenate([pinned, free])
    if w.name == "infer":
        return np.full(w.B, 8192 + 512, dtype=np.int64)
    if w.name == "stu":
        return rng.integers(4096, 16384, size=w.B, endpoint=True).astype(np.int64)
    if w.name == "mot_long":
        return rng.integers(8192, 16384, size=w.B, endpoint=True).astype(np.int64)
    if w.name == "mot_mid":
        return rng.integers(1024, 4096, size=w.B, endpoint=True).astype(np.int64)
    if w.name == "mot_short":
        return rng.integers(128, 1024, size=w.B, endpoint=True).astype(np.int64)
    raise KeyError(w.name)


def draw_timestamps(lengths, num_targets, seed: int) -> np.ndarray:
    """Seeded int32 event times (seconds) for the relative attention bias:
    per sequence a start in [1.6e9, 1.61e9), exponential gaps of mean 600 s
    between history events, and every candidate at the request time (an
    exponential gap after the last history event)."""
    rng = np.random.default_rng(seed)
    out = []
    for L, nt in zip(np.asarray(lengths, np.int64), np.asarray(num_targets, np.int64)):
        Lh = int(L - nt)
        start = 1_600_000_000 + int(rng.integers(0, 10_000_000))
        hist = start + np.cumsum(rng.exponential(600.0, size=Lh).astype(np.int64))
        req = (hist[-1] if Lh else start) + int(rng.exponential(600.0))
        out.append(np.concatenate([hist, np.full(int(nt), req, np.int64)]))
    ts = np.concatenate(out) if out else np.zeros(0, np.int64)
    assert ts.size == 0 or ts.max() < 2 ** 31
    return ts.astype(np.int32)


def draw_rab_tables(H: int, n_pos: int, n_time: int, seed: int):
    """Seeded relative-attention-bias tables [H][buckets], N(0, 0.5^2)."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    return (torch.randn((H, n_pos), generator=g) * 0.5,
            torch.randn((H, n_time), generator=g) * 0.5)


def offsets_from_lengths(lengths) -> np.ndarray:
    lengths = np.asarray(lengths, dtype=np.int64)
    return np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)


def draw_tensors(T: int, H: int, d: int, seed: int, n: int = 4):
    """n bf16 tensors [T, H, d] ~ N(0,1) in the order q, k, v, dout."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    return [torch.randn((T, H, d), generator=g, dtype=torch.float32).to(torch.bfloat16)
            for _ in range(n)]


@dataclasses.dataclass
class Batch:
    workload: Workload
    lengths: np.ndarray          # [B] int64
    seq_offsets: np.ndarray      # [B+1] int64
    num_targets: np.ndarray      # [B] int64
    q: torch.Tensor              # bf16 [T, H, d] (CPU)
    k: torch.Tensor
    v: torch.Tensor
    dout: Optional[torch.Tensor]

    @property
    def T(self) -> int:
        return int(self.seq_offsets[-1])


def make_batch(w: Workload, lengths=None, num_targets=None, seed: Optional[int] = None,
               with_dout: bool = True) -> Batch:
    """Draw the workload's batch.  ``lengths``/``num_targets``/``seed`` override
    the workload's own draw (used for small parity and edge cases)."""
    lengths = draw_lengths(w) if lengths is None else np.asarray(lengths, dtype=np.int64)
    if num_targets is None:
        nt = np.minimum(np.full(len(lengths), w.num_targets, dtype=np.int64), lengths)
    else:
        nt = np.broadcast_to(np.asarray(num_targets, dtype=np.int64), lengths.shape).copy()
    offs = offsets_from_lengths(lengths)
    T = int(offs[-1])
    ts = draw_tensors(T, w.H, w.d, w.seed if seed is None else seed, n=4 if with_dout else 3)
    return Batch(w, lengths, offs, nt, ts[0], ts[1], ts[2], ts[3] if with_dout else None)


def with_params(w: Workload, **kw) -> Workload:
    """A copy of a workload with some fields changed (edge cases)."""
    return dataclasses.replace(w, **kw)


# ----------------------------------------------------------------- STU stack
# The 6-layer STU stack workload: d_model = H * d = 512, truncation after
# layer 3 to contextual + the last 1024 history tokens + the candidates
# (TorchEasyRec "ULTRA HSTU" docs: attn_truncation_tail_len), N = the longest
# sequence of each stage.
STU_LAYERS = 6
STU_TRUNC_AFTER = 3
STU_TAIL = 1024


@dataclasses.dataclass
class StuDraw:
    """Seeded inputs of an STU stack: x, the upstream gradient of the stack
    output, and each layer's parameters as CPU tensors (projections bf16 in
    the x W convention, the rest fp32)."""
    x: torch.Tensor                 # bf16 [T, d_model]
    dout: torch.Tensor              # bf16 [T_out, d_model]
    layers: list                    # per layer: dict of CPU tensors


def draw_stu(T: int, T_out: int, d_model: int, n_layers: int, seed: int,
             perturb: bool = False) -> StuDraw:
    """x, dout ~ N(0, 1); W1 [d_model, 4 d_model] and W2 [d_model, d_model]
    Xavier-uniform (bound sqrt(6 / (fan_in + fan_out))); biases 0 and
    LayerNorm weight 1 / bias 0, or (perturb=True, to exercise those terms)
    biases ~ 0.1 N(0, 1) and LayerNorm weight 1 + 0.1 N(0, 1), bias 0.1 N(0, 1).
    Draw order: x, dout, then per layer W1, W2, then the perturbations."""
    g = torch.Generator(device="cpu").manual_seed(seed)
    x = torch.randn((T, d_model), generator=g).to(torch.bfloat16)
    dout = torch.randn((T_out, d_model), generator=g).to(torch.bfloat16)

    def xavier(fi, fo):
        a = math.sqrt(6.0 / (fi + fo))
        return ((torch.rand((fi, fo), generator=g) * 2 - 1) * a).to(torch.bfloat16)

    layers = []
    for _ in range(n_layers):
        lw = dict(w1=xavier(d_model, 4 * d_model), w2=xavier(d_model, d_model),
                  ln1_w=torch.ones(d_model), ln1_b=torch.zeros(d_model),
                  b1=torch.zeros(4 * d_model), ln2_w=torch.ones(d_model),
                  ln2_b=torch.zeros(d_model), b2=torch.zeros(d_model))
        layers.append(lw)
    if perturb:
        for lw in layers:
            for k in ("ln1_w", "ln2_w"):
                lw[k] = 1.0 + 0.1 * torch.randn(d_model, generator=g)
            for k in ("ln1_b", "ln2_b", "b2"):
                lw[k] = 0.1 * torch.randn(d_model, generator=g)
            lw["b1"] = 0.1 * torch.randn(4 * d_model, generator=g)
    return StuDraw(x, dout, layers)

"""Host-side work accounting for SLA attention: unmasked pairs, FLOPs, bytes.

Pairs follow from the mask in closed form ("Bending the Scaling Law Curve in
Large-Scale Recommendation Systems", section 4.2.1: the SLA cost is
O((K1 + K2) L)): a history row i sees min(i + 1, K1 + K2eff) keys; a candidate
sees min(Lh, K2eff + max(K1 - 1, 0)) history keys plus itself.

FLOPs per unmasked pair per head: forward 4d (Q K^T and P V), backward 10d
(recomputed S, dP, dV, dK, dQ).  Algorithmic HBM bytes per token per head
(bf16): forward q, k, v read + out written = 8d; backward q, k, v, dout read +
dq, dk, dv written = 14d.
"""
from __future__ import annotations

import numpy as np


def history_pairs(Lh: np.ndarray, W: int) -> np.ndarray:
    """sum_{i < Lh} min(i + 1, W) for each history length Lh."""
    Lh = np.asarray(Lh, dtype=np.int64)
    head = np.minimum(Lh, W)
    return head * (head + 1) // 2 + np.maximum(Lh - W, 0) * W


def pairs_per_sequence(lengths, num_targets, contextual_len: int, K1: int, K2: int) -> np.ndarray:
    lengths = np.asarray(lengths, dtype=np.int64)
    nt = np.asarray(num_targets, dtype=np.int64)
    K2e = max(K2, contextual_len)
    Lh = lengths - nt
    tgt = nt * (np.minimum(Lh, K2e + max(K1 - 1, 0)) + 1)
    return history_pairs(Lh, K1 + K2e) + tgt


def candidate_pairs(lengths, num_targets, contextual_len: int, K1: int, K2: int) -> int:
    """Unmasked pairs of the candidate rows alone (one head): what M-FALCON
    scoring computes per candidate."""
    lengths = np.asarray(lengths, dtype=np.int64)
    nt = np.asarray(num_targets, dtype=np.int64)
    K2e = max(K2, contextual_len)
    return int((nt * (np.minimum(lengths - nt, K2e + max(K1 - 1, 0)) + 1)).sum())


def total_pairs(lengths, num_targets, contextual_len, K1, K2) -> int:
    """Unmasked (row, key) pairs of one head over the batch."""
    return int(pairs_per_sequence(lengths, num_targets, contextual_len, K1, K2).sum())


def pairs_per_token(lengths, num_targets, contextual_len: int, K1: int, K2: int):
    """Per token of the jagged batch: keys it sees as a row, and rows that see it
    as a key (both per head), int64 [T] each."""
    lengths = np.asarray(lengths, dtype=np.int64)
    nts = np.asarray(num_targets, dtype=np.int64)
    K2e = max(K2, contextual_len)
    T = int(lengths.sum())
    rp = np.zeros(T, np.int64)
    kp = np.zeros(T, np.int64)
    s0 = 0
    for L, nt in zip(lengths.tolist(), nts.tolist()):
        Lh = L - nt
        i = np.arange(L)
        rp[s0:s0 + L] = np.where(i < Lh, np.minimum(i + 1, K1 + K2e),
                                 min(Lh, K2e + max(K1 - 1, 0)) + 1)
        # key j: a history prefix key is seen by every row from j on; another
        # history key by the history rows of its window and, if it lies in the
        # candidates' window, by every candidate; a candidate key by itself.
        band = np.clip(np.minimum(i + K1 - 1, Lh - 1) - i + 1, 0, None)
        in_tgt_window = (i < Lh) & (Lh - i < K1)
        kp[s0:s0 + L] = np.where(i < min(K2e, Lh), L - i,
                                 np.where(i < Lh, band + nt * in_tgt_window, 1))
        s0 += L
    return rp, kp


def fwd_flops(pairs: int, H: int, d: int) -> float:
    return 4.0 * d * pairs * H


def bwd_flops(pairs: int, H: int, d: int) -> float:
    return 10.0 * d * pairs * H


def fwd_bytes(T: int, H: int, d: int) -> float:
    return 8.0 * d * T * H


def bwd_bytes(T: int, H: int, d: int) -> float:
    return 14.0 * d * T * H

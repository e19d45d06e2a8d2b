"""Splitting a jagged batch across GPUs.

SLA attention has no exchange between sequences, so a global batch shards by
whole sequences with no collective on the data path: each rank gets a subset
of sequences (its own seq_offsets) chosen greedily longest-processing-time
first on the closed-form pair count, which balances the per-rank work.
"""
from __future__ import annotations

import heapq

import numpy as np

from .flops import pairs_per_sequence


def partition_sequences(lengths, num_targets, world_size: int, contextual_len: int, K1: int,
                        K2: int):
    """Returns, per rank, the sorted indices of the sequences it owns."""
    cost = pairs_per_sequence(lengths, num_targets, contextual_len, K1, K2)
    order = np.argsort(-cost, kind="stable")
    heap = [(0, r) for r in range(world_size)]
    owned = [[] for _ in range(world_size)]
    for b in order:
        load, r = heapq.heappop(heap)
        owned[r].append(int(b))
        heapq.heappush(heap, (load + int(cost[b]), r))
    return [sorted(o) for o in owned]


def shard_offsets(lengths, owned):
    """seq_offsets [len(owned)+1] of a rank's sub-batch and the global token
    index of each of its tokens (for gathering its rows)."""
    lengths = np.asarray(lengths, dtype=np.int64)
    starts = np.concatenate([[0], np.cumsum(lengths)])
    sub = lengths[owned]
    offs = np.concatenate([[0], np.cumsum(sub)]).astype(np.int64)
    tokens = np.concatenate([np.arange(starts[b], starts[b] + lengths[b]) for b in owned]) \
        if len(owned) else np.zeros(0, np.int64)
    return offs, tokens.astype(np.int64)

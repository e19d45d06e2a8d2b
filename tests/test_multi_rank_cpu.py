"""The N > 1 path on the CPU: two gloo ranks shard a jagged batch by whole
sequences (sharding.partition_sequences, longest first on the closed-form pair
count), each computes its sub-batch, and the gathered rows equal the single
batch's (sequences are independent: no exchange on the data path).  The
timing reduction bench.py uses (max over ranks) is checked the same way."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from sparse_hstu_attention_b200 import sharding
from workloads import WORKLOADS, make_batch, with_params

WORLD = 2


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, port, result_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=WORLD)
    try:
        import oracle
        w = with_params(WORKLOADS["tiny"], H=2, d=8)
        b = make_batch(w, lengths=np.array([70, 13, 120, 45, 88, 9, 33]), num_targets=[4, 0, 8, 2, 5, 9, 1],
                       seed=3)
        owned = sharding.partition_sequences(b.lengths, b.num_targets, WORLD, w.contextual_len,
                                             w.K1, w.K2)
        mine = owned[rank]
        offs, tokens = sharding.shard_offsets(b.lengths, mine)
        p = oracle.Problem(offs, b.num_targets[mine], w.H, w.d, w.contextual_len, w.K1, w.K2,
                           w.alpha, w.N)
        t = torch.from_numpy(tokens)
        out = p.fwd(b.q[t], b.k[t], b.v[t])
        # gather every rank's (token index, output row) pairs
        n = torch.tensor([len(tokens)])
        sizes = [torch.zeros(1, dtype=torch.int64) for _ in range(WORLD)]
        dist.all_gather(sizes, n)
        cap = int(max(s.item() for s in sizes))
        pad_t = torch.full((cap,), -1, dtype=torch.int64)
        pad_t[:len(tokens)] = t
        pad_o = torch.zeros((cap, w.H, w.d), dtype=torch.float64)
        pad_o[:len(tokens)] = torch.from_numpy(out)
        all_t = [torch.empty_like(pad_t) for _ in range(WORLD)]
        all_o = [torch.empty_like(pad_o) for _ in range(WORLD)]
        dist.all_gather(all_t, pad_t)
        dist.all_gather(all_o, pad_o)
        # max-over-ranks timing, as bench.py reduces it
        ms = torch.tensor([1.5 + rank], dtype=torch.float64)
        dist.all_reduce(ms, op=dist.ReduceOp.MAX)
        if rank == 0:
            full = oracle.Problem.from_batch(b).fwd(b.q, b.k, b.v)
            got = np.zeros_like(full)
            seen = np.zeros(b.T, dtype=np.int64)
            for tt, oo in zip(all_t, all_o):
                keep = tt >= 0
                got[tt[keep].numpy()] = oo[keep].numpy()
                seen[tt[keep].numpy()] += 1
            np.save(os.path.join(result_dir, "check.npy"),
                    np.array([float(np.abs(got - full).max()), float(seen.min()),
                              float(seen.max()), float(ms.item())]))
    finally:
        dist.destroy_process_group()


def test_two_ranks_shard_by_sequence(tmp_path):
    port = _free_port()
    mp.start_processes(_worker, args=(port, str(tmp_path)), nprocs=WORLD, start_method="spawn",
                       join=True)
    err, seen_min, seen_max, ms = np.load(tmp_path / "check.npy")
    assert seen_min == 1 and seen_max == 1      # every token on exactly one rank
    assert err == 0.0                           # per-sequence results are independent of the split
    assert ms == 2.5                            # the job's time is the slowest rank's

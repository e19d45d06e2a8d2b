"""Host-side logic of the package: closed-form work accounting and the
multi-GPU sequence partition (no GPU needed)."""
import numpy as np
import pytest

import oracle
from sparse_hstu_attention_b200 import flops as F
from sparse_hstu_attention_b200.sharding import partition_sequences, shard_offsets
from workloads import WORKLOADS, draw_lengths, offsets_from_lengths


@pytest.mark.parametrize("lengths,nt,ctx,K1,K2", [
    ([1, 2, 3, 100, 257], 5, 3, 7, 2), ([300, 40], 0, 0, 0, 9), ([64, 64], 64, 0, 5, 0),
    ([500, 129, 1], 30, 40, 100000, 0), ([200], 12, 0, 1, 0), ([0, 77, 0], 8, 4, 16, 20),
])
def test_pair_counts_match_oracle(lengths, nt, ctx, K1, K2):
    lengths = np.array(lengths)
    nts = np.minimum(nt, lengths)
    p = oracle.Problem(offsets_from_lengths(lengths), nts, 1, 1, ctx, K1, K2, 1.0, 1.0)
    rows, keys = p.row_counts(), p.key_counts()
    rp, kp = F.pairs_per_token(lengths, nts, ctx, K1, K2)
    np.testing.assert_array_equal(rp, rows)
    np.testing.assert_array_equal(kp, keys)
    assert F.total_pairs(lengths, nts, ctx, K1, K2) == rows.sum() == keys.sum()


def test_workload_draws_follow_recipe():
    l3 = draw_lengths(WORKLOADS["hist16k"])
    assert len(l3) == 8 and (l3[:4] == 16384).all() and l3.sum() <= 96 * 1024
    assert ((l3[4:] >= 4096) & (l3[4:] <= 16384)).all()
    l2 = draw_lengths(WORKLOADS["mid"])
    assert len(l2) == 32 and l2.min() >= 1024 and l2.max() <= 4096
    assert (draw_lengths(WORKLOADS["infer"]) == 8704).all()
    np.testing.assert_array_equal(draw_lengths(WORKLOADS["mid"]), l2)  # seeded


@pytest.mark.parametrize("world", [1, 2, 3, 8])
def test_partition_covers_every_sequence_once(world):
    w = WORKLOADS["mid"]
    lengths = draw_lengths(w)
    nts = np.full(len(lengths), w.num_targets)
    owned = partition_sequences(lengths, nts, world, w.contextual_len, w.K1, w.K2)
    flat = sorted(b for o in owned for b in o)
    assert flat == list(range(len(lengths)))
    cost = F.pairs_per_sequence(lengths, nts, w.contextual_len, w.K1, w.K2)
    loads = [cost[o].sum() for o in owned]
    assert max(loads) - min(loads) <= cost.max()   # greedy LPT bound
    for o in owned:
        offs, toks = shard_offsets(lengths, o)
        assert offs[-1] == len(toks) == lengths[o].sum()


def test_candidate_pairs_match_oracle_row_counts():
    """The M-FALCON scoring work (pairs of candidate rows) equals the oracle's
    per-row counts summed over the candidate rows."""
    import oracle
    from sparse_hstu_attention_b200 import flops as F
    lengths, nts = np.array([40, 17, 90, 5]), np.array([6, 0, 30, 5])
    offs = np.concatenate([[0], np.cumsum(lengths)])
    for c, K1, K2 in [(2, 8, 3), (0, 0, 4), (5, 100, 0)]:
        p = oracle.Problem(offs, nts, 1, 4, c, K1, K2, 1.0, 1.0)
        rc = p.row_counts()
        want = sum(int(rc[offs[b + 1] - nts[b]:offs[b + 1]].sum()) for b in range(len(lengths)))
        assert F.candidate_pairs(lengths, nts, c, K1, K2) == want

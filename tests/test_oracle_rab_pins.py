"""Pins of the oracle's relative attention bias (HSTU notes, section 2.4,
Eq. 2: phi2(Q K^T + rab^{p,t}); the relative time encoding of the talk notes
"基于昇腾 NPU 的生成式推荐 Scaling Law 落地实践": bucketed timestamp difference,
table lookup, added to the scores).  Each compares the C oracle with
something written independently here:

  * the bucket function against the bit length of n + 1;
  * values and every gradient (q, k, v and both tables) against a dense
    fp64 torch formulation built from the definition (bias matrix by explicit
    loops, mask from the predicate), differentiated by autograd;
  * all-zero tables reproduce the bias-free results exactly;
  * central finite differences on table entries.
"""
import math

import numpy as np
import pytest
import torch

import oracle

NP, NT = 6, 8  # table sizes


def _timestamps(lengths, rng):
    """Non-decreasing integer timestamps per sequence (candidates after the
    history, as a request time)."""
    out = []
    for L in lengths:
        gaps = rng.exponential(3000.0, size=L).astype(np.int64)
        out.append(1_600_000_000 + np.cumsum(gaps))
    return np.concatenate(out).astype(np.int64)


def _case(seed=3):
    rng = np.random.default_rng(seed)
    lengths = np.array([21, 34, 9])
    nts = np.array([4, 6, 9])
    offs = np.concatenate([[0], np.cumsum(lengths)])
    T, H, d = int(offs[-1]), 2, 8
    q, k, v, do = (rng.standard_normal((T, H, d)) for _ in range(4))
    ts = _timestamps(lengths, rng)
    rp = rng.standard_normal((H, NP)) * 0.7
    rt = rng.standard_normal((H, NT)) * 0.7
    cfg = dict(H=H, d=d, contextual_len=2, K1=7, K2=3, alpha=0.4, N=40.0)
    return offs, nts, q, k, v, do, ts, rp, rt, cfg


def _bucket_ref(n, nb):
    return min(nb - 1, (int(max(n, 0)) + 1).bit_length() - 1)


def test_bucket_is_floor_log2_of_n_plus_1():
    for n in list(range(0, 300)) + [2 ** e - 2 for e in range(2, 40)] + \
            [2 ** e - 1 for e in range(1, 40)] + [2 ** e for e in range(1, 40)]:
        for nb in (1, 4, 17, 64):
            assert oracle.rab_bucket(n, nb) == _bucket_ref(n, nb), (n, nb)


def _dense(offs, nts, q, k, v, ts, rp, rt, cfg):
    """out and the autograd leaves of a dense per-sequence formulation."""
    H, alpha, N = cfg["H"], cfg["alpha"], cfg["N"]
    qt, kt, vt = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    rpt = torch.tensor(rp, dtype=torch.float64, requires_grad=True)
    rtt = torch.tensor(rt, dtype=torch.float64, requires_grad=True)
    outs = []
    for b in range(len(nts)):
        s0, s1 = int(offs[b]), int(offs[b + 1])
        L, Lh = s1 - s0, s1 - s0 - int(nts[b])
        M = torch.tensor(oracle.mask_matrix(L, int(nts[b]), cfg["contextual_len"], cfg["K1"],
                                            cfg["K2"]), dtype=torch.float64)
        bp = np.zeros((L, L), np.int64)
        bt = np.zeros((L, L), np.int64)
        for i in range(L):
            for j in range(L):
                dpos = i - j if i < Lh else (0 if j == i else Lh - j)
                bp[i, j] = _bucket_ref(dpos, NP)
                bt[i, j] = _bucket_ref(abs(int(ts[s0 + i]) - int(ts[s0 + j])), NT)
        for h in range(H):
            x = alpha * qt[s0:s1, h] @ kt[s0:s1, h].T + rpt[h][torch.from_numpy(bp)] + \
                rtt[h][torch.from_numpy(bt)]
            p = torch.nn.functional.silu(x) * M / N
            outs.append((s0, h, p @ vt[s0:s1, h]))
    out = torch.zeros(q.shape, dtype=torch.float64)
    for s0, h, o in outs:
        out[s0:s0 + o.shape[0], h] = o
    return out, (qt, kt, vt, rpt, rtt)


def test_values_and_gradients_match_a_dense_formulation():
    offs, nts, q, k, v, do, ts, rp, rt, cfg = _case()
    p = oracle.Problem(offs, nts, timestamps=ts, rab_pos=rp, rab_time=rt, **cfg)
    got = p.fwd(q, k, v)
    dq, dk, dv = p.bwd(q, k, v, do)
    drp, drt = p.bwd_rab(q, k, v, do)
    out, leaves = _dense(offs, nts, q, k, v, ts, rp, rt, cfg)
    np.testing.assert_allclose(got, out.detach().numpy(), rtol=1e-12, atol=1e-12)
    (out * torch.tensor(do)).sum().backward()
    for name, mine, leaf in zip(("dq", "dk", "dv", "d rab_pos", "d rab_time"),
                                (dq, dk, dv, drp, drt), leaves):
        np.testing.assert_allclose(mine, leaf.grad.numpy(), rtol=1e-10, atol=1e-12,
                                   err_msg=name)
    assert np.abs(drp).max() > 0 and np.abs(drt).max() > 0


def test_zero_tables_are_the_bias_free_attention():
    offs, nts, q, k, v, do, ts, rp, rt, cfg = _case(5)
    plain = oracle.Problem(offs, nts, **cfg)
    zero = oracle.Problem(offs, nts, timestamps=ts, rab_pos=np.zeros_like(rp),
                          rab_time=np.zeros_like(rt), **cfg)
    assert np.array_equal(plain.fwd(q, k, v), zero.fwd(q, k, v))
    for a, b in zip(plain.bwd(q, k, v, do), zero.bwd(q, k, v, do)):
        assert np.array_equal(a, b)


@pytest.mark.parametrize("table,h,b", [("pos", 0, 0), ("pos", 1, 2), ("time", 0, 3),
                                       ("time", 1, 7)])
def test_table_gradient_by_finite_differences(table, h, b):
    offs, nts, q, k, v, do, ts, rp, rt, cfg = _case(7)

    def loss(rp_, rt_):
        p = oracle.Problem(offs, nts, timestamps=ts, rab_pos=rp_, rab_time=rt_, **cfg)
        return float((p.fwd(q, k, v) * do).sum())

    p = oracle.Problem(offs, nts, timestamps=ts, rab_pos=rp, rab_time=rt, **cfg)
    g = p.bwd_rab(q, k, v, do)[0 if table == "pos" else 1][h, b]
    eps = 1e-6
    plus_p, minus_p, plus_t, minus_t = rp.copy(), rp.copy(), rt.copy(), rt.copy()
    if table == "pos":
        plus_p[h, b] += eps
        minus_p[h, b] -= eps
    else:
        plus_t[h, b] += eps
        minus_t[h, b] -= eps
    fd = (loss(plus_p, plus_t) - loss(minus_p, minus_t)) / (2 * eps)
    assert math.isclose(g, fd, rel_tol=1e-6, abs_tol=1e-9), (g, fd)


def test_both_tables_sum_the_same_pairs():
    """Each unmasked pair adds its gradient to one position bucket and one
    time bucket, so per head the two tables' gradients have equal totals."""
    offs, nts, q, k, v, do, ts, rp, rt, cfg = _case(11)
    p = oracle.Problem(offs, nts, timestamps=ts, rab_pos=rp, rab_time=rt, **cfg)
    dp, dt = p.bwd_rab(q, k, v, do)
    np.testing.assert_allclose(dp.sum(axis=1), dt.sum(axis=1), rtol=1e-12, atol=1e-12)

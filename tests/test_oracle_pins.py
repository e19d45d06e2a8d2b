"""Pins for the CPU oracle: each test ties it to something other than itself.

- the M-FALCON mask figure of the HSTU notes (golden fixture);
- Eq. 7 of "Bending the Scaling Law Curve..." (section 4.2.1) in its literal
  index form, under the row reversal that makes it causal;
- closed-form per-row pair counts (the O((K1+K2) L) cost claim made exact);
- full causal HSTU attention (Eq. 6) when K1 >= L, built with np.tril;
- a pure sliding window (K2 = contextual = 0) and a prefix-only mask (K1 = 0),
  built from band / column slices;
- dense masked attention in numpy and its gradient by torch autograd (fp64);
- central finite differences of the oracle's own forward;
- invariants: linearity in V, 1/N scaling, q = 0, candidate permutation,
  causality, jagged independence.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from workloads import WORKLOADS, make_batch, offsets_from_lengths

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _silu(x):
    return x / (1.0 + np.exp(-x))


def _closed_form_counts(L, nt, ctx, K1, K2):
    """Visible keys per row: history row i sees min(i+1, K1+K2eff) keys; a
    candidate sees min(Lh, K2eff + max(K1-1, 0)) history keys plus itself."""
    K2e = max(K2, ctx)
    Lh = L - nt
    hist = [min(i + 1, K1 + K2e) for i in range(Lh)]
    tgt = [min(Lh, K2e + max(K1 - 1, 0)) + 1] * nt
    return np.array(hist + tgt, dtype=np.int64)


def _dense_mask_textbook(L, nt, ctx, K1, K2):
    """The mask assembled from textbook pieces: lower triangle (Eq. 6), a band
    of K1 diagonals, the first K2eff columns, candidate rows = history block of
    the first candidate plus the identity."""
    K2e = max(K2, ctx)
    Lh = L - nt
    ones = np.ones((L, L), dtype=bool)
    tril = np.tril(ones)
    band = np.tril(ones) & ~np.tril(ones, -K1) if K1 > 0 else np.zeros((L, L), bool)
    prefix = np.zeros((L, L), bool)
    prefix[:, :min(K2e, L)] = True
    hist = tril & (band | prefix)
    m = np.zeros((L, L), bool)
    m[:Lh] = hist[:Lh]
    if nt > 0:
        # a candidate behaves like a history token at position Lh for the history ...
        row = (band | prefix)[Lh] if Lh < L else np.zeros(L, bool)
        row = row.copy()
        row[Lh:] = False
        m[Lh:, :] = row[None, :]
        # ... and sees itself
        m[np.arange(Lh, L), np.arange(Lh, L)] = True
    return m.astype(np.int64)


def _dense_forward(q, k, v, offs, nts, ctx, K1, K2, alpha, N, mask_fn=_dense_mask_textbook):
    out = np.zeros_like(q)
    for b in range(len(offs) - 1):
        s0, s1 = offs[b], offs[b + 1]
        L = s1 - s0
        m = mask_fn(L, nts[b], ctx, K1, K2)
        for h in range(q.shape[1]):
            s = alpha * q[s0:s1, h] @ k[s0:s1, h].T
            p = _silu(s) * m / N
            out[s0:s1, h] = p @ v[s0:s1, h]
    return out


def _rand(T, H, d, seed):
    rng = np.random.default_rng(seed)
    return [rng.standard_normal((T, H, d)) for _ in range(4)]


# --------------------------------------------------------------------------- mask


def test_mfalcon_golden_mask():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "mfalcon_mask.txt"))
            if l.strip() and not l.startswith("#")]
    fig = np.array(rows, dtype=np.int64)
    L, nt = fig.shape[0], 3
    got = oracle.mask_matrix(L, nt, contextual_len=0, K1=10 ** 6, K2=0)
    np.testing.assert_array_equal(got, fig)


@pytest.mark.parametrize("L,K1,K2", [(12, 3, 2), (20, 5, 0), (9, 1, 4), (16, 16, 3)])
def test_eq7_literal_form(L, K1, K2):
    """Eq. 7 as printed: M=1 if L-K1 <= i+j <= L, or if j <= K2 and j <= L-i.
    With rows counted from the end (r = L - i, 1-based key j) it is causal and
    equals the oracle's inclusive-window variant."""
    eq7 = np.zeros((L, L), np.int64)
    for i in range(L):            # equation's row index, r = L - i in 1..L
        for j in range(1, L + 1):  # equation's key index, 1-based
            local = (L - K1 <= i + j) and (i + j <= L)
            glob = (j <= K2) and (j <= L - i)
            eq7[i, j - 1] = int(local or glob)
    ours = oracle.mask_matrix(L, 0, 0, K1, K2, flags=oracle.INCLUSIVE_WINDOW)
    np.testing.assert_array_equal(eq7, ours[::-1, :])


def _count_cases():
    rng = np.random.default_rng(7)
    cases = [(1, 0, 0, 0, 0), (1, 1, 0, 1, 0), (5, 5, 0, 3, 1), (40, 0, 0, 0, 0),
             (40, 8, 4, 0, 0), (40, 8, 4, 0, 16), (40, 0, 50, 7, 0), (64, 64, 0, 0, 0),
             (64, 10, 0, 100, 0), (33, 3, 2, 1, 1)]
    for _ in range(60):
        L = int(rng.integers(1, 120))
        nt = int(rng.integers(0, L + 1))
        cases.append((L, nt, int(rng.integers(0, 20)), int(rng.integers(0, 70)),
                      int(rng.integers(0, 30))))
    return cases


@pytest.mark.parametrize("L,nt,ctx,K1,K2", _count_cases())
def test_row_counts_closed_form(L, nt, ctx, K1, K2):
    p = oracle.Problem([0, L], [nt], 1, 1, ctx, K1, K2, 1.0, 1.0)
    np.testing.assert_array_equal(p.row_counts(), _closed_form_counts(L, nt, ctx, K1, K2))


def test_key_counts_are_column_sums():
    for (L, nt, ctx, K1, K2) in _count_cases()[:30]:
        p = oracle.Problem([0, L], [nt], 1, 1, ctx, K1, K2, 1.0, 1.0)
        np.testing.assert_array_equal(p.key_counts(),
                                      _dense_mask_textbook(L, nt, ctx, K1, K2).sum(axis=0))


def test_mask_matches_textbook_pieces():
    for (L, nt, ctx, K1, K2) in _count_cases()[:40]:
        np.testing.assert_array_equal(oracle.mask_matrix(L, nt, ctx, K1, K2),
                                      _dense_mask_textbook(L, nt, ctx, K1, K2))


def test_full_causal_when_window_covers_sequence():
    """K1 >= L, no prefix, no candidates: the full causal mask of Eq. 6."""
    L = 37
    np.testing.assert_array_equal(oracle.mask_matrix(L, 0, 0, L, 0), np.tril(np.ones((L, L))))


def test_pure_window_and_prefix_only():
    L, K1, K2 = 30, 6, 5
    band = np.tril(np.ones((L, L))) - np.tril(np.ones((L, L)), -K1)
    np.testing.assert_array_equal(oracle.mask_matrix(L, 0, 0, K1, 0), band)
    pre = np.tril(np.ones((L, L)))
    pre[:, K2:] = 0
    np.testing.assert_array_equal(oracle.mask_matrix(L, 0, 0, 0, K2), pre)
    # the contextual prefix extends the global window (K2eff = max(K2, contextual))
    pre2 = np.tril(np.ones((L, L)))
    pre2[:, 9:] = 0
    np.testing.assert_array_equal(oracle.mask_matrix(L, 0, 9, 0, K2), pre2)


def test_unclamped_target_variant_differs_only_for_targets():
    L, nt, ctx, K1, K2 = 40, 10, 2, 5, 3
    a = oracle.mask_matrix(L, nt, ctx, K1, K2)
    b = oracle.mask_matrix(L, nt, ctx, K1, K2, flags=oracle.UNCLAMPED_TARGETS)
    np.testing.assert_array_equal(a[:L - nt], b[:L - nt])
    assert (a[L - nt:] != b[L - nt:]).any()


# ------------------------------------------------------------------ attention values


@pytest.mark.parametrize("lengths,nt,ctx,K1,K2,H,d", [
    ([7, 33, 1, 20], 3, 2, 4, 3, 2, 8),
    ([50], 0, 0, 100, 0, 1, 16),      # full causal
    ([45, 12], 0, 0, 6, 0, 2, 4),     # pure sliding window
    ([45, 12], 5, 0, 0, 7, 2, 4),     # prefix only, candidates
    ([30, 30, 2], 30, 0, 3, 1, 1, 8),  # a batch of candidates only
    ([64, 3], 2, 40, 9, 2, 3, 8),     # contextual longer than a sequence
])
def test_fwd_matches_dense(lengths, nt, ctx, K1, K2, H, d):
    offs = offsets_from_lengths(lengths)
    nts = np.minimum(nt, np.array(lengths))
    q, k, v, _ = _rand(int(offs[-1]), H, d, 11)
    alpha, N = 0.37, 13.0
    p = oracle.Problem(offs, nts, H, d, ctx, K1, K2, alpha, N)
    np.testing.assert_allclose(p.fwd(q, k, v),
                               _dense_forward(q, k, v, offs, nts, ctx, K1, K2, alpha, N),
                               rtol=1e-12, atol=1e-12)


def test_fwd_full_causal_is_textbook_hstu():
    """K1 >= L: out = (SiLU(alpha Q K^T) (.) tril) V / N, HSTU Eq. 3 with Eq. 6's mask."""
    L, H, d = 41, 2, 8
    q, k, v, _ = _rand(L, H, d, 3)
    p = oracle.Problem([0, L], [0], H, d, 0, 10 ** 6, 0, 0.5, 7.0)
    ref = np.stack([(_silu(0.5 * q[:, h] @ k[:, h].T) * np.tril(np.ones((L, L)))) @ v[:, h] / 7.0
                    for h in range(H)], axis=1)
    np.testing.assert_allclose(p.fwd(q, k, v), ref, rtol=1e-12, atol=1e-13)


def test_tiny_workload_bf16_matches_dense():
    w = WORKLOADS["tiny"]
    b = make_batch(w)
    q, k, v = (t.double().numpy() for t in (b.q, b.k, b.v))
    p = oracle.Problem.from_batch(b)
    np.testing.assert_allclose(
        p.fwd(q, k, v),
        _dense_forward(q, k, v, b.seq_offsets, b.num_targets, w.contextual_len, w.K1, w.K2,
                       w.alpha, w.N), rtol=1e-11, atol=1e-12)


def _torch_dense_grads(q, k, v, dout, offs, nts, ctx, K1, K2, alpha, N):
    tq, tk, tv = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v))
    outs = []
    for b in range(len(offs) - 1):
        s0, s1 = int(offs[b]), int(offs[b + 1])
        m = torch.tensor(_dense_mask_textbook(s1 - s0, int(nts[b]), ctx, K1, K2),
                         dtype=torch.float64)
        heads = []
        for h in range(q.shape[1]):
            s = alpha * tq[s0:s1, h] @ tk[s0:s1, h].T
            heads.append((torch.nn.functional.silu(s) * m / N) @ tv[s0:s1, h])
        outs.append(torch.stack(heads, 1))
    out = torch.cat(outs, 0)
    (out * torch.tensor(dout)).sum().backward()
    return tq.grad.numpy(), tk.grad.numpy(), tv.grad.numpy()


@pytest.mark.parametrize("lengths,nt,ctx,K1,K2", [
    ([9, 31, 2], 4, 3, 5, 2),
    ([40], 0, 0, 100, 0),
    ([25, 25], 25, 0, 4, 0),
    ([33], 6, 0, 0, 5),
])
def test_bwd_matches_torch_autograd_dense(lengths, nt, ctx, K1, K2):
    offs = offsets_from_lengths(lengths)
    nts = np.minimum(nt, np.array(lengths))
    H, d = 2, 8
    q, k, v, dout = _rand(int(offs[-1]), H, d, 5)
    alpha, N = 0.6, 3.0
    p = oracle.Problem(offs, nts, H, d, ctx, K1, K2, alpha, N)
    dq, dk, dv = p.bwd(q, k, v, dout)
    rq, rk, rv = _torch_dense_grads(q, k, v, dout, offs, nts, ctx, K1, K2, alpha, N)
    for a, r in ((dq, rq), (dk, rk), (dv, rv)):
        np.testing.assert_allclose(a, r, rtol=1e-11, atol=1e-12)


def test_bwd_finite_differences():
    """Central differences of L = sum(out * dout) at 200 random coordinates."""
    lengths, nt, ctx, K1, K2 = [23, 40], 5, 2, 6, 3
    offs = offsets_from_lengths(lengths)
    nts = np.array([nt, nt])
    H, d = 2, 8
    q, k, v, dout = _rand(int(offs[-1]), H, d, 9)
    alpha, N = 0.8, 5.0
    p = oracle.Problem(offs, nts, H, d, ctx, K1, K2, alpha, N)
    grads = dict(zip("qkv", p.bwd(q, k, v, dout)))
    rng = np.random.default_rng(1)
    eps = 1e-6
    for _ in range(200):
        which = "qkv"[rng.integers(3)]
        idx = (rng.integers(q.shape[0]), rng.integers(H), rng.integers(d))
        args = {"q": q.copy(), "k": k.copy(), "v": v.copy()}
        args[which][idx] += eps
        fp = (p.fwd(args["q"], args["k"], args["v"]) * dout).sum()
        args[which][idx] -= 2 * eps
        fm = (p.fwd(args["q"], args["k"], args["v"]) * dout).sum()
        fd = (fp - fm) / (2 * eps)
        an = grads[which][idx]
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (which, idx, fd, an)


# ------------------------------------------------------------------------ invariants


def _small_problem(seed=2):
    lengths = [17, 40, 5]
    offs = offsets_from_lengths(lengths)
    nts = np.array([3, 6, 5])
    H, d = 2, 8
    q, k, v, dout = _rand(int(offs[-1]), H, d, seed)
    p = oracle.Problem(offs, nts, H, d, 2, 7, 3, 0.45, 11.0)
    return p, offs, nts, q, k, v, dout


def test_linear_in_v_and_scales_with_n():
    p, offs, nts, q, k, v, dout = _small_problem()
    v2 = np.random.default_rng(4).standard_normal(v.shape)
    np.testing.assert_allclose(p.fwd(q, k, 2 * v + v2), 2 * p.fwd(q, k, v) + p.fwd(q, k, v2),
                               rtol=1e-12, atol=1e-12)
    p2 = oracle.Problem(offs, nts, 2, 8, 2, 7, 3, 0.45, 22.0)
    np.testing.assert_allclose(p2.fwd(q, k, v), 0.5 * p.fwd(q, k, v), rtol=1e-13)
    assert np.all(p.fwd(np.zeros_like(q), k, v) == 0.0)


def test_candidates_are_independent_and_permutable():
    p, offs, nts, q, k, v, dout = _small_problem()
    out = p.fwd(q, k, v)
    s0, s1 = offs[1], offs[2]
    tgt = np.arange(s1 - nts[1], s1)
    perm = np.arange(q.shape[0])
    perm[tgt] = tgt[::-1]
    outp = p.fwd(q[perm], k[perm], v[perm])
    np.testing.assert_allclose(outp, out[perm], rtol=1e-12, atol=1e-14)
    # history rows do not depend on any candidate's k / v
    k2, v2 = k.copy(), v.copy()
    k2[tgt] += 3.0
    v2[tgt] -= 1.0
    out2 = p.fwd(q, k2, v2)
    hist = np.arange(s0, s1 - nts[1])
    np.testing.assert_array_equal(out2[hist], out[hist])


def test_jagged_sequences_are_independent():
    p, offs, nts, q, k, v, dout = _small_problem()
    out = p.fwd(q, k, v)
    dq, dk, dv = p.bwd(q, k, v, dout)
    for b in range(len(offs) - 1):
        s0, s1 = offs[b], offs[b + 1]
        pb = oracle.Problem([0, s1 - s0], [nts[b]], 2, 8, 2, 7, 3, 0.45, 11.0)
        np.testing.assert_array_equal(pb.fwd(q[s0:s1], k[s0:s1], v[s0:s1]), out[s0:s1])
        gq, gk, gv = pb.bwd(q[s0:s1], k[s0:s1], v[s0:s1], dout[s0:s1])
        np.testing.assert_array_equal(gq, dq[s0:s1])
        np.testing.assert_array_equal(gk, dk[s0:s1])
        np.testing.assert_array_equal(gv, dv[s0:s1])


def test_sampled_rows_equal_full():
    p, offs, nts, q, k, v, dout = _small_problem()
    rows = np.array([0, 5, 16, 17, 30, 56, 61])
    np.testing.assert_array_equal(p.fwd(q, k, v, rows=rows), p.fwd(q, k, v)[rows])
    np.testing.assert_array_equal(p.bwd_dq(q, k, v, dout, rows=rows),
                                  p.bwd_dq(q, k, v, dout)[rows])
    dk, dv = p.bwd_dkv(q, k, v, dout, keys=rows)
    fk, fv = p.bwd_dkv(q, k, v, dout)
    np.testing.assert_array_equal(dk, fk[rows])
    np.testing.assert_array_equal(dv, fv[rows])


def test_planted_mistake_is_caught():
    """A window off by one (Eq. 7's literal '<=') breaks the closed-form counts."""
    L, nt, ctx, K1, K2 = 50, 4, 2, 6, 3
    p = oracle.Problem([0, L], [nt], 1, 1, ctx, K1, K2, 1.0, 1.0, flags=oracle.INCLUSIVE_WINDOW)
    assert (p.row_counts() != _closed_form_counts(L, nt, ctx, K1, K2)).any()

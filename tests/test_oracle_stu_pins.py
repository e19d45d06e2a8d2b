"""Pins of the STU-layer / STU-stack oracle (oracle/stu.py) to facts that do not
come from the oracle itself: finite differences (the backward against the
forward), LayerNorm moments, the residual identity, the block order of the
U, V, Q, K split (through weight blocks set to zero), and the truncation
rule checked through properties of the kept set.  CPU only."""
import numpy as np
import pytest

from oracle import stu as S
from workloads import offsets_from_lengths

LENGTHS = np.array([9, 14, 6])
NTS = np.array([2, 3, 1])
CFG = S.AttnCfg(H=2, d=4, contextual_len=1, K1=4, K2=2, alpha=0.5, N=10.0, eps=1e-5)
DM = CFG.H * CFG.d


def _weights(rng, dm=DM, scale=0.4):
    return S.Weights.of(ln1_w=1 + 0.2 * rng.standard_normal(dm), ln1_b=0.2 * rng.standard_normal(dm),
                        w1=scale * rng.standard_normal((dm, 4 * dm)),
                        b1=0.2 * rng.standard_normal(4 * dm),
                        ln2_w=1 + 0.2 * rng.standard_normal(dm), ln2_b=0.2 * rng.standard_normal(dm),
                        w2=scale * rng.standard_normal((dm, dm)), b2=0.2 * rng.standard_normal(dm))


def _fd_check(f, x, grad, coords, h=1e-6, tol=1e-6):
    """Central differences of the scalar f at flat coordinates of x."""
    flat = x.reshape(-1)
    for c in coords:
        old = flat[c]
        flat[c] = old + h
        up = f()
        flat[c] = old - h
        dn = f()
        flat[c] = old
        fd = (up - dn) / (2 * h)
        g = grad.reshape(-1)[c]
        assert abs(fd - g) <= tol * max(1.0, abs(fd)), (c, fd, g)


def test_layer_gradients_match_finite_differences():
    rng = np.random.default_rng(7)
    offs = offsets_from_lengths(LENGTHS)
    T = int(offs[-1])
    x = rng.standard_normal((T, DM))
    w = _weights(rng)
    dout = rng.standard_normal((T, DM))

    def loss():
        out, _ = S.layer_fwd(x, w, offs, NTS, CFG)
        return float((out * dout).sum())

    out, cache = S.layer_fwd(x, w, offs, NTS, CFG)
    dx, g = S.layer_bwd(dout, w, cache)
    _fd_check(loss, x, dx, rng.choice(x.size, 24, replace=False))
    for name in ("ln1_w", "ln1_b", "w1", "b1", "ln2_w", "ln2_b", "w2", "b2"):
        p = getattr(w, name)
        _fd_check(loss, p, getattr(g, name), rng.choice(p.size, min(8, p.size), replace=False))


def test_stack_gradients_match_finite_differences():
    """Three layers, truncation after the first (tail 2): the scatter of the
    gradient into the full layout and the per-stage N are exercised."""
    rng = np.random.default_rng(11)
    offs = offsets_from_lengths(LENGTHS)
    T = int(offs[-1])
    x = rng.standard_normal((T, DM))
    ws = [_weights(rng, scale=0.3) for _ in range(3)]
    cfg2 = S.AttnCfg(**{**CFG.__dict__, "N": 7.0})
    idx, _ = S.truncation_index(offs, NTS, CFG.contextual_len, 2)
    dout = rng.standard_normal((len(idx), DM))

    def loss():
        out, _ = S.stack_fwd(x, ws, offs, NTS, CFG, cfg2, 1, 2)
        return float((out * dout).sum())

    out, cache = S.stack_fwd(x, ws, offs, NTS, CFG, cfg2, 1, 2)
    dx, gs = S.stack_bwd(dout, ws, cache)
    _fd_check(loss, x, dx, rng.choice(x.size, 24, replace=False))
    for i in (0, 2):
        _fd_check(loss, ws[i].w1, gs[i].w1, rng.choice(ws[i].w1.size, 6, replace=False))
        _fd_check(loss, ws[i].ln2_w, gs[i].ln2_w, rng.choice(DM, 4, replace=False))
    # dropped rows get no gradient through the truncated layers, only through
    # layer 0 (which sees every row): rows dropped before layer 1 still move
    dropped = np.setdiff1d(np.arange(T), idx)
    assert len(dropped) > 0 and np.abs(dx[dropped]).sum() > 0


def test_layernorm_moments():
    rng = np.random.default_rng(3)
    x = 3.0 + 2.0 * rng.standard_normal((50, 64))
    y, xh, rstd = S.layer_norm(x, np.ones(64), np.zeros(64), 1e-5)
    var = x.var(axis=1)
    assert np.allclose(y.mean(axis=1), 0.0, atol=1e-12)
    # biased variance of the output: var / (var + eps)
    assert np.allclose(y.var(axis=1), var / (var + 1e-5), rtol=1e-12)
    assert np.allclose(rstd[:, 0], 1.0 / np.sqrt(var + 1e-5))


def test_residual_identity():
    """With the output map zero the layer returns its input exactly."""
    rng = np.random.default_rng(5)
    offs = offsets_from_lengths(LENGTHS)
    x = rng.standard_normal((int(offs[-1]), DM))
    w = _weights(rng)
    w.w2[:] = 0.0
    w.b2[:] = 0.0
    out, _ = S.layer_fwd(x, w, offs, NTS, CFG)
    assert np.array_equal(out, x)


def test_block_order_of_the_split():
    """Blocks are U, V, Q, K (column blocks 0..3 of the projection).
    With the V block zeroed the attention output is 0 whatever Q and K are,
    so the layer reduces to out = x + (ln2_b * U) W2 + b2 with U from block 0;
    and perturbing the Q and K blocks then changes nothing."""
    rng = np.random.default_rng(9)
    offs = offsets_from_lengths(LENGTHS)
    x = rng.standard_normal((int(offs[-1]), DM))
    w = _weights(rng)
    w.w1[:, DM:2 * DM] = 0.0
    w.b1[DM:2 * DM] = 0.0
    out, _ = S.layer_fwd(x, w, offs, NTS, CFG)
    mu = x.mean(1, keepdims=True)
    xn = (x - mu) / np.sqrt(x.var(1, keepdims=True) + CFG.eps) * w.ln1_w + w.ln1_b
    pre_u = xn @ w.w1[:, :DM] + w.b1[:DM]
    u = pre_u / (1 + np.exp(-pre_u))
    assert np.allclose(out, x + (w.ln2_b * u) @ w.w2 + w.b2, rtol=1e-12, atol=1e-12)
    w.w1[:, 2 * DM:] += rng.standard_normal((DM, 2 * DM))
    out2, _ = S.layer_fwd(x, w, offs, NTS, CFG)
    assert np.allclose(out2, out, rtol=1e-12, atol=1e-12)
    # and with the Q block zeroed the scores vanish: SiLU(0) = 0, so A = 0 too
    w = _weights(rng)
    w.w1[:, 2 * DM:3 * DM] = 0.0
    w.b1[2 * DM:3 * DM] = 0.0
    out3, c3 = S.layer_fwd(x, w, offs, NTS, CFG)
    assert np.abs(c3["av"]).max() == 0.0


@pytest.mark.parametrize("c,tail", [(1, 2), (0, 3), (4, 100), (2, 0)])
def test_truncation_keeps_what_the_rule_names(c, tail):
    """Per sequence: all contextual and candidate rows survive, order is kept,
    and the surviving history rows past the prefix are the `tail` latest ones
    (all of them when there are no more than `tail`)."""
    lengths = np.array([40, 9, 17, 3])
    nts = np.array([5, 2, 0, 3])
    offs = offsets_from_lengths(lengths)
    idx, new = S.truncation_index(offs, nts, c, tail)
    assert len(idx) == new[-1] and np.all(np.diff(new) >= 0)
    for b in range(len(lengths)):
        keep = idx[new[b]:new[b + 1]] - offs[b]
        L, Lh = lengths[b], lengths[b] - nts[b]
        assert np.all(np.diff(keep) > 0)
        ks = set(keep.tolist())
        assert set(range(min(c, Lh))) <= ks            # contextual prefix
        assert set(range(Lh, L)) <= ks                 # candidates
        hist = sorted(p for p in ks if min(c, Lh) <= p < Lh)
        uih = list(range(min(c, Lh), Lh))
        assert hist == uih[max(0, len(uih) - tail):]   # the latest `tail` history rows

"""GPU parity of the relative attention bias (HSTU notes, section 2.4, Eq. 2:
phi2(Q K^T + rab^{p,t})): forward, dq, dk, dv and both tables' gradients
against the oracle on seeded inputs (TOL of max|ref| per tensor), each table
alone, all-zero tables equal to the bias-free kernels, the forward at
head_dim 64, the refusal of the backward at head_dim 64, and grouped calls
with a bias on some of their problems."""
import numpy as np
import pytest
import torch

import oracle
import sparse_hstu_attention_b200 as sla
from sparse_hstu_attention_b200 import _abi
from workloads import WORKLOADS, draw_rab_tables, draw_timestamps, make_batch, with_params

from parity import TOL, assert_close, kwargs_of, to_gpu

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")
NP, NT = 12, 24


def _case(lengths=(300, 1200, 77, 640, 129), nt=16, H=4, d=128, K1=256, K2=64, ctx=16, seed=21):
    w = with_params(WORKLOADS["tiny"], H=H, d=d, K1=K1, K2=K2, contextual_len=ctx,
                    num_targets=nt, alpha=d ** -0.5, N=float(max(lengths)))
    lengths = np.array(lengths, dtype=np.int64)
    b = make_batch(w, lengths=lengths, num_targets=np.minimum(nt, lengths), seed=seed)
    ts = draw_timestamps(b.lengths, b.num_targets, seed)
    rp, rt = draw_rab_tables(H, NP, NT, seed)
    return b, ts, rp, rt


def _run(b, ts, rp, rt, bwd=True):
    g = to_gpu(b)
    rab = dict(timestamps=torch.from_numpy(ts).to(DEV),
               rab_pos=None if rp is None else rp.to(DEV),
               rab_time=None if rt is None else rt.to(DEV))
    out = sla.hstu_sla_fwd(g["q"], g["k"], g["v"], g["offs"], g["nts"], **kwargs_of(b), **rab)
    res = [out]
    if bwd:
        res += list(sla.hstu_sla_bwd(g["dout"], g["q"], g["k"], g["v"], g["offs"], g["nts"],
                                     **kwargs_of(b), **rab))
    torch.cuda.synchronize()
    return res


def _oracle(b, ts, rp, rt):
    w = b.workload
    return oracle.Problem(b.seq_offsets, b.num_targets, w.H, w.d, w.contextual_len, w.K1, w.K2,
                          w.alpha, w.N, timestamps=ts,
                          rab_pos=None if rp is None else rp.numpy(),
                          rab_time=None if rt is None else rt.numpy())


@pytest.mark.parametrize("tables", ["both", "pos", "time"])
def test_rab_forward_backward_and_table_gradients(tables):
    b, ts, rp, rt = _case()
    rp = rp if tables in ("both", "pos") else None
    rt = rt if tables in ("both", "time") else None
    out, dq, dk, dv, (drp, drt) = _run(b, ts, rp, rt)
    p = _oracle(b, ts, rp, rt)
    assert_close("out", out, p.fwd(b.q, b.k, b.v))
    rq, rk, rv = p.bwd(b.q, b.k, b.v, b.dout)
    assert_close("dq", dq, rq)
    assert_close("dk", dk, rk)
    assert_close("dv", dv, rv)
    rdp, rdt = p.bwd_rab(b.q, b.k, b.v, b.dout)
    if rp is not None:
        assert_close("d rab_pos", drp, rdp)
    if rt is not None:
        assert_close("d rab_time", drt, rdt)


def test_rab_edge_batch():
    """Ragged tiles, a sequence of candidates only, K1 = 0 (prefix only) and
    candidate self-pairs in their own bucket."""
    b, ts, rp, rt = _case(lengths=(1, 130, 64, 65, 257, 9), nt=9, K1=0, K2=40, ctx=8, seed=5)
    out, dq, dk, dv, (drp, drt) = _run(b, ts, rp, rt)
    p = _oracle(b, ts, rp, rt)
    assert_close("out", out, p.fwd(b.q, b.k, b.v))
    rq, rk, rv = p.bwd(b.q, b.k, b.v, b.dout)
    for name, got, ref in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        assert_close(name, got, ref)
    rdp, rdt = p.bwd_rab(b.q, b.k, b.v, b.dout)
    assert_close("d rab_pos", drp, rdp)
    assert_close("d rab_time", drt, rdt)


def test_rab_timestamps_over_the_whole_int32_range():
    """Unsorted timestamps drawn over all of int32 (both ends included) next
    to small ones: differences up to 2^32 - 1, the cap at 2^31 - 1 and every
    time bucket up to 31 of a 32-bucket table, plus a 5-bucket position
    table (most pairs past its last bucket)."""
    b, _, _, _ = _case(lengths=(190, 333, 64, 9), seed=13)
    rng = np.random.default_rng(13)
    T = int(b.seq_offsets[-1])
    wide = rng.integers(-2 ** 31, 2 ** 31, size=T, dtype=np.int64)
    small = rng.integers(-5000, 5000, size=T, dtype=np.int64)
    ts = np.where(rng.random(T) < 0.5, wide, small)
    ts[:6] = [-2 ** 31, 2 ** 31 - 1, 0, -1, 2 ** 31 - 2, -2 ** 31 + 1]
    ts = ts.astype(np.int32)
    rp, rt = draw_rab_tables(b.workload.H, 5, 32, 13)
    out, dq, dk, dv, (drp, drt) = _run(b, ts, rp, rt)
    p = _oracle(b, ts, rp, rt)
    assert_close("out", out, p.fwd(b.q, b.k, b.v))
    rq, rk, rv = p.bwd(b.q, b.k, b.v, b.dout)
    for name, got, ref in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        assert_close(name, got, ref)
    rdp, rdt = p.bwd_rab(b.q, b.k, b.v, b.dout)
    assert_close("d rab_pos", drp, rdp)
    assert_close("d rab_time", drt, rdt)
    assert (np.abs(rdt[:, 30:]) > 0).all()  # the top buckets were reached


def test_zero_tables_equal_the_bias_free_kernels():
    b, ts, rp, rt = _case(seed=8)
    out, dq, dk, dv, _ = _run(b, ts, torch.zeros_like(rp), torch.zeros_like(rt))
    g = to_gpu(b)
    out0 = sla.hstu_sla_fwd(g["q"], g["k"], g["v"], g["offs"], g["nts"], **kwargs_of(b))
    dq0, dk0, dv0 = sla.hstu_sla_bwd(g["dout"], g["q"], g["k"], g["v"], g["offs"], g["nts"],
                                     **kwargs_of(b))
    torch.cuda.synchronize()
    assert torch.equal(out, out0)
    assert torch.equal(dk, dk0) and torch.equal(dv, dv0)
    assert_close("dq", dq, dq0.float().cpu().numpy().astype(np.float64), tol=1e-2)


def test_rab_forward_head_dim_64_and_refusal():
    b, ts, rp, rt = _case(lengths=(200, 77), H=3, d=64, K1=50, K2=8, ctx=4, seed=9)
    (out,) = _run(b, ts, rp, rt, bwd=False)
    assert_close("out d64", out, _oracle(b, ts, rp, rt).fwd(b.q, b.k, b.v))
    with pytest.raises(sla.SLAError) as ex:
        _run(b, ts, rp, rt)
    assert ex.value.code == _abi.ERR_UNSUPPORTED


def test_rab_in_grouped_calls():
    """Three problems in one grouped launch (MoT channels): both tables, the
    position table only, no bias.  Each against the oracle, and against its
    own single call: forward and dk / dv bitwise, the rest to fp32 order."""
    cases = [_case(lengths=(300, 700, 65), K1=256, K2=64, seed=41),
             _case(lengths=(129, 40, 520, 255), nt=8, K1=100, K2=16, ctx=4, seed=42),
             _case(lengths=(90, 333), nt=4, K1=64, K2=8, ctx=2, seed=43)]
    tables = [(True, True), (True, False), (False, False)]
    groups, singles = [], []
    for (b, ts, rp, rt), (use_p, use_t) in zip(cases, tables):
        rp, rt = (rp if use_p else None), (rt if use_t else None)
        g = to_gpu(b)
        rab = dict(timestamps=torch.from_numpy(ts).to(DEV),
                   rab_pos=None if rp is None else rp.to(DEV),
                   rab_time=None if rt is None else rt.to(DEV))
        groups.append(dict(q=g["q"], k=g["k"], v=g["v"], dout=g["dout"], seq_offsets=g["offs"],
                           num_targets=g["nts"], **kwargs_of(b), **rab))
        singles.append(_run(b, ts, rp, rt))
    outs = sla.hstu_sla_fwd_grouped(groups)
    grads = sla.hstu_sla_bwd_grouped(groups)
    torch.cuda.synchronize()
    for (b, ts, rp, rt), (use_p, use_t), out, gr, one in zip(cases, tables, outs, grads, singles):
        rp, rt = (rp if use_p else None), (rt if use_t else None)
        assert torch.equal(out, one[0])
        assert torch.equal(gr[1], one[2]) and torch.equal(gr[2], one[3])
        p = _oracle(b, ts, rp, rt)
        assert_close("out", out, p.fwd(b.q, b.k, b.v))
        rq, rk, rv = p.bwd(b.q, b.k, b.v, b.dout)
        for name, got, ref in (("dq", gr[0], rq), ("dk", gr[1], rk), ("dv", gr[2], rv)):
            assert_close(name, got, ref)
        if rp is None and rt is None:
            assert len(gr) == 3
            continue
        rdp, rdt = p.bwd_rab(b.q, b.k, b.v, b.dout)
        drp, drt = gr[3]
        assert_close("d rab_pos", drp, rdp)
        if rt is None:
            assert drt is None
        else:
            assert_close("d rab_time", drt, rdt)
        for mine, single in zip(gr[3], one[4]):
            if mine is not None:
                assert torch.allclose(mine, single, rtol=1e-5, atol=1e-6 * float(single.abs().max()))


def _table_totals_agree(drp, drt):
    """Both tables partition the same unmasked pairs into buckets, so per
    head their gradients have the same total (up to fp32 summation)."""
    sp, st = drp.double().sum(dim=1), drt.double().sum(dim=1)
    scale = float(drp.double().abs().sum()) + float(drt.double().abs().sum())
    assert torch.allclose(sp, st, atol=1e-4 * scale, rtol=0), (sp, st)


def test_rab_full_size_sampled():
    """hist16k at full size with both tables: forward and dq on sampled rows,
    dk and dv on sampled keys against the oracle one by one; the tables'
    gradients are checked by the equal-totals invariant and for finiteness."""
    from parity import sample_tokens
    b = make_batch(WORKLOADS["hist16k"])
    ts = draw_timestamps(b.lengths, b.num_targets, b.workload.seed)
    rp, rt = draw_rab_tables(b.workload.H, 32, 32, b.workload.seed)
    out, dq, dk, dv, (drp, drt) = _run(b, ts, rp, rt)
    p = _oracle(b, ts, rp, rt)
    rows = sample_tokens(b, 120, seed=11)
    keys = sample_tokens(b, 120, seed=12)
    assert_close("out", out[rows], p.fwd(b.q, b.k, b.v, rows=rows))
    assert_close("dq", dq[rows], p.bwd_dq(b.q, b.k, b.v, b.dout, rows=rows))
    rk, rv = p.bwd_dkv(b.q, b.k, b.v, b.dout, keys=keys)
    assert_close("dk", dk[keys], rk)
    assert_close("dv", dv[keys], rv)
    for t in (out, dq, dk, dv, drp, drt):
        assert torch.isfinite(t.float()).all()
    _table_totals_agree(drp, drt)


def test_rab_table_totals_small():
    b, ts, rp, rt = _case(seed=31)
    *_, (drp, drt) = _run(b, ts, rp, rt)
    _table_totals_agree(drp, drt)

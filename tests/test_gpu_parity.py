"""GPU parity: the CUDA library (through its C ABI) against the oracle on the
same seeded bf16 inputs.  Floating point: max|gpu - ref| <= 2e-2 * max|ref|
per tensor (out, dq, dk, dv).  Pair counts: exact."""
import numpy as np
import pytest
import torch

import sparse_hstu_attention_b200 as sla
from workloads import WORKLOADS, make_batch, with_params

from parity import (TOL, assert_close, gpu_bwd, gpu_fwd, kwargs_of, oracle_problem,
                    sample_tokens, to_gpu)

pytestmark = pytest.mark.gpu


def _edge_batch(lengths, nt, H=2, d=128, K1=40, K2=10, ctx=3, seed=5, alpha=None, N=300.0):
    w = with_params(WORKLOADS["tiny"], H=H, d=d, K1=K1, K2=K2, contextual_len=ctx,
                    num_targets=nt, alpha=alpha if alpha is not None else d ** -0.5, N=N)
    lengths = np.array(lengths, dtype=np.int64)
    return make_batch(w, lengths=lengths, num_targets=np.minimum(nt, lengths), seed=seed)


def _full_check(batch, strided=False, fwd=True, bwd=True):
    g = to_gpu(batch, strided=strided)
    p = oracle_problem(batch)
    if fwd:
        out = gpu_fwd(batch, g)
        assert_close("out", out, p.fwd(batch.q, batch.k, batch.v))
    if bwd:
        dq, dk, dv = gpu_bwd(batch, g)
        rq, rk, rv = p.bwd(batch.q, batch.k, batch.v, batch.dout)
        assert_close("dq", dq, rq)
        assert_close("dk", dk, rk)
        assert_close("dv", dv, rv)


def _count_check(batch):
    g = to_gpu(batch)
    w = batch.workload
    rows, keys = sla.hstu_sla_count_pairs(g["q"], g["k"], g["v"], g["offs"], g["nts"],
                                          contextual_len=w.contextual_len, K1=w.K1, K2=w.K2,
                                          max_seq_len=int(batch.lengths.max()))
    p = oracle_problem(batch)
    np.testing.assert_array_equal(rows.cpu().numpy(), p.row_counts())
    np.testing.assert_array_equal(keys.cpu().numpy(), p.key_counts())


def test_tiny_workload_full():
    b = make_batch(WORKLOADS["tiny"])
    _full_check(b)
    _count_check(b)


EDGE = {
    "ragged": dict(lengths=[1, 2, 17, 64, 65, 127, 128, 129, 300], nt=8),
    "all_candidates": dict(lengths=[5, 70, 130], nt=200),
    "no_candidates": dict(lengths=[190, 33], nt=0),
    "prefix_only_K1_0": dict(lengths=[150, 257], nt=6, K1=0),
    "window_K1_1": dict(lengths=[150, 97], nt=5, K1=1, K2=0, ctx=0),
    "pure_window": dict(lengths=[300, 64], nt=0, K1=50, K2=0, ctx=0),
    "full_causal": dict(lengths=[260, 31], nt=4, K1=100000, K2=0, ctx=0),
    "nothing_but_self": dict(lengths=[140], nt=20, K1=0, K2=0, ctx=0),
    "empty_sequences": dict(lengths=[0, 90, 0, 0, 200, 0], nt=7),
    "contextual_longer_than_seq": dict(lengths=[40, 300], nt=5, ctx=64, K2=2),
    "d64": dict(lengths=[200, 77], nt=9, d=64, H=3),
    "d32": dict(lengths=[200, 77], nt=9, d=32, H=4),
    "big_window_prefix": dict(lengths=[700], nt=64, K1=300, K2=130, ctx=32),
    # sequences one token past a tile boundary, followed by another sequence:
    # the last tile is partial and must stay masked
    "tile_edge_no_candidates": dict(lengths=[129, 300, 257, 65, 193, 64], nt=0, K1=100000,
                                    K2=0, ctx=0),
}


@pytest.mark.parametrize("name", sorted(EDGE))
def test_edge_cases(name):
    b = _edge_batch(**EDGE[name])
    _full_check(b)
    _count_check(b)


def test_strided_fused_projection_views():
    b = _edge_batch(lengths=[150, 260, 9], nt=12)
    _full_check(b, strided=True)


@pytest.mark.parametrize("d", [128, 64])
def test_repeat_calls_reproducible(d):
    """The forward, dk and dv have no atomics: bitwise identical across calls.
    dq at d = 128 sums fp32 partials with atomic additions in no fixed order,
    so two calls agree only to within the bf16 rounding of the same fp32
    sum; at d = 64 (query-tile pass, no atomics) dq is bitwise identical."""
    b = _edge_batch(lengths=[300, 200, 1000], nt=10, d=d)
    g = to_gpu(b)
    o1, o2 = gpu_fwd(b, g), gpu_fwd(b, g)
    assert torch.equal(o1, o2)
    (q1, k1, v1), (q2, k2, v2) = gpu_bwd(b, g), gpu_bwd(b, g)
    assert torch.equal(k1, k2) and torch.equal(v1, v2)
    if d == 128:
        # one bf16 ulp of the larger magnitude (2^-7 relative) bounds the gap,
        # plus a floor for sums that cancel to near zero
        a1, a2 = q1.float(), q2.float()
        bound = 2.0 ** -7 * torch.maximum(a1.abs(), a2.abs()) + 1e-4 * a1.abs().max()
        assert ((a1 - a2).abs() <= bound).all()
    else:
        assert torch.equal(q1, q2)


def test_long_prefix_units():
    """Sequences of ~8K tokens whose prefix key tiles (one or two of them, via
    K2) are each seen by every later row: one backward unit sweeps thousands
    of query steps.  Every tensor against the oracle, dk / dv bitwise
    repeatable; lengths ragged against the 64-row steps."""
    for K2 in (100, 250):
        b = _edge_batch(lengths=[8192 + 77, 8191, 2 * 2048 * 2 + 1], nt=20, K1=64, K2=K2, ctx=6,
                        seed=23)
        g = to_gpu(b)
        dq, dk, dv = gpu_bwd(b, g)
        p = oracle_problem(b)
        rq, rk, rv = p.bwd(b.q, b.k, b.v, b.dout)
        assert_close("dq", dq, rq)
        assert_close("dk", dk, rk)
        assert_close("dv", dv, rv)
        _, dk2, dv2 = gpu_bwd(b, g)
        assert torch.equal(dk, dk2) and torch.equal(dv, dv2)


def test_backward_reuses_a_workspace():
    """One workspace reused across backward calls (same batch, a larger one,
    the first again) gives the oracle's results every time."""
    b1 = _edge_batch(lengths=[300, 200, 1000], nt=10)
    b2 = _edge_batch(lengths=[700, 64, 1500, 90], nt=5, seed=9)
    need = max(sla.hstu_sla_workspace_bytes(1, b.T, len(b.lengths), 2, 128) for b in (b1, b2))
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    for b in (b1, b1, b2, b1):
        g = to_gpu(b)
        dq, dk, dv = sla.hstu_sla_bwd(g["dout"], g["q"], g["k"], g["v"], g["offs"], g["nts"],
                                      workspace=ws, **kwargs_of(b))
        assert sla.hstu_sla_get_error(ws) == 0
        p = oracle_problem(b)
        rq, rk, rv = p.bwd(b.q, b.k, b.v, b.dout)
        assert_close("dq", dq, rq)
        assert_close("dk", dk, rk)
        assert_close("dv", dv, rv)


@pytest.mark.parametrize("wname", ["mid", "hist16k"])
def test_full_size_sampled(wname):
    """The bench workloads at full size, checked on sampled rows (forward, dq)
    and sampled keys (dk, dv) that the oracle computes one by one."""
    b = make_batch(WORKLOADS[wname])
    g = to_gpu(b)
    out = gpu_fwd(b, g)
    dq, dk, dv = gpu_bwd(b, g)
    p = oracle_problem(b)
    rows = sample_tokens(b, 160, seed=1)
    keys = sample_tokens(b, 160, seed=2)
    assert_close("out", out[rows], p.fwd(b.q, b.k, b.v, rows=rows))
    assert_close("dq", dq[rows], p.bwd_dq(b.q, b.k, b.v, b.dout, rows=rows))
    rk, rv = p.bwd_dkv(b.q, b.k, b.v, b.dout, keys=keys)
    assert_close("dk", dk[keys], rk)
    assert_close("dv", dv[keys], rv)
    for t in (out, dq, dk, dv):
        assert torch.isfinite(t.float()).all()


def test_backward_prepared_on_a_side_stream():
    """hstu_sla_bwd_prepare (work list and dQ-accumulator clear) on another
    stream, ordered by an event, then the backward with prepared=True on the
    same workspace: dk and dv equal the plain call's bit for bit, dq matches
    the oracle (its fp32 additions have no fixed order), twice in a row so
    the second prepare clears what the first backward left."""
    b = _edge_batch(lengths=[300, 17, 201, 129], nt=12, K1=96, K2=24, ctx=8)
    g = to_gpu(b)
    kw = kwargs_of(b)
    T, H, d = b.q.shape
    ws = torch.empty(sla.hstu_sla_workspace_bytes(1, T, len(b.lengths), H, d),
                     dtype=torch.uint8, device="cuda")
    dq0, dk0, dv0 = sla.hstu_sla_bwd(g["dout"], g["q"], g["k"], g["v"], g["offs"], g["nts"], **kw)
    side = torch.cuda.Stream()
    main = torch.cuda.current_stream()
    p = oracle_problem(b)
    rq, rk, rv = p.bwd(b.q, b.k, b.v, b.dout)
    for _ in range(2):
        ev0, ev1 = torch.cuda.Event(), torch.cuda.Event()
        ev0.record(main)
        side.wait_event(ev0)
        sla.hstu_sla_bwd_prepare(g["q"], g["offs"], g["nts"], workspace=ws, stream=side, **kw)
        ev1.record(side)
        main.wait_event(ev1)
        dq, dk, dv = sla.hstu_sla_bwd(g["dout"], g["q"], g["k"], g["v"], g["offs"], g["nts"],
                                      workspace=ws, prepared=True, **kw)
        torch.cuda.synchronize()
        assert sla.hstu_sla_get_error(ws) == 0
        assert torch.equal(dk, dk0) and torch.equal(dv, dv0)
        assert_close("dq", dq, rq)
        assert_close("dk", dk, rk)
        assert_close("dv", dv, rv)


def test_mid_full_tensor():
    """The mid-length training batch (32 sequences of 1K-4K tokens, 4 x 128
    heads, K1 256, K2 64) compared element by element over the whole jagged
    tensor: out, dq, dk, dv against the oracle's full forward and backward."""
    b = make_batch(WORKLOADS["mid"])
    g = to_gpu(b)
    out = gpu_fwd(b, g)
    dq, dk, dv = gpu_bwd(b, g)
    p = oracle_problem(b)
    assert_close("out", out, p.fwd(b.q, b.k, b.v))
    rq, rk, rv = p.bwd(b.q, b.k, b.v, b.dout)
    assert_close("dq", dq, rq)
    assert_close("dk", dk, rk)
    assert_close("dv", dv, rv)


def test_candidate_scoring_computes_only_candidate_tiles():
    """M-FALCON scoring (candidates_only): rows of the query tiles that hold
    candidates equal the full forward bit for bit (and the oracle); rows of
    the other tiles keep what the output buffer held."""
    lengths, nts = [700, 1300, 260, 90], [64, 100, 260, 0]
    b = _edge_batch(lengths=lengths, nt=np.array(nts), K1=128, K2=32, ctx=8)
    g = to_gpu(b)
    full = gpu_fwd(b, g)
    out = torch.full_like(g["q"], 7.0)
    sla.hstu_sla_fwd(g["q"], g["k"], g["v"], g["offs"], g["nts"], out=out, candidates_only=True,
                     **kwargs_of(b))
    torch.cuda.synchronize()
    p = oracle_problem(b)
    for i, (L, nt) in enumerate(zip(lengths, nts)):
        s0 = int(b.seq_offsets[i])
        first = ((L - nt) // 128) * 128 if nt > 0 else L
        assert bool((out[s0:s0 + first] == 7.0).all())
        assert torch.equal(out[s0 + first:s0 + L], full[s0 + first:s0 + L])
        if nt:
            rows = np.arange(s0 + L - nt, s0 + L)
            assert_close("candidates", out[rows], p.fwd(b.q, b.k, b.v, rows=rows))


def test_inference_workload_sampled():
    b = make_batch(WORKLOADS["infer"], with_dout=False)
    g = to_gpu(b)
    out = gpu_fwd(b, g)
    p = oracle_problem(b)
    rows = sample_tokens(b, 96, seed=3)
    assert_close("out", out[rows], p.fwd(b.q, b.k, b.v, rows=rows))
    # candidate scoring on the same batch: every candidate row as in the full pass
    cand = sla.hstu_sla_fwd(g["q"], g["k"], g["v"], g["offs"], g["nts"], candidates_only=True,
                            out=torch.zeros_like(out), **kwargs_of(b))
    torch.cuda.synchronize()
    for i in range(len(b.lengths)):
        s0, s1 = int(b.seq_offsets[i]), int(b.seq_offsets[i + 1])
        lo = s1 - int(b.num_targets[i])
        assert torch.equal(cand[lo:s1], out[lo:s1])
    assert torch.isfinite(out.float()).all()


@pytest.mark.parametrize("wname", ["mid", "hist16k"])
def test_full_size_pair_counts(wname):
    _count_check(make_batch(WORKLOADS[wname], with_dout=False))


@pytest.mark.parametrize("bad", ["non_monotone", "targets_exceed_length", "last_offset",
                                 "too_long"])
def test_device_detected_bad_input(bad):
    """Corrupted offsets / targets are caught on the device: the kernels skip all
    work and the status reads ERR_BAD_INPUT; the context stays usable."""
    b = _edge_batch(lengths=[100, 100, 100], nt=4)
    g = to_gpu(b)
    offs, nts = g["offs"].clone(), g["nts"].clone()
    msl = 100
    if bad == "non_monotone":
        offs[1] = 250
    elif bad == "targets_exceed_length":
        nts[2] = 101
    elif bad == "last_offset":
        offs[3] = 299
    else:
        msl = 99
    ws = torch.zeros(sla.hstu_sla_workspace_bytes(1, b.T, 3, b.q.shape[1], b.q.shape[2]),
                     dtype=torch.uint8, device="cuda")
    kw = dict(contextual_len=3, K1=40, K2=10, alpha=0.1, N=300.0, max_seq_len=msl)
    sla.hstu_sla_fwd(g["q"], g["k"], g["v"], offs, nts, workspace=ws, **kw)
    assert sla.hstu_sla_get_error(ws) == -4
    sla.hstu_sla_bwd(g["dout"], g["q"], g["k"], g["v"], offs, nts, workspace=ws, **kw)
    assert sla.hstu_sla_get_error(ws) == -4
    # the same workspace with good inputs clears the status
    sla.hstu_sla_fwd(g["q"], g["k"], g["v"], g["offs"], g["nts"], workspace=ws,
                     **dict(kw, max_seq_len=100))
    assert sla.hstu_sla_get_error(ws) == 0


def test_autograd_wrapper():
    b = _edge_batch(lengths=[120, 64], nt=6)
    g = to_gpu(b)
    q, k, v = (g[n].clone().requires_grad_(True) for n in ("q", "k", "v"))
    out = sla.sla_attention(q, k, v, g["offs"], g["nts"], contextual_len=3, K1=40, K2=10,
                            alpha=128 ** -0.5, N=300.0, max_seq_len=120)
    out.backward(g["dout"])
    p = oracle_problem(b)
    rq, rk, rv = p.bwd(b.q, b.k, b.v, b.dout)
    assert_close("dq", q.grad, rq)
    assert_close("dk", k.grad, rk)
    assert_close("dv", v.grad, rv)

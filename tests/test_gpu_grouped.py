"""GPU parity of the grouped calls (several SLA problems, e.g. the channels of
a Mixture of Transducers, in one kernel launch): each group's results equal
its own separate call (forward, dk, dv bitwise; dq to fp32 summation order)
and the oracle's (TOL of max|ref|), with different sequences, heads, SLA
windows, N and alpha per group; an empty group; per-group candidate scoring;
and a device-side input error in one group reported for the launch."""
import numpy as np
import pytest
import torch

import sparse_hstu_attention_b200 as sla
from sparse_hstu_attention_b200 import _abi
from workloads import WORKLOADS, make_batch, with_params

from parity import assert_close, kwargs_of, oracle_problem, to_gpu

pytestmark = pytest.mark.gpu


def _batch(lengths, nt, H, K1, K2, ctx, N, alpha, seed):
    w = with_params(WORKLOADS["tiny"], H=H, d=128, K1=K1, K2=K2, contextual_len=ctx,
                    num_targets=nt, alpha=alpha, N=N)
    lengths = np.array(lengths, dtype=np.int64)
    return make_batch(w, lengths=lengths, num_targets=np.minimum(nt, lengths), seed=seed)


GROUPS = [
    dict(lengths=[300, 1200, 77, 640, 129], nt=16, H=4, K1=256, K2=64, ctx=16, N=1200.0,
         alpha=128 ** -0.5, seed=11),
    dict(lengths=[50, 400, 260, 31, 129, 64, 200, 333, 90], nt=8, H=2, K1=100000, K2=0, ctx=0,
         N=400.0, alpha=0.05, seed=12),
    dict(lengths=[700, 2100, 1500], nt=64, H=4, K1=128, K2=128, ctx=32, N=2100.0,
         alpha=128 ** -0.5, seed=13),
]


def _group_dict(b, g, **extra):
    d = dict(q=g["q"], k=g["k"], v=g["v"], seq_offsets=g["offs"], num_targets=g["nts"],
             **kwargs_of(b))
    d.update(extra)
    return d


def test_grouped_forward_and_backward():
    batches = [_batch(**c) for c in GROUPS]
    gpus = [to_gpu(b) for b in batches]
    outs = sla.hstu_sla_fwd_grouped([_group_dict(b, g) for b, g in zip(batches, gpus)])
    grads = sla.hstu_sla_bwd_grouped([_group_dict(b, g, dout=g["dout"])
                                      for b, g in zip(batches, gpus)])
    torch.cuda.synchronize()
    for i, (b, g) in enumerate(zip(batches, gpus)):
        one = sla.hstu_sla_fwd(g["q"], g["k"], g["v"], g["offs"], g["nts"], **kwargs_of(b))
        dq1, dk1, dv1 = sla.hstu_sla_bwd(g["dout"], g["q"], g["k"], g["v"], g["offs"], g["nts"],
                                         **kwargs_of(b))
        torch.cuda.synchronize()
        assert torch.equal(outs[i], one), f"group {i}: out differs from its own call"
        dq, dk, dv = grads[i]
        assert torch.equal(dk, dk1) and torch.equal(dv, dv1), f"group {i}: dk / dv differ"
        assert_close(f"group {i} dq vs own call", dq, dq1.float().cpu().numpy().astype(np.float64),
                     tol=1e-2)
        p = oracle_problem(b)
        assert_close(f"group {i} out", outs[i], p.fwd(b.q, b.k, b.v))
        rq, rk, rv = p.bwd(b.q, b.k, b.v, b.dout)
        assert_close(f"group {i} dq", dq, rq)
        assert_close(f"group {i} dk", dk, rk)
        assert_close(f"group {i} dv", dv, rv)


def _empty_group(H):
    """A group of two empty sequences (T = 0; its tensor pointers are null,
    which the library accepts when there are no tokens)."""
    w = with_params(WORKLOADS["tiny"], H=H, d=128, K1=64, K2=8, contextual_len=0, num_targets=4,
                    alpha=0.1, N=10.0)
    b = make_batch(w, lengths=np.array([0, 0]), num_targets=np.array([0, 0]), seed=14)
    t = torch.zeros((0, H, 128), dtype=torch.bfloat16, device="cuda")
    g = dict(q=t, k=t, v=t, dout=t,
             offs=torch.zeros(3, dtype=torch.int32, device="cuda"),
             nts=torch.zeros(2, dtype=torch.int32, device="cuda"))
    return b, g


def test_grouped_with_an_empty_group_and_candidate_scoring():
    full = _batch(**GROUPS[0])
    empty, g_empty = _empty_group(4)
    g_full = to_gpu(full)
    marker = torch.full(g_full["q"].shape, 7.0, dtype=torch.bfloat16, device="cuda")
    outs = sla.hstu_sla_fwd_grouped([
        _group_dict(empty, g_empty),
        _group_dict(full, g_full, candidates_only=True, out=marker)])
    torch.cuda.synchronize()
    assert outs[0].numel() == 0
    ref = oracle_problem(full).fwd(full.q, full.k, full.v)
    offs, nts = full.seq_offsets, full.num_targets
    cand = np.concatenate([np.arange(offs[b + 1] - nts[b], offs[b + 1])
                           for b in range(len(nts))]).astype(np.int64)
    got = outs[1].float().cpu().numpy().astype(np.float64)
    assert_close("candidate rows", got[cand], ref[cand])
    # rows outside the candidates' query tiles keep what the buffer held
    first_tile = [(offs[b] + ((offs[b + 1] - offs[b] - nts[b]) // 128) * 128)
                  for b in range(len(nts))]
    untouched = np.concatenate([np.arange(offs[b], first_tile[b]) for b in range(len(nts))])
    assert np.all(got[untouched.astype(np.int64)] == 7.0)
    grads = sla.hstu_sla_bwd_grouped([_group_dict(empty, g_empty, dout=g_empty["dout"]),
                                      _group_dict(full, g_full, dout=g_full["dout"])])
    torch.cuda.synchronize()
    rq, rk, rv = oracle_problem(full).bwd(full.q, full.k, full.v, full.dout)
    assert_close("dq", grads[1][0], rq)
    assert_close("dk", grads[1][1], rk)


def test_grouped_device_input_error_is_reported():
    """Group 1's offsets end past its token count: its work-list kernel flags
    the batch, the grouped kernel does nothing and the launch's status word
    (the workspace header) carries the error."""
    a, b = _batch(**GROUPS[0]), _batch(**GROUPS[1])
    ga, gb = to_gpu(a), to_gpu(b)
    bad = gb["offs"].clone()
    bad[-1] += 1
    groups = [_group_dict(a, ga), _group_dict(b, gb, seq_offsets=bad)]
    params = [(a.T, len(a.lengths), a.workload.H, 128), (b.T, len(b.lengths), b.workload.H, 128)]
    ws = torch.empty(sla.hstu_sla_grouped_workspace_bytes(_abi.WS_FWD, params), dtype=torch.uint8,
                     device="cuda")
    sla.hstu_sla_fwd_grouped(groups, workspace=ws)
    assert sla.hstu_sla_get_error(ws) == _abi.ERR_BAD_INPUT
    # the same workspace serves a good call afterwards
    groups[1]["seq_offsets"] = gb["offs"]
    sla.hstu_sla_fwd_grouped(groups, workspace=ws)
    assert sla.hstu_sla_get_error(ws) == _abi.OK

"""Guard bands around every output and workspace (the stand-in for an
out-of-bounds write checker): outputs are views into larger buffers whose
rows before and after the T rows hold a sentinel, and each workspace is
followed by sentinel bytes.  After forward, backward and grouped calls (and
on batches whose last tile runs past T), the sentinels must be untouched and
the outputs must still match the oracle."""
import numpy as np
import pytest
import torch

import sparse_hstu_attention_b200 as sla
from workloads import WORKLOADS, make_batch, with_params

from parity import assert_close, kwargs_of, oracle_problem, to_gpu

pytestmark = pytest.mark.gpu

GUARD_ROWS = 9          # sentinel rows before and after each output
GUARD_BYTES = 4096      # sentinel bytes after each workspace
SENTINEL = -1234.0      # exactly representable in bf16
WS_BYTE = 0xA5


def _guarded(T, H, d):
    """An output view of T rows inside a sentinel-filled buffer."""
    buf = torch.full((T + 2 * GUARD_ROWS, H, d), SENTINEL, dtype=torch.bfloat16, device="cuda")
    return buf, buf[GUARD_ROWS:GUARD_ROWS + T]


def _check_rows(name, buf, T):
    head, tail = buf[:GUARD_ROWS], buf[GUARD_ROWS + T:]
    assert bool((head == SENTINEL).all()), f"{name}: write before row 0"
    assert bool((tail == SENTINEL).all()), f"{name}: write past row T - 1"


def _guarded_ws(need):
    ws = torch.full((need + GUARD_BYTES,), WS_BYTE, dtype=torch.uint8, device="cuda")
    return ws


def _check_ws(name, ws, need):
    assert bool((ws[need:] == WS_BYTE).all()), f"{name}: write past the workspace"


def _batch(lengths, nt, d=128, K1=96, K2=24, ctx=8, H=2, seed=11):
    w = with_params(WORKLOADS["tiny"], H=H, d=d, K1=K1, K2=K2, contextual_len=ctx,
                    num_targets=nt, alpha=d ** -0.5, N=500.0)
    lengths = np.array(lengths, dtype=np.int64)
    return make_batch(w, lengths=lengths, num_targets=np.minimum(nt, lengths), seed=seed)


CASES = {
    # last tile of the last sequence ends mid-tile, short middle sequence
    "ragged_d128": dict(lengths=[300, 17, 201], nt=12),
    # a sequence that is only candidates, an empty one, a 1-token one
    "degenerate_d128": dict(lengths=[129, 0, 1, 64, 65], nt=[129, 0, 1, 5, 64]),
    # head_dim 64 and 32 take the two-pass backward
    "ragged_d64": dict(lengths=[190, 77], nt=9, d=64),
    "ragged_d32": dict(lengths=[250, 33, 5], nt=4, d=32),
    # long sequences whose prefix key tiles (one, two, three of them via K2)
    # are seen by thousands of rows, last tile ragged
    "long_prefix1_d128": dict(lengths=[8192 + 37, 5], nt=12),
    "long_prefix2_d128": dict(lengths=[40, 10001], nt=7, K2=200),
    "long_prefix3_d128": dict(lengths=[8200], nt=3, K2=300),
}


@pytest.mark.parametrize("case", sorted(CASES))
def test_outputs_and_workspaces_stay_in_bounds(case):
    b = _batch(**CASES[case])
    g = to_gpu(b)
    T, H, d = b.q.shape
    B = len(b.lengths)
    kw = kwargs_of(b)
    p = oracle_problem(b)
    need_f = sla.hstu_sla_workspace_bytes(0, T, B, H, d)
    need_b = sla.hstu_sla_workspace_bytes(1, T, B, H, d)
    ws_f, ws_b = _guarded_ws(need_f), _guarded_ws(need_b)
    ob, out = _guarded(T, H, d)
    sla.hstu_sla_fwd(g["q"], g["k"], g["v"], g["offs"], g["nts"], out=out, workspace=ws_f, **kw)
    bufs = [_guarded(T, H, d) for _ in range(3)]
    sla.hstu_sla_bwd(g["dout"], g["q"], g["k"], g["v"], g["offs"], g["nts"], dq=bufs[0][1],
                     dk=bufs[1][1], dv=bufs[2][1], workspace=ws_b, **kw)
    torch.cuda.synchronize()
    assert sla.hstu_sla_get_error(ws_f) == 0 and sla.hstu_sla_get_error(ws_b) == 0
    _check_rows("out", ob, T)
    for name, (buf, _) in zip(("dq", "dk", "dv"), bufs):
        _check_rows(name, buf, T)
    _check_ws("forward workspace", ws_f, need_f)
    _check_ws("backward workspace", ws_b, need_b)
    if T:
        assert_close("out", out, p.fwd(b.q, b.k, b.v))
        rq, rk, rv = p.bwd(b.q, b.k, b.v, b.dout)
        for name, got, ref in zip(("dq", "dk", "dv"), (bufs[0][1], bufs[1][1], bufs[2][1]),
                                  (rq, rk, rv)):
            assert_close(name, got, ref)


def test_grouped_calls_stay_in_bounds():
    """Two problems in one grouped launch, each with guarded outputs; the
    grouped workspace is followed by sentinel bytes."""
    batches = [_batch(lengths=[300, 17, 201], nt=12, seed=3),
               _batch(lengths=[140, 260], nt=7, K1=300, K2=0, ctx=0, seed=4)]
    groups, guards = [], []
    for b in batches:
        g = to_gpu(b)
        T, H, d = b.q.shape
        ob, out = _guarded(T, H, d)
        dbufs = [_guarded(T, H, d) for _ in range(3)]
        kw = kwargs_of(b)
        groups.append(dict(q=g["q"], k=g["k"], v=g["v"], dout=g["dout"], seq_offsets=g["offs"],
                           num_targets=g["nts"], out=out, dq=dbufs[0][1], dk=dbufs[1][1],
                           dv=dbufs[2][1], **kw))
        guards.append((T, ob, dbufs))
    sizes = [(b.T, len(b.lengths), b.q.shape[1], b.q.shape[2]) for b in batches]
    need_f = sla.hstu_sla_grouped_workspace_bytes(0, sizes)
    need_b = sla.hstu_sla_grouped_workspace_bytes(1, sizes)
    ws_f, ws_b = _guarded_ws(need_f), _guarded_ws(need_b)
    sla.hstu_sla_fwd_grouped(groups, workspace=ws_f)
    sla.hstu_sla_bwd_grouped(groups, workspace=ws_b)
    torch.cuda.synchronize()
    assert sla.hstu_sla_get_error(ws_f) == 0 and sla.hstu_sla_get_error(ws_b) == 0
    _check_ws("grouped forward workspace", ws_f, need_f)
    _check_ws("grouped backward workspace", ws_b, need_b)
    for b, grp, (T, ob, dbufs) in zip(batches, groups, guards):
        _check_rows("out", ob, T)
        for name, (buf, _) in zip(("dq", "dk", "dv"), dbufs):
            _check_rows(name, buf, T)
        p = oracle_problem(b)
        assert_close("out", grp["out"], p.fwd(b.q, b.k, b.v))
        rq, rk, rv = p.bwd(b.q, b.k, b.v, b.dout)
        assert_close("dq", grp["dq"], rq)
        assert_close("dk", grp["dk"], rk)
        assert_close("dv", grp["dv"], rv)

"""The bounded-wait failure path, on the GPU without a fault: a kernel
instantiation whose pointwise warps each withhold one hand-over arrive (the
test hook hstu_sla_test_wait_timeout) must give up after the short limit it
is given, report HSTU_SLA_ERR_TIMEOUT, drain and release TMEM, and leave the
context usable: the next normal calls on the same inputs match the oracle."""
import ctypes

import numpy as np
import pytest
import torch

import sparse_hstu_attention_b200 as sla
from sparse_hstu_attention_b200 import _abi
from workloads import WORKLOADS, make_batch, with_params

from parity import assert_close, kwargs_of, oracle_problem, to_gpu

pytestmark = pytest.mark.gpu

LIMIT_NS = 5_000_000  # 5 ms: far below the production kernels' 2 s


def _batch():
    w = with_params(WORKLOADS["tiny"], H=2, d=128, K1=200, K2=32, contextual_len=8,
                    num_targets=16, alpha=128 ** -0.5, N=800.0)
    lengths = np.array([700, 333, 512, 90], dtype=np.int64)
    return make_batch(w, lengths=lengths, seed=21)


def _params(g, kw, outs):
    q = g["q"]
    T, H, d = q.shape
    p = _abi.BwdParams()
    f = p.fwd
    f.B, f.H, f.d, f.total_tokens = g["offs"].numel() - 1, H, d, T
    f.max_seq_len = kw["max_seq_len"]
    f.seq_offsets, f.num_targets = g["offs"].data_ptr(), g["nts"].data_ptr()
    f.contextual_len, f.K1, f.K2 = kw["contextual_len"], kw["K1"], kw["K2"]
    f.alpha, f.N = kw["alpha"], kw["N"]
    f.q, f.k, f.v = q.data_ptr(), g["k"].data_ptr(), g["v"].data_ptr()
    f.q_row_stride = f.k_row_stride = f.v_row_stride = q.stride(0)
    f.out, f.out_row_stride = outs[0].data_ptr(), outs[0].stride(0)
    p.dout, p.dout_row_stride = g["dout"].data_ptr(), g["dout"].stride(0)
    p.dq, p.dk, p.dv = (t.data_ptr() for t in outs[1:])
    p.dq_row_stride = p.dk_row_stride = p.dv_row_stride = q.stride(0)
    return p


@pytest.mark.parametrize("which", [0, 1], ids=["forward", "backward"])
def test_stalled_kernel_times_out_and_context_recovers(which):
    lib = _abi.load()
    b = _batch()
    g = to_gpu(b)
    kw = kwargs_of(b)
    T, H, d = b.q.shape
    outs = [torch.zeros_like(g["q"]) for _ in range(4)]
    ws = torch.zeros(sla.hstu_sla_workspace_bytes(which, T, len(b.lengths), H, d),
                     dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    rc = lib.hstu_sla_test_wait_timeout(ctypes.byref(_params(g, kw, outs)), which, LIMIT_NS,
                                        ws.data_ptr(), ws.numel(), stream.cuda_stream)
    e1.record(stream)
    assert rc == _abi.OK, sla.hstu_sla_strerror(rc)
    assert sla.hstu_sla_get_error(ws) == _abi.ERR_TIMEOUT
    ms = e0.elapsed_time(e1)
    # the short limit was the one applied (not the 2 s default), and it was waited out
    assert LIMIT_NS * 1e-6 <= ms < 500.0, ms
    # TMEM released, context usable: normal calls on the same workspace and inputs
    out = sla.hstu_sla_fwd(g["q"], g["k"], g["v"], g["offs"], g["nts"], workspace=ws, **kw) \
        if which == 0 else sla.hstu_sla_fwd(g["q"], g["k"], g["v"], g["offs"], g["nts"], **kw)
    dq, dk, dv = sla.hstu_sla_bwd(g["dout"], g["q"], g["k"], g["v"], g["offs"], g["nts"],
                                  workspace=ws if which == 1 else None, **kw)
    torch.cuda.synchronize()
    assert sla.hstu_sla_get_error(ws) == _abi.OK
    p = oracle_problem(b)
    assert_close("out", out, p.fwd(b.q, b.k, b.v))
    rq, rk, rv = p.bwd(b.q, b.k, b.v, b.dout)
    assert_close("dq", dq, rq)
    assert_close("dk", dk, rk)
    assert_close("dv", dv, rv)


def test_wait_timeout_hook_rejects_bad_arguments():
    lib = _abi.load()
    b = _batch()
    g = to_gpu(b)
    kw = kwargs_of(b)
    outs = [torch.zeros_like(g["q"]) for _ in range(4)]
    p = _params(g, kw, outs)
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    s = torch.cuda.current_stream().cuda_stream
    assert lib.hstu_sla_test_wait_timeout(ctypes.byref(p), 2, LIMIT_NS, ws.data_ptr(),
                                          ws.numel(), s) == _abi.ERR_INVALID_ARG
    assert lib.hstu_sla_test_wait_timeout(ctypes.byref(p), 0, 0, ws.data_ptr(), ws.numel(),
                                          s) == _abi.ERR_INVALID_ARG

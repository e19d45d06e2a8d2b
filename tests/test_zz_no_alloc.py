"""hstu_sla_fwd_noalloc: the forward entry point that allocates nothing, for
callers whose runtime forbids device allocation in the launch path.  It must
give the same result as hstu_sla_fwd (the entry point with a caller-provided
workspace) on consecutive calls, since every call reuses the library's one
scratch array.  Kept in a file of its own, collected last."""
import ctypes

import pytest
import torch

import sparse_hstu_attention_b200 as sla
from sparse_hstu_attention_b200 import _abi
from workloads import WORKLOADS, make_batch

from parity import TOL, kwargs_of, to_gpu

pytestmark = pytest.mark.gpu


def _params(g, kw, out):
    p = _abi.FwdParams()
    q = g["q"]
    T, H, d = q.shape
    p.B, p.H, p.d, p.total_tokens = g["offs"].numel() - 1, H, d, T
    p.max_seq_len = kw["max_seq_len"]
    p.seq_offsets, p.num_targets = g["offs"].data_ptr(), g["nts"].data_ptr()
    p.contextual_len, p.K1, p.K2 = kw["contextual_len"], kw["K1"], kw["K2"]
    p.alpha, p.N = kw["alpha"], kw["N"]
    p.q, p.k, p.v = q.data_ptr(), g["k"].data_ptr(), g["v"].data_ptr()
    p.q_row_stride = p.k_row_stride = p.v_row_stride = q.stride(0)
    p.out, p.out_row_stride = out.data_ptr(), out.stride(0)
    return p


def test_noalloc_matches_workspace_entry_point_on_consecutive_calls():
    """Both entry points run the same kernels on the same work lists, and the
    forward is deterministic: the results must be identical bit for bit, so
    any corruption left in the shared scratch by the previous call shows."""
    lib = _abi.load()
    stream = torch.cuda.current_stream().cuda_stream
    batches = [make_batch(WORKLOADS["mid"], with_dout=False),
               make_batch(WORKLOADS["tiny"], with_dout=False)]
    for b in batches:   # two calls in a row per batch, different batches back to back
        g = to_gpu(b)
        kw = kwargs_of(b)
        ref = sla.hstu_sla_fwd(g["q"], g["k"], g["v"], g["offs"], g["nts"], **kw)
        for _ in range(2):
            out = torch.full_like(ref, float("nan"))
            rc = lib.hstu_sla_fwd_noalloc(ctypes.byref(_params(g, kw, out)), stream)
            assert rc == _abi.OK, sla.hstu_sla_strerror(rc)
            assert lib.hstu_sla_noalloc_get_error(stream) == _abi.OK
            torch.cuda.synchronize()
            assert torch.equal(out, ref)
            scale = ref.float().abs().max().item()
            err = (out.float() - ref.float()).abs().max().item()
            assert err <= TOL * scale, (err, scale)


def test_noalloc_python_binding_and_device_status():
    """The binding's wrapper checks the device status; corrupted offsets are
    reported as BAD_INPUT (out left unwritten), and the next good call
    clears the status."""
    b = make_batch(WORKLOADS["tiny"], with_dout=False)
    g = to_gpu(b)
    kw = kwargs_of(b)
    ref = sla.hstu_sla_fwd(g["q"], g["k"], g["v"], g["offs"], g["nts"], **kw)
    out = sla.hstu_sla_fwd_noalloc(g["q"], g["k"], g["v"], g["offs"], g["nts"], **kw)
    assert torch.equal(out, ref)
    bad = g["offs"].clone()
    bad[1] = bad[2] + 1  # offsets no longer monotone
    out = torch.full_like(ref, float("nan"))
    with pytest.raises(sla.SLAError):
        sla.hstu_sla_fwd_noalloc(g["q"], g["k"], g["v"], bad, g["nts"], out=out, **kw)
    assert sla.hstu_sla_noalloc_get_error() == _abi.ERR_BAD_INPUT
    assert torch.isnan(out.float()).all()
    out = sla.hstu_sla_fwd_noalloc(g["q"], g["k"], g["v"], g["offs"], g["nts"], **kw)
    assert sla.hstu_sla_noalloc_get_error() == _abi.OK
    assert torch.equal(out, ref)


def test_noalloc_rejects_batches_beyond_its_scratch():
    lib = _abi.load()
    b = make_batch(WORKLOADS["tiny"], with_dout=False)
    g = to_gpu(b)
    kw = kwargs_of(b)
    out = torch.empty_like(g["q"])
    p = _params(g, kw, out)
    p.total_tokens = 64 * 140_000   # needs more than the 2 MiB scratch: rejected on the host
    assert lib.hstu_sla_fwd_noalloc(ctypes.byref(p), torch.cuda.current_stream().cuda_stream) \
        == _abi.ERR_WORKSPACE

"""The C-ABI library: it loads without a GPU, exports every symbol the header
declares, and rejects bad arguments on the host before touching CUDA."""
import ctypes

import pytest

import sparse_hstu_attention_b200 as sla
from sparse_hstu_attention_b200 import _abi


@pytest.fixture(scope="module")
def lib():
    from sparse_hstu_attention_b200 import build
    build.build()
    return _abi.load()


def test_exports_every_declared_symbol(lib):
    names = _abi.declared_functions()
    assert {"hstu_sla_fwd", "hstu_sla_bwd", "hstu_sla_workspace_bytes",
            "hstu_sla_count_pairs", "hstu_sla_get_error", "hstu_sla_strerror"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_version_and_messages(lib):
    assert lib.hstu_sla_version() >= 100
    for code in (0, -1, -2, -3, -4, -5, -6):
        assert sla.hstu_sla_strerror(code)
    assert "unknown" in sla.hstu_sla_strerror(-99)


def test_workspace_sizes(lib):
    f = lib.hstu_sla_workspace_bytes
    assert f(_abi.WS_FWD, 0, 1, 1, 32) >= 256
    fwd = f(_abi.WS_FWD, 100_000, 8, 4, 128)
    bwd = f(_abi.WS_BWD, 100_000, 8, 4, 128)
    assert fwd % 256 == 0 and bwd % 256 == 0
    assert bwd >= fwd >= 16 * (100_000 // 64)   # two work lists of (seq, tile) pairs
    assert f(7, 10, 1, 1, 32) == 0
    assert f(_abi.WS_FWD, -1, 1, 1, 32) == 0


FAKE = 0x10000  # never dereferenced: every case below fails a host check first


def _params(**kw):
    p = _abi.FwdParams()
    p.B, p.H, p.d, p.total_tokens, p.max_seq_len = 2, 4, 128, 100, 100
    p.seq_offsets = FAKE
    p.contextual_len, p.K1, p.K2, p.alpha, p.N = 0, 8, 4, 0.1, 10.0
    p.q = p.k = p.v = p.out = FAKE
    p.q_row_stride = p.k_row_stride = p.v_row_stride = p.out_row_stride = 512
    for k, v in kw.items():
        setattr(p, k, v)
    return p


@pytest.mark.parametrize("field,value,code", [
    ("d", 48, _abi.ERR_UNSUPPORTED),
    ("d", 256, _abi.ERR_UNSUPPORTED),
    ("B", 0, _abi.ERR_INVALID_ARG),
    ("H", 0, _abi.ERR_INVALID_ARG),
    ("K1", -1, _abi.ERR_INVALID_ARG),
    ("K2", -3, _abi.ERR_INVALID_ARG),
    ("contextual_len", -1, _abi.ERR_INVALID_ARG),
    ("N", 0.0, _abi.ERR_INVALID_ARG),
    ("N", float("nan"), _abi.ERR_INVALID_ARG),
    ("alpha", float("inf"), _abi.ERR_INVALID_ARG),
    ("q", None, _abi.ERR_INVALID_ARG),
    ("v", FAKE + 8, _abi.ERR_INVALID_ARG),          # not 16-byte aligned
    ("k_row_stride", 500, _abi.ERR_INVALID_ARG),    # < H*d
    ("q_row_stride", 516, _abi.ERR_INVALID_ARG),    # not a multiple of 8
    ("seq_offsets", None, _abi.ERR_INVALID_ARG),
    ("out", None, _abi.ERR_INVALID_ARG),
    ("total_tokens", 1 << 40, _abi.ERR_UNSUPPORTED),
])
def test_fwd_host_validation(lib, field, value, code):
    p = _params(**{field: value})
    assert lib.hstu_sla_fwd(ctypes.byref(p), FAKE * 256, 1 << 30, None) == code


def test_workspace_validation(lib):
    p = _params()
    need = lib.hstu_sla_workspace_bytes(_abi.WS_FWD, 100, 2, 4, 128)
    assert lib.hstu_sla_fwd(ctypes.byref(p), None, need, None) == _abi.ERR_WORKSPACE
    assert lib.hstu_sla_fwd(ctypes.byref(p), FAKE * 256 + 16, need, None) == _abi.ERR_WORKSPACE
    assert lib.hstu_sla_fwd(ctypes.byref(p), FAKE * 256, need - 1, None) == _abi.ERR_WORKSPACE


def test_bwd_host_validation(lib):
    b = _abi.BwdParams()
    b.fwd = _params()
    b.dout = b.dq = b.dk = b.dv = FAKE
    b.dout_row_stride = b.dq_row_stride = b.dk_row_stride = b.dv_row_stride = 512
    b.dk = None
    assert lib.hstu_sla_bwd(ctypes.byref(b), FAKE * 256, 1 << 40, None) == _abi.ERR_INVALID_ARG
    b.dk = FAKE
    b.dv_row_stride = 4
    assert lib.hstu_sla_bwd(ctypes.byref(b), FAKE * 256, 1 << 40, None) == _abi.ERR_INVALID_ARG
    b.dv_row_stride = 512
    need = lib.hstu_sla_workspace_bytes(_abi.WS_BWD, 100, 2, 4, 128)
    assert lib.hstu_sla_bwd(ctypes.byref(b), FAKE * 256, need - 256, None) == _abi.ERR_WORKSPACE
    assert lib.hstu_sla_bwd(None, FAKE * 256, need, None) == _abi.ERR_INVALID_ARG


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(_abi, "_lib", None)
    monkeypatch.setattr(_abi, "LIB_PATH", str(tmp_path / "absent.so"))
    with pytest.raises(_abi.LibraryMissing):
        _abi.load()


def _c_layout(struct_name, fields, tmp_path):
    """sizeof and every field's offsetof as gcc lays the header's struct out."""
    import subprocess
    src = tmp_path / "layout.c"
    lines = ['#include <stdio.h>', '#include <stddef.h>', '#include "hstu_stu.h"',
             'int main(void) {', f'  printf("%zu\\n", sizeof({struct_name}));']
    lines += [f'  printf("%zu\\n", offsetof({struct_name}, {f}));' for f in fields]
    lines += ['  return 0;', '}']
    src.write_text("\n".join(lines))
    exe = tmp_path / "layout"
    subprocess.run(["gcc", "-std=c99", "-I", _abi.INCLUDE_DIR, str(src), "-o", str(exe)],
                   check=True)
    return [int(v) for v in subprocess.run([str(exe)], check=True, capture_output=True,
                                           text=True).stdout.split()]


@pytest.mark.parametrize("py,c", [
    (_abi.FwdParams, "hstu_sla_fwd_params"), (_abi.BwdParams, "hstu_sla_bwd_params"),
    (_abi.StuLayerParams, "hstu_stu_layer_params"),
    (_abi.StuLayerBwdParams, "hstu_stu_layer_bwd_params"), (_abi.GemmParams, "hstu_gemm_params"),
])
def test_binding_structs_match_the_headers(py, c, tmp_path):
    """The binding's ctypes structs have the C compiler's size and offsets."""
    names = [f[0] for f in py._fields_]
    got = _c_layout(c, names, tmp_path)
    assert got[0] == ctypes.sizeof(py)
    assert got[1:] == [getattr(py, n).offset for n in names]


def test_grouped_calls_reject_bad_groups_on_the_host(lib):
    """Host-side checks of the grouped entry points (no CUDA call is reached)."""
    import numpy as np
    G = 2
    arr = (_abi.FwdParams * G)(_params(), _params())
    for p in arr:
        p.out, p.out_row_stride = FAKE, 512
    ws = 0x100000  # 256-byte aligned, never dereferenced
    assert lib.hstu_sla_fwd_grouped(arr, 0, ws, 1 << 30, None) == _abi.ERR_INVALID_ARG
    assert lib.hstu_sla_fwd_grouped(arr, _abi.MAX_GROUPS + 1, ws, 1 << 30, None) == \
        _abi.ERR_INVALID_ARG
    assert lib.hstu_sla_fwd_grouped(arr, G, ws, 255, None) == _abi.ERR_WORKSPACE
    arr[1].d = 64
    assert lib.hstu_sla_fwd_grouped(arr, G, ws, 1 << 30, None) == _abi.ERR_UNSUPPORTED
    b = (_abi.BwdParams * 1)()
    b[0].fwd = _params(d=64, q_row_stride=256, k_row_stride=256, v_row_stride=256)
    b[0].dout = b[0].dq = b[0].dk = b[0].dv = FAKE
    b[0].dout_row_stride = b[0].dq_row_stride = b[0].dk_row_stride = b[0].dv_row_stride = 256
    assert lib.hstu_sla_bwd_grouped(b, 1, ws, 1 << 30, None) == _abi.ERR_UNSUPPORTED
    # the grouped workspace: a 256-byte header, then each group's own workspace
    T = np.array([1000, 500], np.int64)
    B, H, d = np.array([3, 2], np.int32), np.array([4, 2], np.int32), np.array([128, 128], np.int32)
    f = lib.hstu_sla_grouped_workspace_bytes
    want = 256 + sum(lib.hstu_sla_workspace_bytes(_abi.WS_BWD, int(T[i]), int(B[i]), int(H[i]), 128)
                     for i in range(2))
    assert f(_abi.WS_BWD, 2, T.ctypes.data, B.ctypes.data, H.ctypes.data, d.ctypes.data) == want
    assert f(_abi.WS_BWD, 0, T.ctypes.data, B.ctypes.data, H.ctypes.data, d.ctypes.data) == 0


def test_rab_arguments_are_checked_on_the_host(lib):
    """Bucket counts outside 1..32, a time table without timestamps and a
    table without a gradient buffer (one call or grouped) are refused before
    any CUDA call."""
    p = _params(d=128, q_row_stride=512, k_row_stride=512, v_row_stride=512)
    p.out, p.out_row_stride = FAKE, 512
    ws = 0x100000
    p.rab_pos, p.rab_pos_buckets = FAKE, 0
    assert lib.hstu_sla_fwd(ctypes.byref(p), ws, 1 << 30, None) == _abi.ERR_INVALID_ARG
    p.rab_pos_buckets = 33
    assert lib.hstu_sla_fwd(ctypes.byref(p), ws, 1 << 30, None) == _abi.ERR_INVALID_ARG
    p.rab_pos, p.rab_pos_buckets = None, 0
    p.rab_time, p.rab_time_buckets = FAKE, 8
    assert lib.hstu_sla_fwd(ctypes.byref(p), ws, 1 << 30, None) == _abi.ERR_INVALID_ARG
    p.timestamps = FAKE
    b = _abi.BwdParams()
    b.fwd = p
    b.dout = b.dq = b.dk = b.dv = FAKE
    b.dout_row_stride = b.dq_row_stride = b.dk_row_stride = b.dv_row_stride = 512
    # the time table's gradient buffer is missing
    assert lib.hstu_sla_bwd(ctypes.byref(b), ws, 1 << 30, None) == _abi.ERR_INVALID_ARG
    arr = (_abi.BwdParams * 1)(b)
    assert lib.hstu_sla_bwd_grouped(arr, 1, ws, 1 << 30, None) == _abi.ERR_INVALID_ARG


def test_truncation_lengths_follow_the_oracle_index_set():
    """The host helper that sizes the truncated buffers keeps exactly the rows
    the oracle's truncation keeps, sequence by sequence (no GPU needed)."""
    import numpy as np
    from oracle import stu as S
    from sparse_hstu_attention_b200 import stu
    rng = np.random.default_rng(5)
    for c, tail in [(0, 0), (4, 16), (32, 1024), (7, 3)]:
        lengths = rng.integers(0, 3000, size=23)
        lengths[:3] = [0, 1, c + tail]
        nts = np.minimum(rng.integers(0, 80, size=23), lengths)
        got = stu.truncated_lengths(lengths, nts, c, tail)
        for b in range(len(lengths)):
            keep, _ = S.truncation_index(np.array([0, lengths[b]]), nts[b:b + 1], c, tail)
            assert got[b] == len(keep), (b, lengths[b], nts[b], c, tail)
        assert (stu.truncated_lengths(lengths, None, c, tail) ==
                [len(S.truncation_index(np.array([0, L]), np.array([0]), c, tail)[0])
                 for L in lengths]).all()
    lib = _abi.load()
    bad = np.array([10, 5], dtype=np.int32)
    nt = np.array([2, 6], dtype=np.int32)  # more candidates than tokens
    assert lib.hstu_jagged_truncate_lengths(bad.ctypes.data, nt.ctypes.data, 2, 0, 1, None) \
        == _abi.ERR_INVALID_ARG

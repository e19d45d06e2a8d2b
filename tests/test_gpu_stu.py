"""GPU parity of the STU layer around the SLA attention: the tcgen05 GEMM in
every operand layout / epilogue the layer uses, one full layer forward +
backward, the truncation gather / scatter, and the 6-layer truncated stack,
each against oracle/stu.py (fp64) on the same seeded bf16 inputs; and the
FP8 forward projections (E4M3 GEMM, weight quantizer, layer and stack with
fp8) against oracle/fp8.py.

Tolerances: TOL (2e-2 of max|ref|) wherever both sides compute the same
values; TOL_FP8 = 6e-2 for the gradients and the stack under the FP8
forward.  There the two sides quantize activations that already differ by
the bf16 path's rounding (about 2^-8 relative), so a share of the E4M3 codes
differs by one step (2^-3 relative); the oracle alone, with its quantizer's
inputs perturbed by 2^-7 relative noise, moves its parameter gradients by up
to 3.9% and its layer output by 0.9% of their maxima."""
import math

import numpy as np
import pytest
import torch

from oracle import fp8 as F
from oracle import stu as S
from parity import assert_close
from sparse_hstu_attention_b200 import _abi, stu
from workloads import STU_LAYERS, STU_TRUNC_AFTER, draw_stu, offsets_from_lengths

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda")
TOL_FP8 = 6e-2
FIELDS = ("ln1_w", "ln1_b", "w1", "b1", "ln2_w", "ln2_b", "w2", "b2")


def f64(t):
    return t.float().cpu().numpy().astype(np.float64)


GEMM_CASES = [  # (a_mn, b_mn, epilogue, M, N, K, splits)
    (False, True, _abi.GEMM_BIAS_SILU, 300, 512, 512, 1),
    (False, True, _abi.GEMM_BIAS_RESID, 300, 512, 512, 1),
    (False, True, _abi.GEMM_STORE, 129, 1024, 256, 1),
    (False, False, _abi.GEMM_STORE, 300, 512, 2048, 1),
    (True, True, _abi.GEMM_RED_F32, 512, 2048, 1000, 4),
    (True, True, _abi.GEMM_RED_F32, 256, 512, 77, 3),
    (False, False, _abi.GEMM_RED_F32, 300, 256, 640, 2),
]


@pytest.mark.parametrize("a_mn,b_mn,epi,M,N,K,splits", GEMM_CASES)
def test_gemm_layouts_and_epilogues(a_mn, b_mn, epi, M, N, K, splits):
    g = torch.Generator().manual_seed(M * 7 + N + K)
    A = torch.randn((K, M) if a_mn else (M, K), generator=g).to(torch.bfloat16)
    B = torch.randn((K, N) if b_mn else (N, K), generator=g).to(torch.bfloat16)
    bias = torch.randn(N, generator=g)
    resid = torch.randn((M, N), generator=g).to(torch.bfloat16)
    acc0 = torch.randn((M, N), generator=g)
    a64 = f64(A).T if a_mn else f64(A)
    b64 = f64(B).T if b_mn else f64(B)
    ref = a64 @ b64.T                       # D[m][n] = sum_k A[m][k] B[n][k]
    out = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
    out2 = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
    outf = acc0.to(DEV)
    stu.gemm(A.to(DEV), B.to(DEV), M=M, N=N, K=K, a_mn_major=a_mn, b_mn_major=b_mn,
             epilogue=epi, splits=splits, bias=bias.to(DEV), resid=resid.to(DEV), out=out,
             out2=out2, outf=outf)
    torch.cuda.synchronize()
    pre = ref + f64(bias)
    if epi == _abi.GEMM_STORE:
        assert_close("D", out, ref)
    elif epi == _abi.GEMM_BIAS_SILU:
        assert_close("D + bias", out2, pre)
        assert_close("SiLU(D + bias)", out, S.silu(pre))
    elif epi == _abi.GEMM_BIAS_RESID:
        assert_close("D + bias + resid", out, pre + f64(resid))
    else:
        assert_close("acc + D", outf, f64(acc0) + ref, tol=1e-4)


def _e4m3_bytes(x: torch.Tensor) -> torch.Tensor:
    """Seeded E4M3 operands: torch's conversion of fp32 values, as bytes."""
    return x.to(torch.float8_e4m3fn).view(torch.uint8)


def _decode(b: torch.Tensor) -> np.ndarray:
    table = np.array([F.e4m3_decode(c) for c in range(256)])
    return table[b.cpu().numpy().astype(np.int64)]


F8_GEMM_CASES = [  # (epilogue, M, N, K)
    (_abi.GEMM_STORE, 300, 512, 256),
    (_abi.GEMM_STORE, 129, 1024, 208),      # K tail inside a 128-byte k block
    (_abi.GEMM_BIAS_SILU, 300, 2048, 512),
    (_abi.GEMM_BIAS_RESID, 257, 512, 1024),
]


@pytest.mark.parametrize("epi,M,N,K", F8_GEMM_CASES)
def test_fp8_gemm(epi, M, N, K):
    """E4M3 x E4M3 -> fp32 with the row / column scales in the epilogue,
    against fp64 products of the bytes as the format's fields decode them."""
    g = torch.Generator().manual_seed(M + 3 * N + 5 * K)
    A = _e4m3_bytes(torch.randn((M, K), generator=g) * 40)
    B = _e4m3_bytes(torch.randn((N, K), generator=g) * 40)
    sa = torch.rand(M, generator=g) * 2 ** -5 + 2 ** -6
    sb = torch.rand(N, generator=g) * 2 ** -5 + 2 ** -6
    bias = torch.randn(N, generator=g)
    resid = torch.randn((M, N), generator=g).to(torch.bfloat16)
    ref = (_decode(A) @ _decode(B).T) * f64(sa)[:, None] * f64(sb)[None, :]
    out = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
    out2 = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
    stu.gemm(A.to(DEV), B.to(DEV), M=M, N=N, K=K, a_mn_major=False, b_mn_major=False,
             epilogue=epi, bias=bias.to(DEV), resid=resid.to(DEV), out=out, out2=out2,
             a_scale=sa.to(DEV), b_scale=sb.to(DEV))
    torch.cuda.synchronize()
    pre = ref + f64(bias)
    if epi == _abi.GEMM_STORE:
        assert_close("D", out, ref, tol=1e-2)
    elif epi == _abi.GEMM_BIAS_SILU:
        assert_close("D + bias", out2, pre, tol=1e-2)
        assert_close("SiLU(D + bias)", out, S.silu(pre), tol=1e-2)
    else:
        assert_close("D + bias + resid", out, pre + f64(resid), tol=1e-2)


def test_fp8_weight_quantizer_is_bit_exact():
    """Codes and scales of hstu_quant_weight_e4m3 equal the oracle's per-column
    quantization byte for byte (same bf16 inputs, decisions in fp32 on both
    sides), including an all-zero column and a column with one outlier."""
    g = torch.Generator().manual_seed(11)
    K, N = 512, 2048
    W = torch.randn((K, N), generator=g) * torch.exp2(
        torch.randint(-12, 6, (1, N), generator=g).float())
    W[:, 7] = 0.0
    W[3, 9] = 3e4
    W = W.to(torch.bfloat16)
    wq, ws = stu.quantize_weight_e4m3(W.to(DEV))
    torch.cuda.synchronize()
    q, sc = F.quantize_cols(f64(W))
    assert np.array_equal(ws.cpu().numpy().astype(np.float64), sc)
    assert np.array_equal(wq.cpu().numpy(), F.e4m3_code(q).T)


def _margin(tag, name, got, ref, tol):
    """assert_close, and print the error as a fraction of max|ref| beside the
    tolerance (run with -s to see how far inside it each tensor lies)."""
    err, scale = assert_close(name, got, ref, tol=tol)
    print(f"[margin] {tag} {name}: max|err|/max|ref| = {err / max(scale, 1e-30):.2e} "
          f"(tolerance {tol:.0e})")


def _cfgs(lengths, nts, c, K1, K2, tail, trunc=True):
    H, d = 4, 128
    alpha = 1.0 / math.sqrt(d)
    tl = stu.truncated_lengths(lengths, nts, c, tail)
    full = stu.StuConfig(H, d, c, K1, K2, alpha, float(max(lengths)))
    cut = stu.StuConfig(H, d, c, K1, K2, alpha, float(max(tl)))
    return full, cut, tl


def _oracle_cfg(c: stu.StuConfig):
    return S.AttnCfg(c.H, c.d, c.contextual_len, c.K1, c.K2, c.alpha, c.N, c.ln_eps)


def _oracle_weights(lw):
    return S.Weights.of(**{k: f64(lw[k]) for k in FIELDS})


def test_stu_layer_matches_oracle():
    lengths, nts = np.array([300, 520, 180]), np.array([16, 10, 5])
    full, _, _ = _cfgs(lengths, nts, c=8, K1=128, K2=32, tail=64)
    offs = offsets_from_lengths(lengths)
    T = int(offs[-1])
    dr = draw_stu(T, T, full.d_model, 1, seed=2024, perturb=True)
    w = stu.StuWeights.from_host(dr.layers[0], DEV)
    offs_d = torch.tensor(offs, dtype=torch.int32, device=DEV)
    nts_d = torch.tensor(nts, dtype=torch.int32, device=DEV)
    out, st = stu.layer_fwd(dr.x.to(DEV), offs_d, nts_d, w, full, int(lengths.max()))
    dx, g = stu.layer_bwd(dr.dout.to(DEV), st, w, full)
    torch.cuda.synchronize()
    wo = _oracle_weights(dr.layers[0])
    ref, cache = S.layer_fwd(f64(dr.x), wo, offs, nts, _oracle_cfg(full))
    rdx, rg = S.layer_bwd(f64(dr.dout), wo, cache)
    assert_close("out", out, ref)
    assert_close("dx", dx, rdx)
    for name in FIELDS:
        assert_close("d_" + name, getattr(g, name), getattr(rg, name))


def test_stu_layer_remat_matches_plain_and_oracle():
    """Listing 1's save set (u, A, statistics): the forward output is the plain
    layer's bit for bit, the saved bytes drop from 11 to 2 rows of d_model
    bf16 per token (plus the statistics), and the backward (which recomputes
    x^, pre, U|V|Q|K and y) matches the oracle and the plain backward."""
    lengths, nts = np.array([300, 520, 180]), np.array([16, 10, 5])
    full, _, _ = _cfgs(lengths, nts, c=8, K1=128, K2=32, tail=64)
    offs = offsets_from_lengths(lengths)
    T = int(offs[-1])
    dm = full.d_model
    dr = draw_stu(T, T, dm, 1, seed=2025, perturb=True)
    w = stu.StuWeights.from_host(dr.layers[0], DEV)
    offs_d = torch.tensor(offs, dtype=torch.int32, device=DEV)
    nts_d = torch.tensor(nts, dtype=torch.int32, device=DEV)
    x, dout = dr.x.to(DEV), dr.dout.to(DEV)
    out_p, st_p = stu.layer_fwd(x, offs_d, nts_d, w, full, int(lengths.max()))
    out_r, st_r = stu.layer_fwd(x, offs_d, nts_d, w, full, int(lengths.max()), remat=True)
    dx_p, g_p = stu.layer_bwd(dout, st_p, w, full)
    dx_r, g_r = stu.layer_bwd(dout, st_r, w, full)
    torch.cuda.synchronize()
    assert torch.equal(out_r, out_p)
    assert torch.equal(st_r.u, st_p.uvqk[:, :dm]) and torch.equal(st_r.av, st_p.av)
    assert st_r.saved_bytes() == T * dm * 2 * 2 + 4 * T * 4
    assert st_p.saved_bytes() == T * dm * 2 * 11 + 4 * T * 4
    wo = _oracle_weights(dr.layers[0])
    ref, cache = S.layer_fwd(f64(dr.x), wo, offs, nts, _oracle_cfg(full))
    rdx, rg = S.layer_bwd(f64(dr.dout), wo, cache)
    assert_close("out", out_r, ref)
    assert_close("dx", dx_r, rdx)
    assert_close("dx vs plain", dx_r, f64(dx_p.cpu()), tol=1e-2)
    for name in FIELDS:
        assert_close("d_" + name, getattr(g_r, name), getattr(rg, name))
        assert_close("d_" + name + " vs plain", getattr(g_r, name),
                     f64(getattr(g_p, name).cpu()), tol=1e-2)


def test_stu_layer_head_dim_64_matches_oracle():
    """d = 64 heads (8 x 64): the attention's two-pass backward and the
    separate SiLU' / bias-gradient pass (d = 128 fuses them into the
    attention backward)."""
    lengths, nts = np.array([260, 400, 90]), np.array([12, 7, 3])
    H, d = 8, 64
    cfg = stu.StuConfig(H, d, 8, 128, 32, 1.0 / math.sqrt(d), float(lengths.max()))
    offs = offsets_from_lengths(lengths)
    T = int(offs[-1])
    dr = draw_stu(T, T, cfg.d_model, 1, seed=64, perturb=True)
    w = stu.StuWeights.from_host(dr.layers[0], DEV)
    offs_d = torch.tensor(offs, dtype=torch.int32, device=DEV)
    nts_d = torch.tensor(nts, dtype=torch.int32, device=DEV)
    out, st = stu.layer_fwd(dr.x.to(DEV), offs_d, nts_d, w, cfg, int(lengths.max()))
    dx, g = stu.layer_bwd(dr.dout.to(DEV), st, w, cfg)
    torch.cuda.synchronize()
    wo = _oracle_weights(dr.layers[0])
    ref, cache = S.layer_fwd(f64(dr.x), wo, offs, nts, _oracle_cfg(cfg))
    rdx, rg = S.layer_bwd(f64(dr.dout), wo, cache)
    assert_close("out", out, ref)
    assert_close("dx", dx, rdx)
    for name in FIELDS:
        assert_close("d_" + name, getattr(g, name), getattr(rg, name))


def test_stu_layer_fp8_forward_matches_oracle():
    """The layer with E4M3 projections against the oracle's FP8 layer (the
    same quantization rules), forward and the unchanged backward; and it does
    differ from the bf16 layer."""
    lengths, nts = np.array([300, 520, 180]), np.array([16, 10, 5])
    full, _, _ = _cfgs(lengths, nts, c=8, K1=128, K2=32, tail=64)
    offs = offsets_from_lengths(lengths)
    T = int(offs[-1])
    dr = draw_stu(T, T, full.d_model, 1, seed=2024, perturb=True)
    w = stu.StuWeights.from_host(dr.layers[0], DEV)
    q8 = stu.quantize_weights(w)
    offs_d = torch.tensor(offs, dtype=torch.int32, device=DEV)
    nts_d = torch.tensor(nts, dtype=torch.int32, device=DEV)
    x = dr.x.to(DEV)
    out, st = stu.layer_fwd(x, offs_d, nts_d, w, full, int(lengths.max()), fp8=q8)
    dx, g = stu.layer_bwd(dr.dout.to(DEV), st, w, full)
    out_bf, _ = stu.layer_fwd(x, offs_d, nts_d, w, full, int(lengths.max()))
    torch.cuda.synchronize()
    wo = _oracle_weights(dr.layers[0])
    ref, cache = S.layer_fwd(f64(dr.x), wo, offs, nts, _oracle_cfg(full), fp8=True)
    rdx, rg = S.layer_bwd(f64(dr.dout), wo, cache)
    _margin("fp8 layer", "out", out, ref, 2e-2)
    _margin("fp8 layer", "pre", st.pre, cache["pre"], TOL_FP8)
    _margin("fp8 layer", "dx", dx, rdx, 2e-2)
    for name in FIELDS:
        _margin("fp8 layer", "d_" + name, getattr(g, name), getattr(rg, name), TOL_FP8)
    diff = (out.float() - out_bf.float()).abs().max().item()
    assert diff > 1e-3 * out_bf.float().abs().max().item()


def test_truncation_gather_and_scatter_are_exact():
    lengths, nts = np.array([300, 40, 1200, 77]), np.array([16, 3, 64, 0])
    c, tail = 8, 100
    offs = offsets_from_lengths(lengths)
    T = int(offs[-1])
    x = torch.randn((T, 512), generator=torch.Generator().manual_seed(1)).to(torch.bfloat16)
    idx, new = S.truncation_index(offs, nts, c, tail)
    offs_d = torch.tensor(offs, dtype=torch.int32, device=DEV)
    nts_d = torch.tensor(nts, dtype=torch.int32, device=DEV)
    new_d = stu.truncate_offsets(offs_d, nts_d, c, tail)
    y = stu.jagged_truncate(x.to(DEV), offs_d, new_d, nts_d, c, tail, len(idx))
    torch.cuda.synchronize()
    assert np.array_equal(new_d.cpu().numpy(), new)
    assert torch.equal(y.cpu(), x[torch.from_numpy(idx)])
    z = stu.jagged_truncate(y, offs_d, new_d, nts_d, c, tail, T, scatter=True)
    ref = torch.zeros_like(x)
    ref[torch.from_numpy(idx)] = x[torch.from_numpy(idx)]
    assert torch.equal(z.cpu(), ref)


@pytest.mark.parametrize("fp8,remat", [(False, False), (True, False), (False, True)])
def test_stu_stack_matches_oracle(fp8, remat):
    """Six layers, truncation after the third to contextual + the last `tail`
    history tokens + candidates, every gradient compared; fp8: the forward
    projections in E4M3; remat: Listing 1's save set, the rest recomputed in
    the backward."""
    lengths, nts = np.array([700, 400, 1100]), np.array([20, 8, 30])
    c, tail = 16, 128
    full, cut, tl = _cfgs(lengths, nts, c=c, K1=128, K2=32, tail=tail)
    offs = offsets_from_lengths(lengths)
    T, T_out = int(offs[-1]), int(tl.sum())
    dr = draw_stu(T, T_out, full.d_model, STU_LAYERS, seed=77, perturb=True)
    ws = [stu.StuWeights.from_host(lw, DEV) for lw in dr.layers]
    stack = stu.StuStack(ws, full, cut, STU_TRUNC_AFTER, tail, fp8=fp8, remat=remat)
    offs_d = torch.tensor(offs, dtype=torch.int32, device=DEV)
    nts_d = torch.tensor(nts, dtype=torch.int32, device=DEV)
    out, ctx = stack.forward(dr.x.to(DEV), offs_d, nts_d, lengths, nts)
    dx, gs = stack.backward(dr.dout.to(DEV), ctx)
    torch.cuda.synchronize()
    wo = [_oracle_weights(lw) for lw in dr.layers]
    ref, cache = S.stack_fwd(f64(dr.x), wo, offs, nts, _oracle_cfg(full), _oracle_cfg(cut),
                             STU_TRUNC_AFTER, tail, fp8=fp8)
    rdx, rgs = S.stack_bwd(f64(dr.dout), wo, cache)
    tol = TOL_FP8 if fp8 else 2e-2
    tag = ("fp8" if fp8 else "bf16") + (" remat" if remat else "") + " stack"
    assert out.shape[0] == T_out
    _margin(tag, "out", out, ref, tol)
    _margin(tag, "dx", dx, rdx, tol)
    for i in range(STU_LAYERS):
        for name in FIELDS:
            _margin(tag, f"layer {i} d_{name}", getattr(gs[i], name), getattr(rgs[i], name), tol)


@pytest.mark.parametrize("fp8", [False, True])
def test_stu_stack_full_size_sampled(fp8):
    """The 6-layer STU stack workload at full size (16 sequences of
    U{4096..16384} tokens, truncation to 32 + 1024 + 64 after layer 3), forward
    and backward on the GPU, with bf16 or E4M3 forward projections.  Sequences
    are independent, so the oracle runs the whole stack, forward and backward,
    on the shortest sequence alone (same attention settings; per-row and
    per-column quantization make that exact for FP8 too) and its output rows
    and dx rows must match; every output and gradient must be finite.  The
    weight gradients sum over all sequences and are compared at the smaller
    sizes above."""
    from workloads import STU_TAIL, WORKLOADS, draw_lengths
    w = WORKLOADS["stu"]
    lengths = draw_lengths(w)
    nts = np.minimum(np.full(len(lengths), w.num_targets), lengths)
    c, tail = w.contextual_len, STU_TAIL
    tl = stu.truncated_lengths(lengths, nts, c, tail)
    full = stu.StuConfig(w.H, w.d, c, w.K1, w.K2, w.alpha, w.N)
    cut = stu.StuConfig(w.H, w.d, c, w.K1, w.K2, w.alpha, float(c + tail + w.num_targets))
    offs = offsets_from_lengths(lengths)
    T, T_out = int(offs[-1]), int(tl.sum())
    dr = draw_stu(T, T_out, full.d_model, STU_LAYERS, seed=w.seed)
    ws = [stu.StuWeights.from_host(lw, DEV) for lw in dr.layers]
    stack = stu.StuStack(ws, full, cut, STU_TRUNC_AFTER, tail, fp8=fp8)
    offs_d = torch.tensor(offs, dtype=torch.int32, device=DEV)
    nts_d = torch.tensor(nts, dtype=torch.int32, device=DEV)
    out, ctx = stack.forward(dr.x.to(DEV), offs_d, nts_d, lengths, nts)
    dx, gs = stack.backward(dr.dout.to(DEV), ctx)
    torch.cuda.synchronize()
    for t in [out, dx] + [getattr(g, f) for g in gs for f in FIELDS]:
        assert torch.isfinite(t.float()).all()
    tol = TOL_FP8 if fp8 else 2e-2
    wo = [_oracle_weights(lw) for lw in dr.layers]
    new = offsets_from_lengths(tl)
    b = int(np.argmin(lengths))
    s0, s1, n0, n1 = int(offs[b]), int(offs[b + 1]), int(new[b]), int(new[b + 1])
    one = np.array([0, s1 - s0])
    ref, cache = S.stack_fwd(f64(dr.x[s0:s1]), wo, one, nts[b:b + 1], _oracle_cfg(full),
                             _oracle_cfg(cut), STU_TRUNC_AFTER, tail, fp8=fp8)
    assert_close("out rows of the shortest sequence", out[n0:n1], ref, tol=tol)
    rdx, _ = S.stack_bwd(f64(dr.dout[n0:n1]), wo, cache)
    assert_close("dx rows of the shortest sequence", dx[s0:s1], rdx, tol=tol)


def test_stu_stack_full_size_two_shortest_sequences_all_gradients():
    """Every weight gradient at full sequence lengths: the two shortest
    sequences of the full-size STU draw (thousands of tokens each, the
    workload's windows, N and truncation), the workload's weights, run
    through the GPU stack as one jagged batch and compared tensor by tensor
    with the oracle's stack on the same two sequences."""
    from workloads import STU_TAIL, WORKLOADS, draw_lengths
    w = WORKLOADS["stu"]
    all_lengths = draw_lengths(w)
    pick = np.sort(np.argsort(all_lengths, kind="stable")[:2])
    lengths = all_lengths[pick]
    nts = np.minimum(np.full(len(lengths), w.num_targets), lengths)
    c, tail = w.contextual_len, STU_TAIL
    tl = stu.truncated_lengths(lengths, nts, c, tail)
    full = stu.StuConfig(w.H, w.d, c, w.K1, w.K2, w.alpha, w.N)
    cut = stu.StuConfig(w.H, w.d, c, w.K1, w.K2, w.alpha, float(c + tail + w.num_targets))
    offs = offsets_from_lengths(lengths)
    T, T_out = int(offs[-1]), int(tl.sum())
    dr = draw_stu(T, T_out, full.d_model, STU_LAYERS, seed=w.seed, perturb=True)
    ws = [stu.StuWeights.from_host(lw, DEV) for lw in dr.layers]
    stack = stu.StuStack(ws, full, cut, STU_TRUNC_AFTER, tail)
    offs_d = torch.tensor(offs, dtype=torch.int32, device=DEV)
    nts_d = torch.tensor(nts, dtype=torch.int32, device=DEV)
    out, ctx = stack.forward(dr.x.to(DEV), offs_d, nts_d, lengths, nts)
    dx, gs = stack.backward(dr.dout.to(DEV), ctx)
    torch.cuda.synchronize()
    wo = [_oracle_weights(lw) for lw in dr.layers]
    ref, cache = S.stack_fwd(f64(dr.x), wo, offs, nts, _oracle_cfg(full), _oracle_cfg(cut),
                             STU_TRUNC_AFTER, tail)
    rdx, rgs = S.stack_bwd(f64(dr.dout), wo, cache)
    tag = f"full-size pair {lengths.tolist()}"
    _margin(tag, "out", out, ref, 2e-2)
    _margin(tag, "dx", dx, rdx, 2e-2)
    for i in range(STU_LAYERS):
        for name in FIELDS:
            _margin(tag, f"layer {i} d_{name}", getattr(gs[i], name), getattr(rgs[i], name), 2e-2)

"""Pins of oracle/fp8.py (E4M3 quantization of the FP8 forward projections)
against what the format's definition and independent routines fix:

  * every byte, decoded from its sign / exponent / mantissa fields (OCP
    8-bit floating point, E4M3: bias 7, no infinities, NaN = S.1111.111),
    equals torch's float8_e4m3fn reading of the same byte, and each finite
    value rounds to itself and encodes back to its byte;
  * halfway cases round to the even mantissa, in the normal and the
    subnormal range; values past 448 saturate;
  * rounding and encoding agree with torch's float8_e4m3fn conversion on
    random fp32 values spanning the whole exponent range;
  * bf16 rounding agrees with torch's bfloat16 conversion;
  * row / column scaling maps each row's maximum to exactly +-448, keeps
    every normal value within half a step (2^-4 relative), and leaves an
    all-zero row at scale 1;
  * the quantized product stays inside the first-order error bound of E4M3
    rounding on both operands, and differs from the exact product.
"""
import numpy as np
import torch

from oracle import fp8 as F

CODES = np.arange(256)


def _torch_values():
    return torch.from_numpy(CODES.astype(np.uint8)).view(torch.float8_e4m3fn).float().numpy()


def test_every_code_decodes_as_torch_reads_it_and_round_trips():
    vals = np.array([F.e4m3_decode(int(c)) for c in CODES])
    tv = _torch_values().astype(np.float64)
    nan = np.isnan(vals)
    assert np.array_equal(np.isnan(tv), nan) and nan.sum() == 2      # 0x7F and 0xFF
    assert np.array_equal(vals[~nan], tv[~nan])
    assert vals[0x7E] == 448.0 and vals[0x01] == 2.0 ** -9 and vals[0x08] == 2.0 ** -6
    fin = vals[~nan]
    assert np.array_equal(F.e4m3_round(fin), fin)
    assert np.array_equal(F.e4m3_code(fin), CODES[~nan].astype(np.uint8))


def test_ties_to_even_and_saturation():
    cases = {
        1.0 + 1 / 16: 1.0,            # halfway between 1 and 1.125 -> even (1.0)
        1.0 + 3 / 16: 1.25,           # halfway between 1.125 and 1.25 -> even (1.25)
        2.0 ** -10: 0.0,              # half the smallest subnormal -> 0
        3 * 2.0 ** -10: 2.0 ** -8,    # halfway between 1 and 2 subnormal steps -> 2
        432.0: 448.0,                 # halfway between 416 and 448 -> even (448)
        460.0: 448.0, 464.0: 448.0, 1e9: 448.0, -1e9: -448.0,
        0.3: 0.3125,                  # nearest of 0.28125 / 0.3125
    }
    for v, want in cases.items():
        assert F.e4m3_round(np.float64(v)) == want, v
    assert F.e4m3_code(np.float64(-0.0)) == 0x80
    assert F.e4m3_code(F.e4m3_round(np.float64(-2.0 ** -11))) == 0x80


def test_rounding_matches_torch_conversion():
    rng = np.random.default_rng(7)
    x = (rng.standard_normal(400000) * np.exp2(rng.uniform(-13, 9, 400000))).astype(np.float32)
    x = np.clip(x, -447.9, 447.9)   # torch's conversion does not saturate
    t = torch.from_numpy(x).to(torch.float8_e4m3fn)
    r = F.e4m3_round(x)
    assert np.array_equal(t.float().numpy().astype(np.float64), r)
    assert np.array_equal(t.view(torch.uint8).numpy(), F.e4m3_code(r))


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(8)
    x = (rng.standard_normal(300000) * np.exp2(rng.uniform(-30, 30, 300000))).astype(np.float32)
    want = torch.from_numpy(x).bfloat16().float().numpy().astype(np.float64)
    assert np.array_equal(F.bf16_round(x), want)


def test_row_scaling():
    rng = np.random.default_rng(9)
    x = F.bf16_round(rng.standard_normal((64, 512)) * np.exp2(rng.uniform(-8, 8, (64, 1))))
    x[5] = 0.0
    q, s = F.quantize_rows(x)
    assert s[5] == 1.0 and not q[5].any()
    live = np.arange(64) != 5
    assert np.array_equal(np.abs(q[live]).max(axis=1), np.full(63, 448.0))
    # within half a step of 3 mantissa bits wherever the scaled value is normal
    deq = q * s[:, None]
    normal = np.abs(x) / s[:, None] >= 2.0 ** -6
    rel = np.abs(deq - x)[normal] / np.abs(x)[normal]
    assert rel.max() <= 2.0 ** -4 * (1 + 1e-6)
    # column scaling is row scaling of the transpose
    qc, sc = F.quantize_cols(x.T)
    assert np.array_equal(qc, q.T) and np.array_equal(sc, s)


def test_quantized_product_error_bound():
    rng = np.random.default_rng(10)
    x = F.bf16_round(rng.standard_normal((40, 256)))
    w = F.bf16_round(rng.standard_normal((256, 96)) * 0.05)
    got = F.fp8_matmul(x, w)
    exact = x @ w
    # |Q(a)Q(b) - ab| <= (2u + u^2)|a||b| per term, u = 2^-4, plus the
    # subnormal floor of each operand (half a step of 2^-9 times its scale)
    u = 2.0 ** -4
    _, xs = F.quantize_rows(x)
    _, ws = F.quantize_cols(w)
    floor_x = 2.0 ** -10 * xs[:, None] * np.ones_like(x)
    floor_w = 2.0 ** -10 * ws[None, :] * np.ones_like(w)
    bound = (2 * u + u * u) * (np.abs(x) @ np.abs(w)) + floor_x @ np.abs(w) \
        + np.abs(x) @ floor_w + floor_x @ floor_w
    assert np.all(np.abs(got - exact) <= bound)
    assert np.abs(got - exact).max() > 1e-3 * np.abs(exact).max()

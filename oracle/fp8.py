"""E4M3 quantization as the FP8 forward projections use it -- TEST
INFRASTRUCTURE ONLY (tests and the benchmark's CPU-baseline leg).

"Bending the Scaling Law Curve in Large-Scale Recommendation Systems",
section 4.2.2 (mixed-precision training and inference) and Figure 4: both
projections of a layer take FP8 operands, everything else stays BF16, and the
row-wise scale and the quantization of the activations are computed inside
the LayerNorm that precedes each projection.  Those sources fix neither the FP8
format nor the weights' scaling; the readings taken here:

  * the format is E4M3 as the OCP 8-bit floating-point specification defines
    it: 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits, subnormals
    below 2^-6 in steps of 2^-9, largest finite value 1.75 * 2^8 = 448, no
    infinities (exponent 15 with mantissa 7 is NaN);
  * conversion rounds to nearest, ties to even, and saturates to +-448;
  * an activation row is scaled by s = max|row| / 448 (1 for an all-zero row)
    so that its largest element maps to 448; a weight is scaled the same way
    per output column;
  * what gets quantized is the bf16 value the LayerNorm writes (the saved
    activation), and the scale / division / product that decide each code are
    taken in fp32, the precision the kernels take them in.

Pins: tests/test_oracle_fp8_pins.py (every one of the 256 codes decoded from
the format's fields round-trips; ties to even; saturation; agreement with
torch's float8_e4m3fn conversion; the row maximum lands on 448).
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
_INV_MAX = np.float32(1.0) / np.float32(E4M3_MAX)  # 1/448 rounded once to fp32


def bf16_round(x):
    """Round to the nearest bf16 value (ties to even), from fp32: the value a
    kernel's fp32 result takes when stored as bf16.  Returns fp64."""
    b = np.ascontiguousarray(np.asarray(x, dtype=np.float32)).view(np.uint32).astype(np.uint64)
    lsb = (b >> np.uint64(16)) & np.uint64(1)
    r = ((b + np.uint64(0x7FFF) + lsb) >> np.uint64(16)) << np.uint64(16)
    return r.astype(np.uint32).view(np.float32).astype(np.float64)


def e4m3_round(v):
    """Nearest E4M3 value of each element (ties to even, saturating)."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    with np.errstate(divide="ignore"):
        e = np.where(a > 0, np.floor(np.log2(np.where(a > 0, a, 1.0))), -6.0)
    e = np.maximum(e, -6.0)                 # below 2^-6: the subnormal step 2^-9
    q = np.exp2(e - 3.0)                    # spacing of 3 mantissa bits in [2^e, 2^(e+1))
    r = np.round(a / q) * q                 # numpy rounds halves to even
    r = np.minimum(r, E4M3_MAX)
    return np.copysign(r, v)


def e4m3_decode(code: int) -> float:
    """Value of one byte from its fields (NaN for the two NaN codes)."""
    s, e, m = (code >> 7) & 1, (code >> 3) & 15, code & 7
    if e == 15 and m == 7:
        return float("nan")
    mag = (m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return -mag if s else mag


def e4m3_code(v):
    """Byte code of each (already E4M3-representable) value; the sign bit
    follows the sign of v, so -0.0 and negative values that round to 0 give
    0x80."""
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    sign = np.signbit(v).astype(np.int64) << 7
    with np.errstate(divide="ignore"):
        e = np.where(a >= 2.0 ** -6, np.floor(np.log2(np.where(a > 0, a, 1.0))), -7.0)
    normal = a >= 2.0 ** -6
    mant_n = np.round((a / np.exp2(np.where(normal, e, 0.0)) - 1.0) * 8.0)
    mant_s = np.round(a / 2.0 ** -9)
    code = np.where(normal, ((e + 7).astype(np.int64) << 3) | mant_n.astype(np.int64),
                    mant_s.astype(np.int64))
    return (sign | code).astype(np.uint8)


def _scaled(amax):
    """fp32 scale max/448 (1 where max is 0) and its fp32 reciprocal."""
    amax = np.asarray(amax, dtype=np.float32)
    sc = np.where(amax > 0, amax * _INV_MAX, np.float32(1.0)).astype(np.float32)
    inv = (np.float32(1.0) / sc).astype(np.float32)
    return sc, inv


def quantize_rows(x):
    """Row-wise E4M3 of a matrix of bf16 values: returns (q, scale) with q the
    E4M3 values (fp64) and q[i] * scale[i] ~ x[i]."""
    x32 = np.asarray(x, dtype=np.float32)
    sc, inv = _scaled(np.abs(x32).max(axis=1))
    v = (x32 * inv[:, None]).astype(np.float32)
    return e4m3_round(v), sc.astype(np.float64)


def quantize_cols(w):
    """Column-wise E4M3 of a weight W [K][N]: (q [K][N], scale [N]) with
    q[:, n] * scale[n] ~ W[:, n]."""
    q, sc = quantize_rows(np.asarray(w, dtype=np.float32).T)
    return q.T, sc


def fp8_matmul(x, w):
    """x W with x quantized per row and W per column, products and sums in
    fp64 on the dequantized values."""
    xq, xs = quantize_rows(x)
    wq, ws = quantize_cols(w)
    return (xq * xs[:, None]) @ (wq * ws[None, :])

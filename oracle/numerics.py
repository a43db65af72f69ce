"""bf16 and FP8 E4M3 rounding, written from the formats' definitions.

TEST INFRASTRUCTURE ONLY (see the package docstring).

bf16: 1 sign, 8 exponent, 7 stored mantissa bits (8 significant bits), the
fp32 exponent range; subnormal quantum 2**-133.  Rounding is
round-to-nearest-even from the exact (fp64) value, so no double rounding.

E4M3 (OCP 8-bit floating point, "E4M3FN"): exponent bias 7, 3 mantissa bits,
no infinities, NaN = S.1111.111, largest finite 448 = 1.75 * 2**8, smallest
normal 2**-6, subnormals m * 2**-9 (m = 1..7).  The quantisation scale
convention amax / 448 ties the scale to this largest finite value (TensorRT
PR "qwen3_omni: record why FP8 is not shipped", section "Recipe that was
measured").  Encoding rounds to nearest even and saturates to +-448
("satfinite"); NaN encodes as 0x7F; the sign of zero is kept.
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
E4M3_NAN = 0x7F


def bf16_round(x) -> np.ndarray:
    """Round fp64 values to the nearest bf16 value (ties to even), returned as fp64
    (bfloat16 format definition; the block's activations are bf16 [FRT s3])."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                       # x = m * 2**e, 0.5 <= |m| < 1
    out = np.ldexp(np.rint(m * 256.0), e - 8)  # 8 significant bits
    sub = (e < -125) & (x != 0)              # |x| < 2**-126: fixed quantum 2**-133
    if np.any(sub):
        out = np.where(sub, np.ldexp(np.rint(np.ldexp(x, 133)), -133), out)
    big = np.abs(out) > 3.3895313892515355e38  # beyond the largest finite bf16
    if np.any(big):
        out = np.where(big, np.copysign(np.inf, x), out)
    return np.where(np.isnan(x), np.nan, out)


def _e4m3_value(c) -> np.ndarray:
    """Exact value of each E4M3 code from the format's fields, fp64."""
    c = np.asarray(c, dtype=np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    exp = (c >> 3) & 0xF
    man = c & 0x7
    val = np.where(exp == 0, np.ldexp(man.astype(np.float64), -9),
                   np.ldexp((8 + man).astype(np.float64), exp - 10))
    val = np.where((c & 0x7F) == 0x7F, np.nan, val)
    return sign * val


_E4M3_TABLE = _e4m3_value(np.arange(256))


def e4m3_decode(codes) -> np.ndarray:
    """Exact value of each E4M3 code (uint8 array) as fp64; 0x7F/0xFF give NaN
    (OCP E4M3 definition; FP8 E4M3 GEMM operands [FRT s1])."""
    return _E4M3_TABLE[np.asarray(codes).astype(np.uint8)]


def e4m3_encode(v) -> np.ndarray:
    """E4M3 code of each fp32 value: round to nearest even, saturate to +-448
    (OCP E4M3 definition; the 448 of the scale amax / 448 [TRT recipe])."""
    v = np.asarray(v, dtype=np.float32)
    sign = np.signbit(v).astype(np.int64) << 7
    a = np.abs(v.astype(np.float64))
    # Subnormal range (below 2**-6): the grid is k * 2**-9; k = 8 is the
    # smallest normal, whose code is also 8.
    sub_code = np.rint(np.ldexp(np.minimum(a, 1.0), 9))
    # Normal range: a = sig * 2**E with 1 <= sig < 2, mantissa rounded to 3 bits.
    m, e = np.frexp(np.where(np.isfinite(a) & (a > 0), a, 1.0))
    q = np.rint(m * 16.0)                    # = rint(sig * 8), in [8, 16]
    E = e - 1 + (q == 16)
    q = np.where(q == 16, 8, q)
    norm_code = ((E + 7) << 3) + (q.astype(np.int64) - 8)
    code = np.where(a < 2.0 ** -6, sub_code.astype(np.int64), norm_code)
    code = np.where(a > E4M3_MAX, 0x7E, np.minimum(code, 0x7E))
    code = code | sign
    code = np.where(np.isnan(a), E4M3_NAN, code)
    return code.astype(np.uint8)


def bf16_bits_to_f64(bits) -> np.ndarray:
    """bf16 bit patterns (uint16) to their exact fp64 values (bfloat16 format definition)."""
    b = np.asarray(bits, dtype=np.uint32) << 16
    return b.view(np.float32).astype(np.float64)

"""Host checks of the arithmetic the quantisation kernels rely on.

The GPU computes the block scale fl32(amax / 448) without dividing: q0 =
fl32(amax * R) with R = fl32(1/448), then q1 = fl32(q0 + fl32(amax - q0 * 448) * R)
(two fused multiply-adds).  Every amax the kernels see is a bf16 value, so the
identity q1 == fl32(amax / 448) can be checked for all of them; below 2^-100 the
kernels divide.  The fused multiply-adds are evaluated here in exact rational
arithmetic with one final rounding to fp32, as the hardware FMA does.
"""
from fractions import Fraction as F

import numpy as np


def _rn32(x: F) -> np.float32:
    """Round an exact rational to the nearest fp32 (ties to even), normal range."""
    if x == 0:
        return np.float32(0.0)
    sign = -1 if x < 0 else 1
    x = abs(x)
    e = x.numerator.bit_length() - x.denominator.bit_length()
    while F(2) ** e > x:
        e -= 1
    while F(2) ** (e + 1) <= x:
        e += 1
    scale = F(2) ** (23 - e)
    m = x * scale
    fl = m.numerator // m.denominator
    rem = m - fl
    if rem > F(1, 2) or (rem == F(1, 2) and fl % 2 == 1):
        fl += 1
    return np.float32(sign * float(F(fl) / scale))


def test_rn32_helper_matches_numpy_rounding():
    rng = np.random.default_rng(3)
    for v in rng.standard_normal(2000) * 10.0 ** rng.integers(-20, 20, 2000):
        assert _rn32(F(float(v))) == np.float32(v)


def test_scale_by_fma_correction_equals_ieee_division_for_every_bf16_amax():
    R = np.float32(1.0) / np.float32(448.0)
    fr = F(float(R))
    bits = np.arange(0x0D80, 0x7F80, dtype=np.uint32) << 16   # 2^-100 .. the largest finite bf16
    amax = bits.view(np.float32)
    ref = amax / np.float32(448.0)
    q0 = (amax * R).astype(np.float32)
    bad = 0
    for a, q, want in zip(amax.tolist(), q0.tolist(), ref.tolist()):
        rem = _rn32(F(a) - F(q) * 448)
        got = _rn32(F(q) + F(float(rem)) * fr)
        bad += got != np.float32(want)
    assert bad == 0, f"{bad} bf16 amax values where the corrected product differs from the quotient"

"""Arithmetic identities the CUDA kernels rely on, proven on the host in exact arithmetic.

The kernels compute the block scale's b / 6 (fp4_optimization.py, quantize_weight_to_float4:
block_amax / FLOAT4_MAX) without a division routine: q0 = RN(b * c) with c = RN(1/6), then
one Markstein correction, q = RN(q0 + RN(b - 6 q0) * c) (each step one fp32 rounding, the
last two fused multiply-adds).  That form must equal the correctly rounded quotient RN(b / 6)
for every value b the kernels can meet: the largest |x| of a block, a non-negative bf16.
This test checks every positive finite bf16 value, subnormals included, with rationals and
an exact fp32 rounding written here from the format's definition.
"""
import math
import struct
from fractions import Fraction as F


def rn32(q: F) -> F:
    """Round a rational to the nearest fp32 value, ties to even (subnormals included; the
    values here never overflow)."""
    if q == 0:
        return F(0)
    sign = -1 if q < 0 else 1
    a = abs(q)
    e = math.floor(math.log2(a.numerator) - math.log2(a.denominator))
    while F(2) ** e > a:
        e -= 1
    while F(2) ** (e + 1) <= a:
        e += 1
    ulp = F(2) ** (max(e, -126) - 23)
    m = a / ulp
    fl = m.numerator // m.denominator
    rem = m - fl
    if rem > F(1, 2) or (rem == F(1, 2) and fl % 2 == 1):
        fl += 1
    return sign * fl * ulp


def test_rn32_on_known_values():
    assert rn32(F(1, 3)) == F(struct.unpack("<f", struct.pack("<I", 0x3EAAAAAB))[0])
    assert rn32(F(1, 6)) == F(struct.unpack("<f", struct.pack("<I", 0x3E2AAAAB))[0])
    assert rn32(F(2) ** -149) == F(2) ** -149           # smallest subnormal
    assert rn32(F(2) ** -150) == 0                       # half of it: tie to even (zero)
    assert rn32(F(3) * F(2) ** -151) == F(2) ** -149     # above the tie


def test_div6_by_reciprocal_and_one_correction_is_exact_for_every_bf16():
    c = rn32(F(1, 6))
    wrong_plain = 0
    for bits in range(1, 0x7F80):  # every positive finite bf16
        b = F(struct.unpack("<f", struct.pack("<I", bits << 16))[0])
        want = rn32(b / 6)
        q0 = rn32(b * c)
        wrong_plain += q0 != want
        r = rn32(b - 6 * q0)
        assert rn32(q0 + r * c) == want, f"bf16 {bits:#06x}"
    assert wrong_plain > 0  # the correction step is needed: one multiply alone is not exact

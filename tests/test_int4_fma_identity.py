"""The decode kernels' single-FMA INT4 dequantisation, checked exhaustively in
exact arithmetic (no GPU).

For an offset-binary nibble u (q = u - 8) and a bf16 scale s the kernels want
bf16(q * s).  Masking a code word leaves bf16 bit patterns u (nibble in bits
3:0) or 16 u (bits 7:4); they compute fma(v, m, b) in bf16 with v that
pattern's value, m = s * 2^133 (resp. s * 2^129) and b = -8 s, the three
built by adding 0x4280, 0x4080 and 0x8180 to the scale's bit pattern.  The
FMA rounds once, so the identity holds when v * m + b equals q * s exactly.
This file checks, for every normal bf16 scale below 2^-5 (the fast path's
range) and every nibble in both positions, that the added patterns are the
intended values and that the sum is exact; and that the scales outside the
range are the ones whose added patterns would not be those values.
"""
from fractions import Fraction

import pytest

TWO = Fraction(2)


def bf16_value(bits: int) -> Fraction:
    """Exact value of a finite bf16 bit pattern."""
    bits &= 0xFFFF
    sign = -1 if bits & 0x8000 else 1
    e = (bits >> 7) & 0xFF
    m = bits & 0x7F
    assert e != 0xFF, "not finite"
    if e == 0:
        return sign * Fraction(m, 128) * TWO ** -126
    return sign * (1 + Fraction(m, 128)) * TWO ** (e - 127)


def test_patterns_below_256_are_linear():
    # exponent field 0 (subnormals) and 1: value = pattern * 2^-133
    for p in range(256):
        assert bf16_value(p) == p * TWO ** -133


# every normal bf16 scale below 2^-5 (INT4 scales are amax / 7: never negative)
FAST_SCALES = list(range(0x0080, 0x3D00))


def test_fast_path_scale_range():
    assert bf16_value(0x3CFF) < TWO ** -5 <= bf16_value(0x3D00)
    assert bf16_value(0x0080) == TWO ** -126  # the smallest normal


@pytest.mark.parametrize("chunk", range(8))
def test_single_fma_is_exact_for_every_fast_path_scale_and_nibble(chunk):
    scales = FAST_SCALES[chunk::8]
    lo = [bf16_value(u) for u in range(16)]        # nibble in bits 3:0
    hi = [bf16_value(u << 4) for u in range(16)]   # nibble in bits 7:4
    for sb in scales:
        s = bf16_value(sb)
        m0, m1, b = bf16_value(sb + 0x4280), bf16_value(sb + 0x4080), bf16_value(sb + 0x8180)
        assert m0 == s * TWO ** 133 and m1 == s * TWO ** 129 and b == -8 * s, hex(sb)
        for u in range(16):
            assert lo[u] * m0 + b == (u - 8) * s
            assert hi[u] * m1 + b == (u - 8) * s


def test_scales_outside_the_range_need_the_two_step_path():
    # from 2^-5 up, s * 2^133 leaves the finite bf16 range (exponent field 255 or beyond)
    assert ((0x3D00 + 0x4280) >> 7) & 0xFF == 0xFF
    # subnormal scales: adding to the exponent field does not multiply by a power of two
    for sb in (0x0001, 0x0040, 0x007F):
        assert bf16_value(sb + 0x4280) != bf16_value(sb) * TWO ** 133

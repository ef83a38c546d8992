"""Exact rounding of rationals to binary32 and bf16 (round to nearest, ties to
even, normal range), written from the formats' definitions: the worked examples
of the oracle pins derive their expected values with these, in exact arithmetic,
independently of numpy's and the oracle's conversions."""
from fractions import Fraction


def _round_to_bits(x: Fraction, p: int) -> Fraction:
    """x rounded to p significant bits (no exponent limits)."""
    if x == 0:
        return Fraction(0)
    sign = -1 if x < 0 else 1
    a = abs(x)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    q = Fraction(2) ** (e - p + 1)  # spacing of the binade [2^e, 2^(e+1))
    return sign * round(a / q) * q  # Fraction.__round__ rounds half to even


def fl32(x) -> Fraction:
    """Nearest binary32 value (24 significant bits) of a rational in the normal range."""
    return _round_to_bits(Fraction(x), 24)


def bf16(x) -> Fraction:
    """Nearest bf16 value (8 significant bits) of a rational in the normal range."""
    return _round_to_bits(Fraction(x), 8)


def f32_of_bits(u: int) -> Fraction:
    """The binary32 value with bit pattern u (finite, normal), exactly."""
    sign = -1 if u >> 31 else 1
    e = (u >> 23) & 0xFF
    m = u & 0x7FFFFF
    assert 0 < e < 255
    return sign * Fraction(0x800000 | m, 1 << 23) * Fraction(2) ** (e - 127)

"""Exact rational emulation of IEEE binary32 / bf16 rounding, for pinning the
CPU oracle against the mathematics rather than against itself.

Every value is a ``fractions.Fraction``; ``rn32`` rounds a rational to the
nearest binary32 number (ties to even, with subnormals), ``rn_bf16`` to the
nearest bf16 number.  Nothing here calls a floating-point operation on the
value being rounded.
"""
from fractions import Fraction
import struct


def _rn_binary(r: Fraction, mant_bits: int, emin: int) -> Fraction:
    """Round r to the nearest number with ``mant_bits`` significand bits
    (including the hidden bit) and minimum normal exponent ``emin``; ties go
    to the even significand.  Overflow is not modelled (callers stay in range).
    """
    if r == 0:
        return Fraction(0)
    sign = -1 if r < 0 else 1
    a = -r if r < 0 else r
    # exponent e with 2^e <= a < 2^(e+1)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e = max(e, emin)  # subnormal range: fixed quantum
    quantum = Fraction(2) ** (e - (mant_bits - 1))
    n = a / quantum
    k = round(n)  # Fraction.__round__ rounds half to even
    return sign * k * quantum


def rn32(r) -> Fraction:
    return _rn_binary(Fraction(r), 24, -126)


def rn_bf16(r) -> Fraction:
    return _rn_binary(Fraction(r), 8, -126)


def f32_bits(v: Fraction) -> int:
    """Bits of an exactly representable binary32 value."""
    f = float(v)
    assert Fraction(f) == v
    return struct.unpack("<I", struct.pack("<f", f))[0]


def bf16_bits(v: Fraction) -> int:
    b = f32_bits(v)
    assert b & 0xFFFF == 0, "not a bf16 value"
    return b >> 16


def from_bf16_bits(h: int) -> Fraction:
    return Fraction(struct.unpack("<f", struct.pack("<I", (h & 0xFFFF) << 16))[0])


def from_f32(x) -> Fraction:
    return Fraction(float(struct.unpack("<f", struct.pack("<f", float(x)))[0]))


def round_half_even(r: Fraction) -> int:
    return round(r)


def quant_element(x: Fraction, amax: Fraction):
    """The quantisation of one element, each fp32 step rounded exactly once:
    s = RN32(amax / 127); v = RN32(x / s); q = clamp(rint_even(v), -127, 127).
    """
    if amax == 0:
        return Fraction(0), 0
    s = rn32(amax / 127)
    v = rn32(x / s)
    q = max(-127, min(127, round_half_even(v)))
    return s, q


def epilogue_element(acc: int, a_s: Fraction, w_s: Fraction, bias) -> int:
    """bf16 bits of RN_bf16(RN32(RN32(RN32(acc) * a_s) * w_s) [+ bias])."""
    t = rn32(Fraction(acc))
    t = rn32(t * a_s)
    t = rn32(t * w_s)
    if bias is not None:
        t = rn32(t + bias)
    r = rn_bf16(t)
    if r == 0:
        # sign of zero: follows IEEE for the operations above
        return None
    return bf16_bits(r)

"""Exact-rational brute force of the block codecs, written independently of the
oracle (Python ``fractions`` + integer arithmetic; no floating point on the path).

Used only to pin the oracle on tiny inputs.  Format definitions:
  * binary32/binary16/bfloat16: IEEE-754 style binary formats, round to nearest,
    ties to even (the rounding the codec definitions name).
  * E4M3 per "FP8 Formats for Deep Learning" (abstract): 4 exponent bits,
    3 mantissa bits, no infinities, one NaN mantissa pattern.  The value table
    below is built from the bit fields and the nearest entry is found by search.
"""
import bisect
from fractions import Fraction
import math
import struct

HALF = Fraction(1, 2)


def floor_log2(fr: Fraction) -> int:
    """floor(log2(fr)) for fr > 0, by integer bit lengths (exact)."""
    num, den = fr.numerator, fr.denominator
    e = num.bit_length() - den.bit_length()
    # 2^e <= num/den < 2^(e+1) after at most one correction
    if e >= 0:
        if num < (den << e):
            e -= 1
    else:
        if (num << -e) < den:
            e -= 1
    return e


def round_half_even(fr: Fraction) -> int:
    f = math.floor(fr)
    rem = fr - f
    if rem > HALF:
        return f + 1
    if rem < HALF:
        return f
    return f if f % 2 == 0 else f + 1


def round_binary(fr: Fraction, p: int, emin: int) -> Fraction:
    """Nearest value with a p-bit significand and exponent >= emin (ties to even)."""
    if fr == 0:
        return Fraction(0)
    sign = -1 if fr < 0 else 1
    a = abs(fr)
    e = max(floor_log2(a), emin)
    quantum = Fraction(2) ** (e - p + 1)
    return sign * round_half_even(a / quantum) * quantum


def rn32(fr):
    return round_binary(Fraction(fr), 24, -126)


def rn16_sat(fr):
    """binary16 RNE with the codec's saturation at 65504 (an overflow becomes 65504)."""
    r = round_binary(Fraction(fr), 11, -14)
    if abs(r) > 65504:
        r = Fraction(65504) * (1 if r > 0 else -1)
    return r


def f32_exact(x: float) -> Fraction:
    """Exact value of a binary32 number (Python floats are binary64, a superset)."""
    return Fraction(struct.unpack("<f", struct.pack("<f", x))[0])


def bf16_exact(bits: int) -> Fraction:
    return Fraction(struct.unpack("<f", struct.pack("<I", (bits & 0xFFFF) << 16))[0])


# ---- E4M3 value table built from the bit fields -----------------------------
def e4m3_value(code: int):
    sign = -1 if code & 0x80 else 1
    ef, mf = (code >> 3) & 0xF, code & 0x7
    if ef == 0xF and mf == 0x7:
        return None                                     # the single NaN pattern
    if ef == 0:
        return sign * Fraction(mf, 8) * Fraction(2) ** -6
    return sign * (1 + Fraction(mf, 8)) * Fraction(2) ** (ef - 7)


E4M3_POS = sorted((e4m3_value(c), c) for c in range(0x00, 0x7F))     # +0 .. 448
E4M3_VALUES = [v for v, _ in E4M3_POS]


def e4m3_rne_satfinite(fr: Fraction) -> int:
    """Nearest finite E4M3 code (ties to the even mantissa), saturating at 448.

    The table is sorted, so the nearest entry is one of the two that bracket |fr|.
    """
    sign = 0x80 if fr < 0 else 0x00
    a = abs(fr)
    if a >= 448:
        return sign | 0x7E
    k = bisect.bisect_left(E4M3_VALUES, a)
    cands = [E4M3_POS[i] for i in (k - 1, k) if 0 <= i < len(E4M3_POS)]
    best = None
    for v, c in cands:
        d = abs(v - a)
        if best is None or d < best[0] or (d == best[0] and (c & 1) == 0):
            best = (d, c)
    return sign | best[1]


# ---- codec brute force on one 32-element block ------------------------------
def quant_block_int(xs, bits):
    """xs: Fractions (exact inputs).  Returns (scale as Fraction, list of codes)."""
    qmax = 2 ** (bits - 1) - 1
    a = max(abs(x) for x in xs)
    s = rn16_sat(rn32(a / qmax))
    codes = []
    for x in xs:
        q = 0 if s == 0 else max(-qmax, min(qmax, round_half_even(x / s)))
        codes.append(q + 2 ** (bits - 1))
    return s, codes


def quant_block_fp8(xs):
    a = max(abs(x) for x in xs)
    s = rn32(a / 448)
    if s < Fraction(2) ** -126:
        return Fraction(0), [0] * len(xs)
    inv = rn32(1 / s)
    return s, [e4m3_rne_satfinite(rn32(x * inv)) for x in xs]


# ---- MXFP4: E2M1 elements with one power-of-two (E8M0) scale per block -------
# The eight E2M1 magnitudes, listed in code order 0..7 (1 sign bit above them).
E2M1_MAGNITUDES = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2),
                   Fraction(2), Fraction(3), Fraction(4), Fraction(6)]


def e2m1_rne_satfinite(fr: Fraction, negative: bool) -> int:
    """Nearest E2M1 code to a real value by search over the eight magnitudes:
    ties go to the code with an even mantissa bit (code & 1 == 0), magnitudes
    above 6 saturate, and the sign bit follows `negative` (so -0 keeps it)."""
    a = abs(fr)
    best = None
    for c, v in enumerate(E2M1_MAGNITUDES):
        d = abs(v - a)
        if best is None or d < best[0] or (d == best[0] and (c & 1) == 0):
            best = (d, c)
    code = best[1] if a <= 6 else 7
    return code | (0x8 if negative else 0)


def mx_shared_exponent(a: Fraction) -> int:
    """The integer E with 4 * 2^E <= a < 8 * 2^E (the absmax scaled into the
    top binade of E2M1), clamped to the E8M0 range; -127 for a == 0.  Found by
    search from a bracket, not by a logarithm formula."""
    if a == 0:
        return -127
    E = 0
    while Fraction(4) * Fraction(2) ** E > a:
        E -= 1
    while Fraction(8) * Fraction(2) ** E <= a:
        E += 1
    return max(-127, min(127, E))


def quant_block_mxfp4(xs, negs):
    """xs: exact values, negs: their sign bits.  Returns (E, codes)."""
    E = mx_shared_exponent(max(abs(x) for x in xs))
    return E, [e2m1_rne_satfinite(x / Fraction(2) ** E, n) for x, n in zip(xs, negs)]

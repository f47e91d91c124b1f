"""Exact-arithmetic helpers for pinning the oracle (test-only, no oracle code).

These restate nothing from the oracle: bf16 rounding here is done either by
exhaustive comparison of neighbouring bf16 values with exact rationals
(``fractions.Fraction``) or by integer manipulation of the float64 bit
pattern, and the second is itself checked against the first.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np


def bf16_value(bits: int) -> Fraction:
    """Exact value of a finite bf16 bit pattern."""
    f = np.array([bits << 16], dtype=np.uint32).view(np.float32)[0]
    return Fraction(float(f))


def bf16_round_bruteforce(v: float) -> int:
    """Nearest bf16 to the double ``v`` (ties to the even pattern), found by
    comparing the exact distance to every bf16 pattern near ``v``."""
    if v == 0.0:
        return 0x8000 if np.signbit(v) else 0
    sign = 0x8000 if v < 0 else 0
    a = abs(v)
    if a >= 2.0 ** 128:
        return sign | 0x7F80
    # A start point within a couple of patterns of the answer.
    with np.errstate(over="ignore"):
        f32 = np.float32(a)
    b0 = min(0x7F7F, int(np.array([f32], dtype=np.float32).view(np.uint32)[0]) >> 16)
    target = Fraction(a)
    best = None
    for b in range(max(0, b0 - 3), min(0x7F7F, b0 + 3) + 1):
        d = abs(bf16_value(b) - target)
        key = (d, b & 1)  # nearer first; on a tie the even pattern
        if best is None or key < best[0]:
            best = (key, b)
    b = best[1]
    # Above the largest finite value: rounds to inf when at least half an ulp past it.
    top = bf16_value(0x7F7F)
    if target > top and target - top >= Fraction(2) ** 119:
        return sign | 0x7F80
    return sign | b


def bf16_round_bits64(v: np.ndarray) -> np.ndarray:
    """Vectorised nearest-even rounding of float64 to bf16 bits, from the
    float64 bit pattern (normal bf16 range and zero only; checked against
    ``bf16_round_bruteforce`` in the tests)."""
    v = np.ascontiguousarray(v, dtype=np.float64)
    b = v.view(np.uint64)
    sign = ((b >> np.uint64(63)) & np.uint64(1)).astype(np.uint32) << np.uint32(15)
    exp = ((b >> np.uint64(52)) & np.uint64(0x7FF)).astype(np.int64) - 1023
    mant = b & np.uint64((1 << 52) - 1)
    kept = (mant >> np.uint64(45)).astype(np.int64)
    rem = mant & np.uint64((1 << 45) - 1)
    half = np.uint64(1 << 44)
    up = (rem > half) | ((rem == half) & ((kept & 1) == 1))
    body = ((exp + 127) << 7) + kept + up.astype(np.int64)
    body = np.where(exp + 127 >= 255, 0x7F80, body)
    zero = (b & np.uint64((1 << 63) - 1)) == 0
    if np.any(~zero & (exp < -126)):
        raise ValueError("subnormal bf16 results are outside this helper's range")
    body = np.where(zero, 0, body)
    return (sign | body.astype(np.uint32)).astype(np.uint16)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def f64_to_bf16_bits(vals) -> np.ndarray:
    """Exact-valued doubles (already bf16-representable) -> bf16 bits."""
    f = np.asarray(vals, dtype=np.float64).astype(np.float32)
    assert np.all(f.astype(np.float64) == np.asarray(vals, dtype=np.float64))
    bits = f.view(np.uint32)
    assert np.all((bits & np.uint32(0xFFFF)) == 0), "value is not a bf16"
    return (bits >> np.uint32(16)).astype(np.uint16)


# ---- formats beyond bf16 (exact rationals; nothing here calls the oracle) ----

def round_half_even(v: Fraction) -> int:
    """Nearest integer to an exact rational, ties to the even integer."""
    fl = v.numerator // v.denominator
    rem = v - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        return fl + 1
    return fl


def _floor_log2(a: Fraction) -> int:
    """k with 2^k <= a < 2^(k+1), for a > 0."""
    k = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** k > a:
        k -= 1
    while Fraction(2) ** (k + 1) <= a:
        k += 1
    return k


def f32_round(v: Fraction) -> Fraction:
    """Float32 nearest to an exact rational (ties to even, subnormals kept,
    no overflow handling: callers stay inside the finite range)."""
    if v == 0:
        return Fraction(0)
    sign = -1 if v < 0 else 1
    a = abs(v)
    e = max(_floor_log2(a), -126)
    ulp = Fraction(2) ** (e - 23)
    return sign * round_half_even(a / ulp) * ulp


def e4m3_table():
    """(value, code) of the 127 non-negative finite OCP E4M3 codes 0x00..0x7E:
    exponent field 0 holds m * 2^-9, field f > 0 holds (1 + m/8) * 2^(f-7)."""
    out = []
    for code in range(0x7F):
        f, m = code >> 3, code & 7
        val = Fraction(m, 2 ** 9) if f == 0 else (1 + Fraction(m, 8)) * Fraction(2) ** (f - 7)
        out.append((val, code))
    return out


_E4M3 = e4m3_table()


def e4m3_nearest(v: Fraction) -> int:
    """E4M3 code nearest to v by exhaustive comparison (ties to the even code,
    magnitudes above 448 saturate to 448)."""
    sign = 0x80 if v < 0 else 0
    a = abs(v)
    if a > 448:
        return sign | 0x7E
    best = min(_E4M3, key=lambda vc: (abs(vc[0] - a), vc[1] & 1))
    return sign | best[1]


def pow2_ceil_exponent(v: Fraction) -> int:
    """Smallest k with 2^k >= v (v > 0)."""
    k = _floor_log2(v)
    return k if Fraction(2) ** k == v else k + 1


def fp16_nearest(v: Fraction) -> int:
    """IEEE binary16 bit pattern nearest to an exact rational, by comparing the
    exact distance to every finite half value near a start point (ties to the
    even pattern; at or beyond 65520 infinity)."""
    sign = 0x8000 if v < 0 else 0
    a = abs(v)
    if a >= 65520:
        return sign | 0x7C00
    with np.errstate(over="ignore"):
        start = int(np.array([float(a)], np.float64).astype(np.float16).view(np.uint16)[0])
    start = min(start, 0x7BFF)
    best = None
    for bits in range(max(0, start - 4), min(0x7BFF, start + 4) + 1):   # a start point +- 4 patterns
        f, m = bits >> 10, bits & 0x3FF
        val = Fraction(m, 2 ** 24) if f == 0 else (1 + Fraction(m, 1024)) * Fraction(2) ** (f - 15)
        key = (abs(val - a), bits & 1)
        if best is None or key < best[0]:
            best = (key, bits)
    return sign | best[1]

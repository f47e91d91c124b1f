"""The whole oracle against a straight-line brute-force restatement on tiny
inputs (no GPU).

The restatement shares nothing with the oracle's C++: the forward and
backward values are computed in 60-digit decimal arithmetic (``decimal``),
each rounded to the nearest bf16 by comparing exact distances to the
neighbouring bf16 values (``fractions``), and the quantization uses exact
rationals: the scale is amax/127 rounded once to float32, each code the
round-half-even of the quotient rounded once to float32.  On M = 4 tokens
(a tail token group of 4) and K = 128 channels, every output byte of the
oracle must equal it.
"""
from __future__ import annotations

from decimal import Decimal, getcontext
from fractions import Fraction

import numpy as np
import pytest

import oracle
import workloads as W
from tests.exact import bf16_value, f32_round, round_half_even


def _bf16_nearest(t: Fraction) -> int:
    """Nearest finite bf16 pattern to an exact rational, ties to even."""
    if t == 0:
        return 0
    sign = 0x8000 if t < 0 else 0
    a = abs(t)
    f = np.float32(float(a))
    b0 = min(0x7F7F, int(np.array([f], dtype=np.float32).view(np.uint32)[0]) >> 16)
    best = None
    for b in range(max(0, b0 - 3), min(0x7F7F, b0 + 3) + 1):
        key = (abs(bf16_value(b) - a), b & 1)
        if best is None or key < best[0]:
            best = (key, b)
    return sign | best[1]


def _dec(fr: Fraction) -> Decimal:
    return Decimal(fr.numerator) / Decimal(fr.denominator)


def _stage1(g: Fraction, u: Fraction, dy: Fraction):
    gd, ud, dyd = _dec(g), _dec(u), _dec(dy)
    s = Decimal(1) / (Decimal(1) + (-gd).exp())
    silu = gd * s
    dsilu = s * (Decimal(1) + gd * (Decimal(1) - s))
    return (_bf16_nearest(Fraction(silu * ud)), _bf16_nearest(Fraction(dyd * ud * dsilu)),
            _bf16_nearest(Fraction(dyd * silu)))


def _quant(vals):
    """Codes and scale of one group of exact bf16 values."""
    amax = max(abs(v) for v in vals)
    if amax == 0:
        return [0] * len(vals), Fraction(1)
    scale = f32_round(amax / 127)
    return [max(-127, min(127, round_half_even(f32_round(v / scale)))) for v in vals], scale


@pytest.mark.parametrize("seed,outliers", [(2, 0.0), (8, 0.05)])
def test_whole_oracle_equals_bruteforce_on_4x128(seed, outliers):
    getcontext().prec = 60
    M, K, G = 4, 128, 128
    w = W.small_workload(M, K, seed=seed, sigma_x=2.0, sigma_grad_y=0.5, outlier_frac=outliers,
                         outlier_mult=20.0)
    x, gy = W.make_inputs(w)
    y = np.zeros((M, K), np.uint16)
    dg = np.zeros((M, K), np.uint16)
    du = np.zeros((M, K), np.uint16)
    for m in range(M):
        for k in range(K):
            y[m, k], dg[m, k], du[m, k] = _stage1(bf16_value(int(x[m, k])), bf16_value(int(x[m, K + k])),
                                                  bf16_value(int(gy[m, k])))
    giq, gis, yqt, yst = oracle.silu_dot_fwd_bwd_quant_fuse(x, gy)
    assert np.array_equal(oracle.swiglu_bwd_bf16(x, gy)[0], y)
    for m in range(M):
        for half, src in ((0, dg), (1, du)):
            q, s = _quant([bf16_value(int(v)) for v in src[m]])
            assert list(giq[m, half * K:(half + 1) * K]) == q, (m, half)
            assert Fraction(float(gis[m, half])) == s, (m, half)
    for k in range(K):
        q, s = _quant([bf16_value(int(y[m, k])) for m in range(M)])
        assert list(yqt[k]) == q, k
        assert Fraction(float(yst[k, 0])) == s, k

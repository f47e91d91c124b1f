"""Pins of the forward-side oracle (SwiGLU forward + q8_1 rows, the
activation path whose launcher is kquant_swiglu_q8_1_rows on the page with
the K-quant kernels: h = bf16(swiglu(gate, up) * w[row]), then 36-byte q8_1
blocks of 32 int8 + half2 (d, sum)), to things other than the oracle (no GPU):
numpy's float16 conversion, exhaustive nearest-value search with exact
rationals, closed-form cases, and invariants of the block format.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np
import pytest

import oracle
import workloads as W
from tests.exact import (bf16_round_bits64, bf16_to_f64, bf16_value, f32_round, f64_to_bf16_bits,
                         fp16_nearest, round_half_even)


def _half_tricky(rng, n):
    vals = []
    for _ in range(n):
        e = int(rng.integers(-26, 16))
        m = int(rng.integers(0, 1024))
        lo = (1 + Fraction(m, 1024)) * Fraction(2) ** e if e >= -14 else Fraction(m, 2 ** 24)
        step = Fraction(2) ** (max(e, -14) - 10)
        for v in (lo, lo + step / 2, lo + step / 2 + step / 2 ** 20, lo + step / 2 - step / 2 ** 20):
            vals.append(float(v) * (-1 if rng.random() < 0.5 else 1))
    return vals


def test_fp16_rne_against_numpy_float16_conversion():
    rng = np.random.default_rng(1)
    vals = np.array(_half_tricky(rng, 500) + list(rng.normal(0, 100, 2000)) + [65504.0, 65519.0, 65520.0,
                                                                                 1e6, -7e4, 0.0], np.float64)
    with np.errstate(over="ignore"):
        want = vals.astype(np.float16).view(np.uint16)
    got = np.array([oracle.fp16_rne(float(v)) for v in vals], np.uint16)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, [(vals[i], hex(got[i]), hex(want[i])) for i in bad[:5]]


def test_fp16_rne_bruteforce_exact_rationals():
    rng = np.random.default_rng(2)
    for v in _half_tricky(rng, 40):
        assert oracle.fp16_rne(v) == fp16_nearest(Fraction(v)), v


def _expected_block(h_bits):
    """A q8_1 block from its definition, with exact rationals."""
    vals = [bf16_value(int(b)) for b in h_bits]
    amax = max(abs(v) for v in vals)
    if amax == 0:
        return bytes(36)
    d = f32_round(amax / 127)
    q = [max(-127, min(127, round_half_even(f32_round(v / d)))) for v in vals]
    d16 = fp16_nearest(d)
    s16 = fp16_nearest(d * sum(q))
    return (np.array([d16, s16], np.uint16).tobytes() + np.array(q, np.int8).tobytes())


def _bf16_exact(v):
    v = np.where(np.abs(v) < 2.0 ** -126, 0.0, v)
    return bf16_to_f64(bf16_round_bits64(v))


def test_q8_1_block_against_its_definition():
    rng = np.random.default_rng(3)
    groups = [f64_to_bf16_bits(_bf16_exact(rng.normal(0, sc, 32))) for sc in (1.0, 1e-3, 300.0, 1e-6)]
    groups.append(np.zeros(32, np.uint16))
    groups.append(f64_to_bf16_bits(np.full(32, -0.75)))
    for g in groups:
        assert oracle.q8_1_block(g).tobytes() == _expected_block(g)


def test_q8_1_block_invariants():
    rng = np.random.default_rng(4)
    for sc in (1.0, 0.05, 40.0):
        g = f64_to_bf16_bits(_bf16_exact(rng.normal(0, sc, 32)))
        blk = oracle.q8_1_block(g)
        d, s = blk[:4].view(np.float16).astype(np.float64)
        q = blk[4:].view(np.int8).astype(np.int64)
        v = bf16_to_f64(g)
        assert np.abs(q).max() == 127 and q[np.argmax(np.abs(v))] == np.sign(v[np.argmax(np.abs(v))]) * 127
        assert np.all(np.abs(q * d - v) <= d * 0.51 + np.abs(v) * 2 ** -10)   # fp16 d: rel. 2^-11
        assert abs(s - d * q.sum()) <= abs(d * q.sum()) * 2 ** -10 + 2 ** -24
        assert np.all((np.sign(q) == np.sign(v)) | (q == 0))


def _closed_case(rows, inter, limit):
    """gate = 32 (sigma(32) = 1 - 1.3e-14, so silu(32) * u * w rounds to 32*u*w
    whenever 32*u*w has at most 8 significant bits), up in {+-1, +-3, +-5, +-7}
    cycling over channels, w = 2^-(m % 4)."""
    gate = np.full((rows, inter), 32.0)
    uc = np.array([1.0, -3.0, 5.0, -7.0])
    up = np.tile(uc, (rows, inter // 4))
    w = (2.0 ** -(np.arange(rows) % 4)).astype(np.float32)
    return f64_to_bf16_bits(gate), f64_to_bf16_bits(up), w


@pytest.mark.parametrize("limit", [0.0, float("nan"), 1e9])
def test_swiglu_rows_closed_form_without_clamp(limit):
    rows, inter = 6, 64
    g, u, w = _closed_case(rows, inter, limit)
    h, q8 = oracle.swiglu_q8_1_rows(g, u, w, limit)
    want = 32.0 * bf16_to_f64(u) * w[:, None]
    assert np.array_equal(h, f64_to_bf16_bits(want))
    # every block holds u = 1, -3, 5, -7 (times 32 w): amax 7*32w, q = round(u*127/7)
    for m in range(rows):
        for b in range(inter // 32):
            q = q8[m, b, 4:].view(np.int8)
            assert list(q[:4]) == [18, -54, 91, -127]
            d = np.float32(np.float32(7 * 32 * w[m]) / np.float32(127))
            assert q8[m, b, :2].view(np.uint16)[0] == oracle.fp16_rne(float(d))


def test_swiglu_rows_limit_clamps_gate_above_and_up_both_ways():
    rows, inter = 4, 32
    g = f64_to_bf16_bits(np.full((rows, inter), 100.0))
    u = f64_to_bf16_bits(np.tile(np.array([100.0, -100.0, 3.0, -3.0]), (rows, 8)))
    h, _ = oracle.swiglu_q8_1_rows(g, u, None, 32.0)
    # gate -> 32 (silu(32) ~ 32), up -> +-32 or +-3 (inside the limit)
    want = np.tile(np.array([1024.0, -1024.0, 96.0, -96.0]), (rows, 8))
    assert np.array_equal(h, f64_to_bf16_bits(want))
    # a gate below -limit is not clamped (silu is bounded below): silu(-40) * u
    g2 = f64_to_bf16_bits(np.full((rows, inter), -40.0))
    h2, _ = oracle.swiglu_q8_1_rows(g2, u, None, 32.0)
    assert np.all(np.abs(bf16_to_f64(h2)) < 1e-14) and np.any(h2 != 0)


def test_swiglu_rows_blocks_are_the_rows_32_value_blocks():
    w = W.small_workload(37, 96, seed=7)
    x, _ = W.make_inputs(w)
    g, u = x[:, :96], x[:, 96:]
    wt = np.linspace(0.1, 1.0, 37).astype(np.float32)
    h, q8 = oracle.swiglu_q8_1_rows(g, u, wt, 0.0)
    for m in range(37):
        for b in range(3):
            assert np.array_equal(q8[m, b], oracle.q8_1_block(h[m, 32 * b:32 * (b + 1)]))
    # and each h is the bf16 of silu(g) * u * w from an independent fp64 route
    from scipy.special import expit
    gf, uf = bf16_to_f64(g), bf16_to_f64(u)
    ref = bf16_round_bits64(np.where(np.abs(gf * expit(gf) * uf * wt[:, None]) < 2.0 ** -126, 0.0,
                                     gf * expit(gf) * uf * wt[:, None]))
    assert (h != ref).mean() < 1e-3


def test_swiglu_rows_zero_block_and_rejections():
    g = np.zeros((2, 64), np.uint16)
    u = f64_to_bf16_bits(np.ones((2, 64)))
    h, q8 = oracle.swiglu_q8_1_rows(g, u)           # silu(0) = 0: h = 0, all-zero blocks
    assert not h.any() and not q8.any()
    with pytest.raises(ValueError):
        oracle.swiglu_q8_1_rows(np.zeros((2, 48), np.uint16), np.zeros((2, 48), np.uint16))

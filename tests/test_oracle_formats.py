"""Pins of the oracle's output formats (FP8 E4M3 codes, E8M0 scales, the
[Mg, K] layout of y_s_t) to things other than the oracle (no GPU).

The page only says the outputs feed quantized GEMMs; the formats follow the
public OCP definitions: 8-bit floating point E4M3 (bias 7, no infinities,
largest finite 448) and the Microscaling E8M0 scale byte (value 2^(e-127)).
Each test ties an oracle function to exact rational arithmetic
(``tests/exact.py``), to torch's float8_e4m3fn conversion, to the pinned INT8
whole op, or to a closed-form case.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests.exact import (bf16_round_bits64, bf16_to_f64, bf16_value, e4m3_nearest, e4m3_table, f32_round,
                         f64_to_bf16_bits, pow2_ceil_exponent, round_half_even)

FORMATS = [(c, s) for c in (0, 1) for s in (0, 1)]   # (codes, scales)
QMAX = {0: 127, 1: 448}


# ----------------------------------------------------------------------------
# E4M3 encode / decode
# ----------------------------------------------------------------------------

def _e4m3_tricky(rng, n):
    """Values at, near and between E4M3 points, subnormals included."""
    tab = [v for v, _ in e4m3_table()]
    vals = []
    for _ in range(n):
        i = int(rng.integers(0, len(tab) - 1))
        lo, hi = tab[i], tab[i + 1]
        mid = (lo + hi) / 2
        eps = (hi - lo) * Fraction(1, 2 ** int(rng.integers(4, 20)))
        for v in (lo, hi, mid, mid + eps, mid - eps, lo + (hi - lo) / 3):
            vals.append(float(v) * (-1 if rng.random() < 0.5 else 1))
    return vals


def test_e4m3_rne_against_torch_float8_conversion():
    # inside the finite range torch's float32 -> float8_e4m3fn conversion
    # rounds to nearest even; float32 inputs avoid a double rounding in torch
    rng = np.random.default_rng(1)
    vals = np.array(_e4m3_tricky(rng, 400) + list(rng.normal(0, 50, 2000)) +
                    list(rng.uniform(-448, 448, 2000)), np.float32)
    vals = vals[np.abs(vals) <= 448]
    want = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_rne(float(v)) for v in vals], np.uint8)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, [(float(vals[i]), hex(got[i]), hex(want[i])) for i in bad[:5]]


def test_e4m3_rne_bruteforce_exact_rationals():
    rng = np.random.default_rng(2)
    vals = _e4m3_tricky(rng, 500) + [460.0, 464.0, 470.0, 480.0, 1e6, -1e30, 2.0 ** -10,
                                     2.0 ** -10 * 3, 2.0 ** -11, 0.0, -0.0, 2.0 ** -40]
    for v in vals:
        want = e4m3_nearest(Fraction(v))
        if v == 0 and np.signbit(v):
            want = 0x80
        assert oracle.e4m3_rne(v) == want, (v, hex(oracle.e4m3_rne(v)), hex(want))


def test_e4m3_value_roundtrip_all_codes():
    for code in range(256):
        v = oracle.e4m3_value(code)
        if code & 0x7F == 0x7F:
            assert np.isnan(v)
            continue
        want = dict((c, val) for val, c in e4m3_table())[code & 0x7F]
        assert Fraction(v) == (-want if code & 0x80 else want)
        assert oracle.e4m3_rne(v) == code or (code == 0x80 and v == 0)


# ----------------------------------------------------------------------------
# E8M0 scale: smallest power of two >= s
# ----------------------------------------------------------------------------

def test_e8m0_ceil_bruteforce():
    rng = np.random.default_rng(3)
    exps = rng.integers(-149, 127, 3000)
    mant = rng.uniform(1, 2, 3000)
    vals = np.ldexp(mant, exps).astype(np.float32)
    vals = np.concatenate([vals, np.ldexp(np.ones(40), np.arange(-140, 120, 6.5).astype(int)).astype(np.float32)])
    vals = vals[vals > 0]
    for s in vals:
        k = min(127, max(-127, pow2_ceil_exponent(Fraction(float(s)))))
        assert oracle.e8m0_ceil(float(s)) == k + 127, float(s)
        assert oracle.e8m0_value(k + 127) == 2.0 ** k


# ----------------------------------------------------------------------------
# one group in each format, against an exact restatement of its definition
# ----------------------------------------------------------------------------

def _expected_group(bits, codes, scales):
    """(code bytes, scale) from the definitions, with exact rationals."""
    vals = [bf16_value(int(b)) for b in bits]
    amax = max(abs(v) for v in vals)
    if amax == 0:
        s, k = Fraction(1), 0
    else:
        s = f32_round(amax / QMAX[codes])
        if scales:
            k = min(127, max(-127, pow2_ceil_exponent(s)))
            s = Fraction(2) ** k
    out = []
    for b, v in zip(bits, vals):
        t = f32_round(v / s)
        if codes:   # a quotient that is zero keeps v's sign (rationals have no -0)
            out.append((0x80 if int(b) & 0x8000 else 0) if t == 0 else e4m3_nearest(t))
        else:
            out.append(round_half_even(t) & 0xFF)
    return out, ((k + 127) if scales else float(s))


def _groups(rng):
    gs = []
    for sc in (1.0, 1e-3, 3e4, 1e-30, 2.0 ** -120, 1e30):
        v = rng.normal(0, sc, 128)
        gs.append(v)
    gs.append(np.zeros(128))
    gs.append(np.full(128, -0.75))
    out = [f64_to_bf16_bits(_bf16_exact(v)) for v in gs]
    signed_zero = np.zeros(128, np.uint16)
    signed_zero[::3] = 0x8000             # an all-zero group with -0.0 elements
    out.append(signed_zero)
    mixed = out[0].copy()
    mixed[7] = 0x8000                     # a -0.0 element in a non-zero group
    out.append(mixed)
    return out


def _bf16_exact(v):
    """Nearest bf16 values (as doubles) of v, values below the normal range
    set to zero."""
    v = np.where(np.abs(v) < 2.0 ** -126, 0.0, v)
    return bf16_to_f64(bf16_round_bits64(v))


@pytest.mark.parametrize("codes,scales", FORMATS)
def test_quant_group_fmt_bruteforce(codes, scales):
    rng = np.random.default_rng(10 + 2 * codes + scales)
    groups = _groups(rng)
    g = np.zeros(128, np.uint16)
    g[3] = 0x0001                          # bf16 subnormal amax
    g[9] = 0x8001
    groups.append(g)
    for bits in groups:
        q, s = oracle.quant_group_fmt(bits, codes, scales)
        want_q, want_s = _expected_group(bits, codes, scales)
        assert s == want_s, (codes, scales, s, want_s)
        assert list(q) == want_q, (codes, scales)


@pytest.mark.parametrize("codes,scales", FORMATS)
def test_quant_group_fmt_invariants(codes, scales):
    rng = np.random.default_rng(20 + 2 * codes + scales)
    for sc in (1.0, 0.02, 700.0, 1e-20):
        bits = f64_to_bf16_bits(_bf16_exact(rng.normal(0, sc, 128)))
        q, s = oracle.quant_group_fmt(bits, codes, scales)
        v = bf16_to_f64(bits)
        amax = np.abs(v).max()
        sv = oracle.e8m0_value(s) if scales else s
        qv = np.array([oracle.e4m3_value(c) for c in q]) if codes else q.view(np.int8).astype(np.float64)
        assert np.all(np.abs(qv) <= QMAX[codes])
        assert np.all((np.sign(qv) == np.sign(v)) | (qv == 0))
        top = np.abs(qv[np.argmax(np.abs(v))])
        if scales:      # scale / 2 < amax / Qmax <= scale: the amax code lies in the top binade
            s32 = np.float32(np.float32(amax) / np.float32(QMAX[codes]))
            assert sv / 2 < s32 <= sv
            assert QMAX[codes] / 2 - 1 <= top <= QMAX[codes]
        else:
            assert top == QMAX[codes]


def test_quant_group_fmt_default_equals_pinned_int8():
    rng = np.random.default_rng(30)
    for sc in (1.0, 1e-3, 1e5):
        bits = f64_to_bf16_bits(_bf16_exact(rng.normal(0, sc, 128)))
        q, s = oracle.quant_group_fmt(bits, 0, 0)
        q0, s0 = oracle.quant_group(bits)
        assert s == s0 and np.array_equal(q.view(np.int8), q0)


# ----------------------------------------------------------------------------
# the whole op in each format
# ----------------------------------------------------------------------------

def test_whole_op_fmt_default_equals_pinned_op():
    w = W.small_workload(200, 384, seed=4)
    x, gy = W.make_inputs(w)
    a = oracle.silu_dot_fwd_bwd_quant_fuse(x, gy)
    b = oracle.silu_dot_fwd_bwd_quant_fuse_fmt(x, gy, 128, 0, 0, 0)
    assert np.array_equal(a[0], b[0].view(np.int8)) and np.array_equal(a[2], b[2].view(np.int8))
    assert np.array_equal(a[1], b[1]) and np.array_equal(a[3], b[3])


@pytest.mark.parametrize("codes,scales", FORMATS)
def test_whole_op_fmt_ys_layouts_transpose(codes, scales):
    w = W.small_workload(300, 256, seed=5)
    x, gy = W.make_inputs(w)
    a = oracle.silu_dot_fwd_bwd_quant_fuse_fmt(x, gy, 128, codes, scales, 0)
    b = oracle.silu_dot_fwd_bwd_quant_fuse_fmt(x, gy, 128, codes, scales, 1)
    assert a[3].shape == (256, 3) and b[3].shape == (3, 256)
    assert np.array_equal(a[3].T, b[3])
    for u, v in zip(a[:3], b[:3]):
        assert np.array_equal(u, v)


@pytest.mark.parametrize("G", [256, 128, 64, 32])
@pytest.mark.parametrize("codes,scales", FORMATS)
def test_whole_op_fmt_groups_relate_to_stage1(codes, scales, G):
    # every group of all four outputs equals the exact restatement of the
    # format applied to that group's bf16 intermediates (M = 40: a tail group)
    M, K = 40, 256
    w = W.small_workload(M, K, seed=6)
    x, gy = W.make_inputs(w)
    giq, gis, yqt, yst = oracle.silu_dot_fwd_bwd_quant_fuse_fmt(x, gy, G, codes, scales, 0)
    assert gis.shape == (M, 2 * K // G) and yst.shape == (K, (M + G - 1) // G)
    y, dg, du = oracle.swiglu_bwd_bf16(x, gy)
    V = np.concatenate([dg, du], axis=1)
    for m in range(0, M, 3):
        for j in range(2 * K // G):
            want_q, want_s = _expected_group(V[m, j * G:(j + 1) * G], codes, scales)
            assert list(giq[m, j * G:(j + 1) * G]) == want_q
            assert gis[m, j] == want_s
    for k in range(0, K, 5):
        for i in range((M + G - 1) // G):
            want_q, want_s = _expected_group(y[i * G:(i + 1) * G, k], codes, scales)
            assert list(yqt[k, i * G:(i + 1) * G]) == want_q
            assert yst[k, i] == want_s


def test_whole_op_e4m3_gate32_closed_form():
    """gate = 32, up = a(m)*w(k), grad_y = 2^-e(m) (as in the INT8 pins):
    d_gate = 2^-e*a*w with row amax 7*a*2^-e, so scale = a*2^-e/64 exactly and
    the codes are w*64 = 64, 192, 320, 448 (E4M3 0x68, 0x74, 0x7A, 0x7E);
    d_up = 32*2^-e is constant along the row: every code is 448 (0x7E)."""
    A_ROW, W_COL = [1, 2, 3, 5, 6, 7, 8], [1, 3, 5, 7]
    M, K = 70, 256
    a = np.array([A_ROW[m % 7] for m in range(M)], np.float64)
    wv = np.array([W_COL[k % 4] for k in range(K)], np.float64)
    e = np.array([m % 5 for m in range(M)], np.float64)
    x = np.concatenate([np.full((M, K), 32.0), np.outer(a, wv)], axis=1)
    gy = np.repeat((2.0 ** -e)[:, None], K, axis=1)
    giq, gis, yqt, yst = oracle.silu_dot_fwd_bwd_quant_fuse_fmt(
        f64_to_bf16_bits(x), f64_to_bf16_bits(gy), 128, 1, 0, 0)
    code_of_w = {1: 0x68, 3: 0x74, 5: 0x7A, 7: 0x7E}
    for m in range(M):
        assert np.all(gis[m, :2] == np.float32(a[m] * 2.0 ** -e[m] / 64))
        assert np.all(giq[m, :K] == np.array([code_of_w[int(t)] for t in wv], np.uint8))
        assert np.all(giq[m, K:] == 0x7E)
        assert np.all(gis[m, 2:] == np.float32(np.float32(32 * 2.0 ** -e[m]) / np.float32(448)))
    # y = 32*a*w; the one token group holds a = 8, so amax = 256*w and the
    # codes are about 56*a: exact E4M3 points for a = 1, 2, 7, 8 (56, 112, 392, 448)
    want = {1: 0x66, 2: 0x6E, 7: 0x7C, 8: 0x7E}
    for t in range(M):
        if int(a[t]) in want:
            assert np.all(yqt[:, t] == want[int(a[t])]), t


# ----------------------------------------------------------------------------
# G not dividing K: each half of [d_gate | d_up] ends in a shorter group
# ----------------------------------------------------------------------------

def _pad_channels(a, K, Kp):
    """[M, K] (or the two halves of [M, 2K]) widened to Kp channels with zeros."""
    if a.shape[1] == K:
        return np.concatenate([a, np.zeros((a.shape[0], Kp - K), a.dtype)], axis=1)
    return np.concatenate([_pad_channels(a[:, :K], K, Kp), _pad_channels(a[:, K:], K, Kp)], axis=1)


@pytest.mark.parametrize("K,G", [(200, 128), (144, 128), (208, 64), (80, 32), (16, 128), (1040, 128), (384, 256)])
@pytest.mark.parametrize("fmt", [(0, 0, 0), (1, 1, 1), (0, 1, 1)])
def test_short_last_group_equals_the_zero_padded_op(K, G, fmt):
    """Zero channels change no amax and quantize to zero, so the op on K
    channels equals the op on K padded with zeros to a multiple of G (where
    every group is whole), restricted to the K real channels of each half."""
    M = 131
    Kp = (K + G - 1) // G * G
    x, gy = W.make_inputs(W.small_workload(M, K, seed=K + G, zero_group_every=0))
    got = oracle.silu_dot_fwd_bwd_quant_fuse_fmt(x, gy, G, *fmt)
    pad = oracle.silu_dot_fwd_bwd_quant_fuse_fmt(_pad_channels(x, K, Kp), _pad_channels(gy, K, Kp), G, *fmt)
    assert np.array_equal(got[0], np.concatenate([pad[0][:, :K], pad[0][:, Kp:Kp + K]], axis=1))
    assert np.array_equal(got[1], pad[1])               # ceil(K/G) groups per half either way
    assert np.array_equal(got[2], pad[2][:K])
    ys = pad[3][:, :K] if fmt[2] else pad[3][:K]
    assert np.array_equal(got[3], ys)
    assert got[1].shape == (M, 2 * ((K + G - 1) // G))

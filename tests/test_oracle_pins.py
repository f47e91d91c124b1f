"""Pins of the CPU oracle to things other than itself (no GPU).

Each test ties one oracle function to an independent fact: exact rational
arithmetic, a library routine that computes the same mathematical object by
another route (scipy's expit, torch float64 autograd), finite differences, or
a closed-form case derived by hand from the op's definition on
"kernelgen-challenge-9-task3-silu-quant" (outputs section; constraints list).
A plausible slip in the oracle -- a dropped term, a wrong sign, swapped gate
and up, swapped d_gate and d_up, a transposed y, a wrong group index, round
half away from zero, 128 in place of 127 -- fails at least one of them.
"""
from __future__ import annotations

import math
from fractions import Fraction

import numpy as np
import pytest
import torch
from scipy.special import expit

import oracle
import workloads as W
from tests.exact import (bf16_round_bits64, bf16_round_bruteforce, bf16_to_f64,
                         bf16_value, f64_to_bf16_bits)


# ----------------------------------------------------------------------------
# bf16 round-to-nearest-even from fp64 (constraints list, third item: the bf16
# round-trip before quantization)
# ----------------------------------------------------------------------------

def _tricky_doubles(rng, n):
    vals = []
    for _ in range(n):
        b = int(rng.integers(0x0080, 0x7F7F))  # a normal bf16 pattern
        lo = bf16_value(b)
        hi = bf16_value(b + 1)
        mid = (lo + hi) / 2
        eps = (hi - lo) * Fraction(1, 2 ** int(rng.integers(20, 44)))
        for v in (mid, mid + eps, mid - eps, lo, hi, lo + (hi - lo) / 3):
            vals.append(float(v))
    return vals


def test_bf16_rne_bruteforce_exact_rationals():
    rng = np.random.default_rng(11)
    vals = _tricky_doubles(rng, 400)
    vals += [0.0, -0.0, 1.0, -1.0, 3.0e38, 3.3895313892515355e38, 3.4e38, 1e39,
             -1e39, 1.1754943508222875e-38, 2.0 ** -126 * 1.00390625]
    for v in vals:
        for s in (1.0, -1.0):
            x = s * v
            assert oracle.bf16_rne(x) == bf16_round_bruteforce(x), x


def test_bf16_rne_against_torch_float32_conversion():
    # float32 -> bfloat16 in torch is a single nearest-even rounding, so for
    # inputs that are float32 values it is an independent reference.
    rng = np.random.default_rng(12)
    bits = rng.integers(0, 2 ** 32, size=20000, dtype=np.uint64).astype(np.uint32)
    bits = bits[((bits >> 23) & 0xFF) != 0xFF]           # finite only
    ties = (rng.integers(0, 0x7F7F, size=2000).astype(np.uint32) << 16) | 0x8000
    bits = np.concatenate([bits, ties, ties | 0x80000000])
    f = bits.view(np.float32)
    ref = torch.from_numpy(f.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.bf16_rne(float(v)) for v in f], dtype=np.uint16)
    assert np.array_equal(got, ref)


def test_bits64_helper_matches_bruteforce():
    rng = np.random.default_rng(13)
    v = np.array(_tricky_doubles(rng, 300))
    v = np.concatenate([v, -v, [0.0, -0.0]])
    got = bf16_round_bits64(v)
    ref = np.array([bf16_round_bruteforce(float(x)) for x in v], dtype=np.uint16)
    assert np.array_equal(got, ref)


# ----------------------------------------------------------------------------
# sigmoid, silu, silu'
# ----------------------------------------------------------------------------

G_GRID = np.concatenate([np.linspace(-40, 40, 801), [-745.0, -300.0, 300.0, 745.0]])


def test_sigmoid_matches_library_expit():
    for g in G_GRID:
        ref = float(expit(g))
        got = oracle.sigmoid(g)
        assert got == pytest.approx(ref, rel=4e-16, abs=1e-300), g


def test_sigmoid_silu_closed_forms():
    assert oracle.sigmoid(0.0) == 0.5
    assert oracle.silu(0.0) == 0.0
    assert oracle.silu_grad(0.0) == 0.5
    for g in np.linspace(-30, 30, 121):
        assert oracle.sigmoid(g) + oracle.sigmoid(-g) == pytest.approx(1.0, abs=4.5e-16)
        assert oracle.silu(g) - oracle.silu(-g) == pytest.approx(g, abs=4e-15 * max(1, abs(g)))
    # saturation: no NaN at the far ends
    assert oracle.sigmoid(-800.0) == 0.0 and oracle.sigmoid(800.0) == 1.0
    assert oracle.silu_grad(800.0) == 1.0 and oracle.silu_grad(-800.0) == 0.0


def test_silu_grad_matches_finite_difference():
    # Richardson-extrapolated central differences of the oracle's own silu.
    for g in np.linspace(-20, 20, 161):
        h = 1e-3
        d1 = (oracle.silu(g + h) - oracle.silu(g - h)) / (2 * h)
        d2 = (oracle.silu(g + h / 2) - oracle.silu(g - h / 2)) / h
        fd = (4 * d2 - d1) / 3
        assert oracle.silu_grad(g) == pytest.approx(fd, rel=1e-8, abs=1e-11), g


# ----------------------------------------------------------------------------
# one element of forward recompute + backward, fp64
# ----------------------------------------------------------------------------

def _torch_autograd(g, u, dy):
    gt = torch.tensor(g, dtype=torch.float64, requires_grad=True)
    ut = torch.tensor(u, dtype=torch.float64, requires_grad=True)
    y = torch.nn.functional.silu(gt) * ut
    (y * torch.tensor(dy, dtype=torch.float64)).sum().backward()
    return y.detach().numpy(), gt.grad.numpy(), ut.grad.numpy()


def test_swiglu_bwd_fp64_matches_torch_autograd():
    rng = np.random.default_rng(21)
    n = 3000
    g = rng.normal(0, 3, n)
    g[:50] *= 40  # saturation region
    u = rng.normal(0, 1, n)
    dy = rng.normal(0, 0.02, n)
    y_ref, dg_ref, du_ref = _torch_autograd(g, u, dy)
    for i in range(n):
        y, dg, du = oracle.swiglu_bwd_fp64(g[i], u[i], dy[i])
        scale = 1e-300
        assert y == pytest.approx(y_ref[i], rel=1e-13, abs=scale)
        assert dg == pytest.approx(dg_ref[i], rel=1e-12, abs=1e-13 * abs(dy[i] * u[i]) + scale)
        assert du == pytest.approx(du_ref[i], rel=1e-13, abs=scale)


def test_swiglu_bwd_fp64_finite_differences():
    # d_gate = dy * dy/dg and d_up = dy * dy/du of y(g, u) = silu(g) * u.
    rng = np.random.default_rng(22)
    for _ in range(300):
        g, u, dy = rng.normal(0, 3), rng.normal(0, 2), rng.normal(0, 1)
        y, dg, du = oracle.swiglu_bwd_fp64(g, u, dy)
        h = 1e-4
        yg = lambda gg: oracle.swiglu_bwd_fp64(gg, u, dy)[0]
        yu = lambda uu: oracle.swiglu_bwd_fp64(g, uu, dy)[0]
        fd_g = (8 * (yg(g + h) - yg(g - h)) - (yg(g + 2 * h) - yg(g - 2 * h))) / (12 * h)
        fd_u = (yu(u + h) - yu(u - h)) / (2 * h)
        assert dg == pytest.approx(dy * fd_g, rel=1e-7, abs=1e-9)
        assert du == pytest.approx(dy * fd_u, rel=1e-9, abs=1e-12)


def test_stage1_bf16_equals_rounded_torch_autograd():
    # The whole first stage on random bf16 inputs: each of y, d_gate, d_up is
    # the nearest bf16 of the exact-ish fp64 gradient computed by torch.
    w = W.small_workload(64, 256, seed=5)
    x, gy = W.make_inputs(w)
    y, dg, du = oracle.swiglu_bwd_bf16(x, gy)
    K = w.K
    g = bf16_to_f64(x[:, :K]).ravel()
    u = bf16_to_f64(x[:, K:]).ravel()
    d = bf16_to_f64(gy).ravel()
    y_ref, dg_ref, du_ref = _torch_autograd(g, u, d)
    for got, ref in ((y, y_ref), (dg, dg_ref), (du, du_ref)):
        assert np.array_equal(got.ravel(), bf16_round_bits64(ref))


# ----------------------------------------------------------------------------
# group quantization
# ----------------------------------------------------------------------------

def _group(vals):
    return f64_to_bf16_bits(np.asarray(vals, dtype=np.float64))


def _random_group(rng, n=128, scale=1.0):
    f = (rng.normal(0, scale, n)).astype(np.float32)
    return W.f32_to_bf16_bits(f)


def test_quant_scale_is_amax_over_127_rounded_once():
    rng = np.random.default_rng(31)
    for _ in range(400):
        v = _random_group(rng, scale=float(10 ** rng.uniform(-6, 3)))
        q, s = oracle.quant_group(v)
        amax = max(abs(bf16_value(int(b))) for b in v)
        exact = amax / 127
        s_f = Fraction(float(s))
        up = Fraction(float(np.nextafter(np.float32(s), np.float32(np.inf))))
        dn = Fraction(float(np.nextafter(np.float32(s), np.float32(-np.inf))))
        assert abs(s_f - exact) <= abs(up - exact) and abs(s_f - exact) <= abs(dn - exact)


def test_quant_nearest_integer_and_bounds():
    rng = np.random.default_rng(32)
    for _ in range(300):
        v = _random_group(rng, n=int(rng.integers(1, 200)), scale=float(10 ** rng.uniform(-4, 2)))
        q, s = oracle.quant_group(v)
        vals = [bf16_value(int(b)) for b in v]
        amax = max(abs(t) for t in vals)
        sf = Fraction(float(s))
        assert s > 0
        assert np.all(np.abs(q.astype(np.int32)) <= 127)
        for t, qi in zip(vals, q.tolist()):
            err = abs(t / sf - qi)
            # fp32 quotient: at most half a step plus the quotient's rounding
            assert err <= Fraction(1, 2) + Fraction(1, 2 ** 16)
            if qi != 0:
                assert (qi > 0) == (t > 0)
        # the amax element maps to +-127
        k = int(np.argmax([abs(t) for t in vals]))
        assert abs(int(q[k])) == 127
        assert amax > 0


def test_quant_ties_to_even_and_symmetry():
    # amax = 127 -> scale = 1 exactly, so v/scale = v and exact halves are ties.
    vals = [127.0, 2.5, -2.5, 3.5, -3.5, 0.5, -0.5, 1.5, 126.5, -125.5, 0.0, -0.0]
    q, s = oracle.quant_group(_group(vals))
    assert s == 1.0
    assert q.tolist() == [127, 2, -2, 4, -4, 0, 0, 2, 126, -126, 0, 0]
    rng = np.random.default_rng(33)
    for _ in range(100):
        v = _random_group(rng)
        q1, s1 = oracle.quant_group(v)
        q2, s2 = oracle.quant_group(v ^ np.uint16(0x8000))
        assert s1 == s2 and np.array_equal(q1, -q2)


def test_quant_monotone():
    rng = np.random.default_rng(34)
    v = _random_group(rng, n=128)
    q, s = oracle.quant_group(v)
    order = np.argsort(bf16_to_f64(v), kind="stable")
    assert np.all(np.diff(q[order].astype(np.int32)) >= 0)


def test_quant_zero_and_constant_groups():
    q, s = oracle.quant_group(np.zeros(128, np.uint16))
    assert s == 1.0 and not q.any()
    q, s = oracle.quant_group(np.full(128, 0x8000, np.uint16))  # all -0.0
    assert s == 1.0 and not q.any()
    for c in (3.0, -0.0078125, 1.5 * 2.0 ** -17, 2.0 ** 100):
        b = f64_to_bf16_bits([c])[0]
        q, s = oracle.quant_group(np.full(128, b, np.uint16))
        assert s == np.float32(np.float32(abs(bf16_value(int(b)))) / np.float32(127))
        assert np.all(q == (127 if c > 0 else -127))


# ----------------------------------------------------------------------------
# the whole op: closed forms derived by hand from the definition
# ----------------------------------------------------------------------------

A_ROW = [1, 2, 3, 5, 6, 7, 8]  # a(m) = A_ROW[m % 7]
W_COL = [1, 3, 5, 7]           # w(k) = W_COL[k % 4]


def _gate32_case(M, K):
    """gate = 32, up[m,k] = a(m)*w(k), grad_y[m,k] = 2^-(m % 5).

    sigma(32) = 1 - 1.3e-14, so in fp64 silu(32) and silu'(32) are within
    1e-12 of 32 and 1; every product below has at most 8 significant bits,
    so the bf16 values are exact:
        y = 32*a*w,  d_gate = 2^-e * a * w,  d_up = 32 * 2^-e   (e = m % 5).
    """
    a = np.array([A_ROW[m % 7] for m in range(M)], np.float64)
    w = np.array([W_COL[k % 4] for k in range(K)], np.float64)
    e = np.array([m % 5 for m in range(M)], np.float64)
    up = np.outer(a, w)
    x = np.concatenate([np.full((M, K), 32.0), up], axis=1)
    gy = np.repeat((2.0 ** -e)[:, None], K, axis=1)
    return f64_to_bf16_bits(x), f64_to_bf16_bits(gy), a, w, e


@pytest.mark.parametrize("M,K,G", [(200, 256, 128), (7, 128, 128), (129, 384, 128),
                                   (200, 256, 64), (129, 128, 32), (300, 512, 256), (256, 256, 256)])
def test_whole_op_gate32_closed_form(M, K, G):
    x, gy, a, w, e = _gate32_case(M, K)
    giq, gis, yqt, yst = oracle.silu_dot_fwd_bwd_quant_fuse(x, gy, G)
    Kg, Mg = K // G, (M + G - 1) // G
    f32 = np.float32
    # d_gate groups: amax over a G-channel group (G >= 32 holds the whole cycle
    # w = 1, 3, 5, 7) = 7 * a(m) * 2^-e -> q = round(w * 127 / 7) = 18, 54, 91, 127
    # (no value near a half).
    q_dg = {1: 18, 3: 54, 5: 91, 7: 127}
    for m in range(M):
        s_dg = f32(f32(7 * a[m] * 2.0 ** -e[m]) / f32(127))
        s_du = f32(f32(32 * 2.0 ** -e[m]) / f32(127))
        assert np.all(gis[m, :Kg] == s_dg), m
        assert np.all(gis[m, Kg:] == s_du), m
        assert np.all(giq[m, :K] == np.array([q_dg[int(t)] for t in w], np.int8))
        assert np.all(giq[m, K:] == 127)       # d_up is constant along the row
    # y column groups (over tokens): amax = 32 * 8 * w(k) when a = 8 is among the
    # group's tokens; q = round(a * 127 / 8) = 16, 32, 48, 79, 95, 111, 127.
    q_y = {1: 16, 2: 32, 3: 48, 5: 79, 6: 95, 7: 111, 8: 127}
    for i in range(Mg):
        t0, t1 = i * G, min(M, i * G + G)
        amax_a = max(a[t0:t1])
        for k in range(K):
            assert yst[k, i] == f32(f32(32 * amax_a * w[k]) / f32(127)), (k, i)
        if amax_a == 8:
            want = np.array([q_y[int(t)] for t in a[t0:t1]], np.int8)
            assert np.all(yqt[:, t0:t1] == want[None, :])
    assert yqt.shape == (K, M) and yst.shape == (K, Mg) and gis.shape == (M, 2 * Kg)


def test_whole_op_gate_zero_closed_form():
    # gate = 0: silu(0) = 0 and silu'(0) = 1/2, so y = 0, d_up = 0 and
    # d_gate = grad_y * up / 2.  With grad_y = 2 and integer up, d_gate = up.
    M, K = 130, 256
    rng = np.random.default_rng(41)
    up = rng.integers(-127, 128, size=(M, K)).astype(np.float64)
    up[:, ::128] = 127.0            # every group holds 127, so scale = 1 exactly
    x = f64_to_bf16_bits(np.concatenate([np.zeros((M, K)), up], axis=1))
    gy = f64_to_bf16_bits(np.full((M, K), 2.0))
    giq, gis, yqt, yst = oracle.silu_dot_fwd_bwd_quant_fuse(x, gy)
    assert np.all(gis[:, :2] == 1.0) and np.all(gis[:, 2:] == 1.0)
    assert np.array_equal(giq[:, :K], up.astype(np.int8))
    assert not giq[:, K:].any()
    assert np.all(yst == 1.0) and not yqt.any()


def test_whole_op_up_zero_closed_form():
    # up = 0: y = 0 and d_gate = 0, d_up = grad_y * silu(gate) (nonzero).
    M, K = 64, 128
    rng = np.random.default_rng(42)
    g = rng.normal(0, 1, (M, K))
    x = np.concatenate([W.f32_to_bf16_bits(g.astype(np.float32)), np.zeros((M, K), np.uint16)], axis=1)
    gy = W.f32_to_bf16_bits(np.full((M, K), 0.5, np.float32))
    giq, gis, yqt, yst = oracle.silu_dot_fwd_bwd_quant_fuse(x, gy)
    assert np.all(gis[:, 0] == 1.0) and not giq[:, :K].any()
    assert np.all(yst == 1.0) and not yqt.any()
    du_ref = 0.5 * bf16_to_f64(x[:, :K]) * expit(bf16_to_f64(x[:, :K]))
    for m in range(M):
        amax = np.abs(bf16_to_f64(bf16_round_bits64(du_ref[m]))).max()
        assert gis[m, 1] == np.float32(np.float32(amax) / np.float32(127))
        assert np.abs(giq[m, K:]).max() == 127


def test_tail_single_token_group():
    # M = 129: token group 1 holds one token, so each of its columns maps to
    # +-127 (or 0 with scale 1 when y is zero there).
    w = W.small_workload(129, 128, seed=9)
    x, gy = W.make_inputs(w)
    _, _, yqt, yst = oracle.silu_dot_fwd_bwd_quant_fuse(x, gy)
    y, _, _ = oracle.swiglu_bwd_bf16(x, gy)
    last = bf16_to_f64(y[128])
    for k in range(128):
        if last[k] == 0:
            assert yst[k, 1] == 1.0 and yqt[k, 128] == 0
        else:
            assert abs(int(yqt[k, 128])) == 127
            assert yst[k, 1] == np.float32(np.float32(abs(last[k])) / np.float32(127))


def test_whole_op_groups_relate_to_stage1():
    # On seeded random inputs: every group's scale is its own amax/127 and every
    # q dequantizes to within half a step of its own bf16 value -- checks the
    # indexing of all four outputs against the bf16 intermediates.
    w = W.small_workload(200, 384, seed=3)
    x, gy = W.make_inputs(w)
    giq, gis, yqt, yst = oracle.silu_dot_fwd_bwd_quant_fuse(x, gy)
    y, dg, du = (bf16_to_f64(a) for a in oracle.swiglu_bwd_bf16(x, gy))
    G, M, K = 128, w.M, w.K
    V = np.concatenate([dg, du], axis=1)
    for j in range(2 * K // G):
        blk = V[:, j * G:(j + 1) * G]
        amax = np.abs(blk).max(axis=1)
        assert np.array_equal(gis[:, j], (amax.astype(np.float32) / np.float32(127)))
        deq = giq[:, j * G:(j + 1) * G].astype(np.float64) * gis[:, j:j + 1]
        assert np.all(np.abs(deq - blk) <= gis[:, j:j + 1] * (0.5 + 2 ** -15))
    for i in range((M + G - 1) // G):
        blk = y[i * G:(i + 1) * G, :]          # [tokens, K]
        amax = np.abs(blk).max(axis=0)
        s = np.where(amax == 0, np.float32(1), amax.astype(np.float32) / np.float32(127))
        assert np.array_equal(yst[:, i], s)
        deq = yqt[:, i * G:(i + 1) * G].astype(np.float64) * yst[:, i:i + 1]
        assert np.all(np.abs(deq - blk.T) <= yst[:, i:i + 1] * (0.5 + 2 ** -15))


def test_page_format_is_the_format_op_at_int8_fp32():
    """The page-format entry is the format op with INT8 codes, fp32 scales and
    y_s_t [K, Mg] (one quantizer), also where G does not divide K (a shorter
    last channel group in each half); a group size below 1 is rejected."""
    for M, K, G, seed in [(40, 256, 128, 1), (37, 100, 128, 2), (20, 100, 50, 3), (9, 208, 64, 4)]:
        x, gy = W.make_inputs(W.small_workload(M, K, seed=seed))
        a = oracle.silu_dot_fwd_bwd_quant_fuse(x, gy, group_size=G)
        b = oracle.silu_dot_fwd_bwd_quant_fuse_fmt(x, gy, G, 0, 0, 0)
        Kg = (K + G - 1) // G
        assert a[1].shape == (M, 2 * Kg) and a[3].shape == (K, (M + G - 1) // G)
        assert np.array_equal(a[0].view(np.uint8), b[0]) and np.array_equal(a[2].view(np.uint8), b[2])
        assert np.array_equal(a[1], b[1]) and np.array_equal(a[3], b[3])
    x = np.zeros((4, 2 * 100), np.uint16)
    gy = np.zeros((4, 100), np.uint16)
    with pytest.raises(ValueError):
        oracle.silu_dot_fwd_bwd_quant_fuse(x, gy, group_size=0)

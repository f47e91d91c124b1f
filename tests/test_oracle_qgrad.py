"""Pins of the oracle's quantized-grad_y path (no GPU).

Reading (the page lists grad_y as a bf16 input; the chained backward hands it
over already quantized): codes q int8 [M, K] and fp32 scales s [M, K/128],
one per token and 128 consecutive channels -- the row-group format the op
writes for grad_input -- standing for q * s.

Pins, each against something other than the oracle's own dequantization:
  * power-of-two scales make every q * s a bf16 value, so the whole op must
    equal the pinned bf16-grad_y whole op on that grad_y, bit for bit, in
    every group size and output format;
  * with any scales the first stage must equal torch's float64 autograd of
    sum(dy * silu(g) * u), dy built by repeating each scale over its 128
    channels, rounded by the pinned bf16 rounding.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads as W


def _bf16_of_exact_f32(v: np.ndarray) -> np.ndarray:
    """bf16 bits of float32 values that are bf16 values (checked)."""
    u = np.ascontiguousarray(v, dtype=np.float32).view(np.uint32)
    assert not (u & 0xFFFF).any(), "value is not a bf16 value"
    return (u >> 16).astype(np.uint16)


@pytest.mark.parametrize("G", [128, 64, 32])
@pytest.mark.parametrize("fmt", [(0, 0, 0), (1, 1, 1), (0, 1, 1), (1, 0, 0)])
@pytest.mark.parametrize("M,K", [(300, 384), (129, 256), (129, 208)])
def test_whole_op_pow2_scales_equals_bf16_op(M, K, G, fmt):
    w = W.small_workload(M, K, seed=M + K + G, zero_group_every=7)
    x, _ = W.make_inputs(w)
    q, s = W.quantized_grad_y(w, pow2_scales=True)
    assert len(np.unique(s)) > 3 and (s[:, :, None] != s[:1, :1, None]).any()
    gy = _bf16_of_exact_f32(q.astype(np.float32) * np.repeat(s, 128, axis=1)[:, :K])
    got = oracle.silu_dot_fwd_bwd_quant_fuse_qgrad(x, q, s, G, *fmt)
    ref = oracle.silu_dot_fwd_bwd_quant_fuse_fmt(x, gy, G, *fmt)
    for a, b, name in zip(got, ref, ("grad_input_q", "grad_input_s", "y_q_t", "y_s_t")):
        assert np.array_equal(a, b, equal_nan=True), name


def test_first_stage_against_autograd():
    M, K = 6, 256
    w = W.small_workload(M, K, seed=5, zero_group_every=4)
    x, _ = W.make_inputs(w)
    q, s = W.quantized_grad_y(w)
    assert (s != np.exp2(np.rint(np.log2(s)))).all()      # not powers of two
    dy = torch.tensor(q.astype(np.float64) * np.repeat(s.astype(np.float64), 128, axis=1))
    xf = torch.tensor(W.bf16_bits_to_f32(x).astype(np.float64))
    g = xf[:, :K].clone().requires_grad_(True)
    u = xf[:, K:].clone().requires_grad_(True)
    y = torch.nn.functional.silu(g) * u
    (y * dy).sum().backward()
    want = [np.array([oracle.bf16_rne(float(v)) for v in t.detach().reshape(-1).tolist()],
                     np.uint16).reshape(M, K) for t in (y, g.grad, u.grad)]
    got = oracle.swiglu_bwd_bf16_dy(x, oracle.dequant_grad_y(q, s))
    for a, b, name in zip(got, want, ("y", "d_gate", "d_up")):
        assert np.array_equal(a, b), name
    assert (q[0, :128] == 0).all() and (got[1][0, :128] == 0).all()   # a zero code group


def test_dequant_is_exact_in_fp64():
    """q * s has at most 8 + 24 significant bits: the fp64 product is exact,
    so dividing back by the scale returns the code."""
    w = W.small_workload(64, 384, seed=11)
    q, s = W.quantized_grad_y(w)
    dy = oracle.dequant_grad_y(q, s)
    back = dy / np.repeat(s.astype(np.float64), 128, axis=1)
    assert np.array_equal(back, q.astype(np.float64))


def test_qgrad_short_last_scale_group():
    """K = 200: a row's second scale covers its last 72 channels only."""
    w = W.small_workload(16, 200, seed=13)
    q, s = W.quantized_grad_y(w)
    assert s.shape == (16, 2)
    dy = oracle.dequant_grad_y(q, s)
    assert np.array_equal(dy[:, 128:], q[:, 128:].astype(np.float64) * s[:, 1:2].astype(np.float64))
    assert np.array_equal(dy[:, :128], q[:, :128].astype(np.float64) * s[:, :1].astype(np.float64))

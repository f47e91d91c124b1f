"""The forward-side neighbour on the GPU (SwiGLU forward + q8_1 rows) against
the oracle on the same seeded inputs: h, the codes, d and sum of every block.
Tolerances: tests/gpu_util.py (compare_fwd).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests import gpu_util as U

pytestmark = pytest.mark.gpu


def _check(g, u, w, limit=0.0, where="", ld_pad=0):
    got = U.run_cuda_fwd(g, u, w, limit, ld_pad)
    ref = oracle.swiglu_q8_1_rows(g, u, w, limit)
    return U.compare_fwd(got, ref, where)


@pytest.mark.parametrize("idx,limit", [(0, 0.0), (1, 0.0), (3, 7.0), (2, float("nan"))])
def test_fwd_full_workloads(idx, limit):
    """gate and up are the halves of the workload's x (views with row stride 2K)."""
    w = W.WORKLOADS[idx]
    g, u, wt = W.fwd_inputs(w)
    _check(g, u, wt, limit, w.name)


@pytest.mark.parametrize("rows,inter", [(1, 32), (3, 96), (37, 288), (5, 544), (130, 1408), (2, 2080)])
@pytest.mark.parametrize("with_w", [False, True])
def test_fwd_odd_shapes(rows, inter, with_w):
    w = W.small_workload(rows, inter if inter % 128 == 0 else 128 * (inter // 128 + 1), seed=rows + inter)
    x, _ = W.make_inputs(w)
    g, u = x[:, :inter], x[:, w.K:w.K + inter]
    wt = W.row_weights(rows + inter, rows) if with_w else None
    _check(g, u, wt, 0.0, f"rows={rows} inter={inter}")


def test_fwd_tiny_zero_clamped_and_padded():
    w = W.small_workload(64, 256, seed=61, sigma_x=1e-19)     # h ~ 1e-38: the divide path
    g, u, wt = W.fwd_inputs(w)
    _check(g, u, wt, 0.0, "tiny")
    w = W.small_workload(64, 256, seed=62, sigma_x=20.0)      # saturated sigmoid, clamp at 5
    g, u, wt = W.fwd_inputs(w)
    _check(g, u, wt, 5.0, "clamped")
    _check(g, u, wt, -1.0, "negative limit: no clamp")
    g0 = g.copy()
    g0[:, 32:96] = 0                                        # silu(0) = 0: zero blocks (signed h)
    _check(g0, u, wt, 0.0, "zero blocks")
    _check(g, u, wt, 0.0, "padded rows", ld_pad=24)


def test_fwd_full_size_sampled_rows():
    """M=16384, inter=7168 in one launch; rows are independent, so the oracle
    runs on a sample of rows."""
    w = W.WORKLOADS[4]
    g, u, wt = W.fwd_inputs(w)
    h, q8 = U.run_cuda_fwd(g, u, wt)
    rng = np.random.default_rng(4)
    rows = np.unique(np.concatenate([[0, w.M - 1], rng.integers(0, w.M, 30)]))
    ref = oracle.swiglu_q8_1_rows(np.ascontiguousarray(g[rows]), np.ascontiguousarray(u[rows]), wt[rows])
    U.compare_fwd((h[rows], q8[rows]), ref, "M16384 sampled rows")


def test_fwd_gates_below_the_fp32_sigmoid_range():
    """gate in [-130, -60]: silu(g) * u * w is a normal or subnormal bf16 down to
    about g = -92, although sigma(g) leaves the normal fp32 range below -87."""
    rows, inter = 8, 256
    gv = np.linspace(-130.0, -60.0, rows * inter).reshape(rows, inter)
    uv = np.tile(np.array([1.0, -3.5, 40.0, -0.25]), (rows, inter // 4))
    from tests.exact import bf16_round_bits64
    g, u = bf16_round_bits64(gv), bf16_round_bits64(uv)
    wt = np.linspace(0.1, 1.0, rows).astype(np.float32)
    st = _check(g, u, wt, 0.0, "deep negative gates")
    h, _ = U.run_cuda_fwd(g, u, wt)
    assert (h & 0x7FFF).astype(bool).sum() > inter      # many nonzero h where fp32 sigma underflows
    del st


@pytest.mark.slow
def test_fwd_maximum_inter_sampled_rows():
    """inter = 2^20 (the largest accepted) on a few rows; rows are independent,
    so the oracle runs on every row here."""
    w = W.small_workload(3, 1 << 20, seed=98)
    g, u, wt = W.fwd_inputs(w)
    _check(g, u, wt, 0.0, "inter 2^20")

"""CUDA path vs the oracle with quantization groups of 32, 64 and 256 (the
page's group_size argument; 128 is covered by the other parity tests), in the
page's output format and the others, on the same seeded inputs.

A 128 x 128 tile holds 16 (4) groups of 32 (64) on each axis; token groups
wholly past M in a tail tile are not written, which the guarded, prefilled
outputs check.  Groups of 256 run the kernel with 256 x 256 units: with
K % 256 != 0 the last unit holds a shorter channel group (K = 128, 384 and
1408 below), with M % 256 != 0 a tail token group.  Tolerances:
tests/gpu_util.py (compare_fmt).
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
import workloads as W
from tests import gpu_util as U

pytestmark = pytest.mark.gpu

ALL_FORMATS = [(c, s, l) for c in (0, 1) for s in (0, 1) for l in (0, 1)]
FMT_IDS = [f"{'e4m3' if c else 'int8'}-{'e8m0' if s else 'fp32'}-{'mgk' if l else 'kmg'}"
           for c, s, l in ALL_FORMATS]


def _check(x, gy, G, fmt, where):
    codes, scales, layout = fmt
    got = U.run_cuda_fmt(x, gy, codes, scales, layout, G)
    ref = oracle.silu_dot_fwd_bwd_quant_fuse_fmt(x, gy, G, codes, scales, layout)
    return U.compare_fmt(got, ref, codes, scales, layout, f"{where} G={G} {fmt}", G)


@pytest.mark.parametrize("fmt", ALL_FORMATS, ids=FMT_IDS)
@pytest.mark.parametrize("G", [32, 64, 256])
@pytest.mark.parametrize("idx", [0, 1])
def test_group_sizes_full_workloads(idx, G, fmt):
    w = W.WORKLOADS[idx]
    x, gy = W.make_inputs(w)
    _check(x, gy, G, fmt, w.name)


@pytest.mark.parametrize("G", [32, 64, 256])
@pytest.mark.parametrize("M,K", [(1, 128), (31, 384), (33, 128), (65, 256), (129, 128), (200, 384),
                                 (257, 256), (1000, 128), (513, 640), (300, 16)])
def test_group_sizes_odd_and_tail_shapes(M, K, G):
    x, gy = W.make_inputs(W.small_workload(M, K, seed=M * 13 + K + G))
    _check(x, gy, G, (0, 0, 0), f"M={M} K={K}")
    _check(x, gy, G, (1, 1, 1), f"M={M} K={K}")


@pytest.mark.parametrize("G", [32, 64, 256])
def test_group_sizes_outliers_zero_groups_and_tiny(G):
    x, gy = W.make_inputs(W.WORKLOADS[3])          # outliers, zero groups, a 32-token tail group
    _check(x, gy, G, (0, 0, 0), "outliers")
    _check(x, gy, G, (1, 0, 1), "outliers")
    x, gy = W.make_inputs(W.small_workload(300, 256, seed=51, sigma_grad_y=1e-36))
    _check(x, gy, G, (0, 0, 0), "tiny")
    _check(x, gy, G, (1, 1, 0), "tiny")


@pytest.mark.parametrize("G", [32, 64, 256])
def test_group_sizes_over_the_whole_exponent_range(G):
    """gate = 32, grad_y = 1, up = a_i on token group i (of G tokens): the
    group amaxes sweep one bf16 value per exponent field, subnormals included."""
    pats = [0x0001, 0x0005, 0x0041, 0x007F] + [(e << 7) | ((e * 37) % 128) for e in range(1, 249)]
    a = np.array(pats, dtype=np.uint16)
    M, K = G * len(pats), 128
    x = np.empty((M, 2 * K), np.uint16)
    x[:, :K] = 0x4200                                   # 32.0
    x[:, K:] = np.repeat(a, G)[:, None]
    gy = np.full((M, K), 0x3F80, np.uint16)             # 1.0
    _check(x, gy, G, (0, 0, 0), "exponent sweep")
    _check(x, gy, G, (1, 1, 0), "exponent sweep")


@pytest.mark.slow
@pytest.mark.parametrize("idx", [3, 2, 4])
def test_group_256_on_the_outlier_and_large_workloads(idx):
    """Groups of 256 in full, in the page's format: M=4000 K=2048 (outliers,
    zero groups, a 160-token tail group), M=8192 K=4096 and M=16384 K=7168."""
    x, gy = W.make_inputs(W.WORKLOADS[idx])
    _check(x, gy, 256, (0, 0, 0), W.WORKLOADS[idx].name)

"""CUDA path vs the oracle in every output format (FP8 E4M3 codes, E8M0
scales, y_s_t [Mg, K]), element by element on the same seeded inputs.

Tolerances and their derivation: tests/gpu_util.py (compare_fmt).  Outputs
are guarded and prefilled with bytes the op never writes, as in the INT8
parity tests.
"""
from __future__ import annotations

import json
import os

import numpy as np
import pytest

import oracle
import workloads as W
from tests import gpu_util as U

pytestmark = pytest.mark.gpu

# (codes, scales, ys_layout); the page's own format (0, 0, 0) is covered by
# the INT8 parity tests
FORMATS = [(c, s, l) for c in (0, 1) for s in (0, 1) for l in (0, 1) if (c, s, l) != (0, 0, 0)]
FMT_IDS = [f"{'e4m3' if c else 'int8'}-{'e8m0' if s else 'fp32'}-{'mgk' if l else 'kmg'}"
           for c, s, l in FORMATS]

_STATS = {}
_REF = {}


def _check(w: W.Workload, fmt, x=None, gy=None):
    codes, scales, layout = fmt
    if x is None:
        x, gy = W.make_inputs(w)
    got = U.run_cuda_fmt(x, gy, codes, scales, layout)
    key = (w.name, w.M, w.K, w.seed, fmt)
    ref = oracle.silu_dot_fwd_bwd_quant_fuse_fmt(x, gy, 128, codes, scales, layout)
    st = U.compare_fmt(got, ref, codes, scales, layout, f"{w.name} {fmt}")
    _STATS[f"{w.name}/{fmt}"] = st
    return got, ref


@pytest.fixture(scope="module", autouse=True)
def _report():
    yield
    path = os.environ.get("SDQ_PARITY_REPORT")
    if path:
        path = path.replace(".json", "_formats.json")
        with open(path, "w") as f:
            json.dump(_STATS, f, indent=1)


@pytest.mark.parametrize("fmt", FORMATS, ids=FMT_IDS)
@pytest.mark.parametrize("idx", [0, 1, 3])
def test_formats_full_workloads(idx, fmt):
    _check(W.WORKLOADS[idx], fmt)


@pytest.mark.parametrize("fmt", FORMATS, ids=FMT_IDS)
@pytest.mark.parametrize("M,K", [(1, 128), (33, 384), (127, 128), (129, 256), (257, 384), (1000, 128)])
def test_formats_odd_and_tail_shapes(M, K, fmt):
    _check(W.small_workload(M, K, seed=M * 11 + K), fmt)


@pytest.mark.parametrize("fmt", FORMATS, ids=FMT_IDS)
def test_formats_tiny_saturated_and_zero_groups(fmt):
    # tiny d_gate/d_up groups (amax below 2^-117: the out-of-line scale path),
    # saturated sigmoid, outliers, and all-zero groups with -0.0 elements
    # (gate = 0 -> y = 0 * up keeps up's sign)
    _check(W.small_workload(300, 256, seed=41, sigma_x=1.0, sigma_grad_y=1e-36), fmt)
    _check(W.small_workload(300, 256, seed=42, sigma_x=30.0, sigma_grad_y=3.0,
                            outlier_frac=0.02, outlier_mult=50.0), fmt)
    w = W.small_workload(300, 384, seed=43)
    x, gy = W.make_inputs(w)
    x[:128, 128:256] = 0          # y = +-0 for tokens 0..127, channels 128..255
    x[200, :] = 0                 # token 200: both row groups all-zero
    x[:, 384 + 300] = 0           # up = 0 in one channel
    _check(w, fmt, x, gy)


@pytest.mark.parametrize("fmt", FORMATS, ids=FMT_IDS)
def test_formats_over_the_whole_exponent_range(fmt):
    """gate = 32, grad_y = 1, up = a_i on token group i: the group amaxes sweep
    one bf16 value per exponent field, subnormals included, so every scale
    path (table, out-of-line, clamped E8M0) is compared with the oracle."""
    G = 128
    pats = [0x0001, 0x0005, 0x0041, 0x007F] + [(e << 7) | ((e * 37) % 128) for e in range(1, 249)]
    a = np.array(pats, dtype=np.uint16)
    M, K = G * len(pats), 128
    x = np.empty((M, 2 * K), np.uint16)
    x[:, :K] = 0x4200                                   # 32.0
    x[:, K:] = np.repeat(a, G)[:, None]
    gy = np.full((M, K), 0x3F80, np.uint16)             # 1.0
    w = W.small_workload(M, K, seed=0)
    _check(w, fmt, x, gy)


@pytest.mark.slow
@pytest.mark.parametrize("fmt,G", [((1, 1, 1), 128), ((0, 0, 0), 64), ((1, 0, 0), 32)])
def test_formats_full_size_sampled_tiles(fmt, G):
    """M=16384, K=7168 in one launch (the bench's largest workload) in another
    format or group size: 24 sampled 128x128 tiles against the format oracle
    on each tile (every group lies inside one tile)."""
    import torch
    import swiglu_backward_int8_b200 as sdq
    codes, scales, layout = fmt
    w = W.WORKLOADS[4]
    x, gy = W.make_inputs(w)
    M, K = w.M, w.K
    xd, gyd = U.to_device_bf16(x), U.to_device_bf16(gy)
    names = ("e4m3" if codes else "int8", "e8m0" if scales else "fp32", "mg_k" if layout else "k_mg")
    outs = sdq.allocate_outputs(M, K, "cuda", G, *names)
    sdq.silu_dot_fwd_bwd_quant_fuse(xd, gyd, *outs, group_size=G, codes=names[0], scales=names[1],
                                    y_scale_layout=names[2])
    torch.cuda.synchronize()
    assert sdq.sdq_device_status() == 0
    giq, gis, yqt, yst = (t.view(torch.uint8).cpu().numpy() if t.dtype != torch.float32 else t.cpu().numpy()
                          for t in outs)
    if layout:
        yst = yst.T
    rng = np.random.default_rng(7)
    tiles = {(0, 0), (M // 128 - 1, K // 128 - 1)}
    while len(tiles) < 24:
        tiles.add((int(rng.integers(M // 128)), int(rng.integers(K // 128))))
    per = 128 // G
    n_diff = 0
    for i, j in sorted(tiles):
        r0, c0 = 128 * i, 128 * j
        xt = np.concatenate([x[r0:r0 + 128, c0:c0 + 128], x[r0:r0 + 128, K + c0:K + c0 + 128]], axis=1)
        ref = oracle.silu_dot_fwd_bwd_quant_fuse_fmt(xt, gy[r0:r0 + 128, c0:c0 + 128], G, codes, scales, 0)
        got = (np.concatenate([giq[r0:r0 + 128, c0:c0 + 128], giq[r0:r0 + 128, K + c0:K + c0 + 128]], axis=1),
               np.concatenate([gis[r0:r0 + 128, j * per:(j + 1) * per],
                               gis[r0:r0 + 128, K // G + j * per:K // G + (j + 1) * per]], axis=1),
               yqt[c0:c0 + 128, r0:r0 + 128], yst[c0:c0 + 128, i * per:(i + 1) * per])
        st = U.compare_fmt(got, ref, codes, scales, 0, f"M16384 tile ({i},{j}) {fmt} G={G}", G,
                           max_frac=1.0)                 # the 0.1 % bound applies to the whole sample
        for name in ("grad_input_q", "y_q_t"):
            n_diff += st[name]["n_diff"]
    total = 24 * 128 * 128 * 3
    assert n_diff <= 1e-3 * total, f"{n_diff} of {total} sampled codes differ"

"""CUDA path vs the CPU oracle, element by element, on the same seeded inputs.

Tolerances and their derivation are in tests/gpu_util.py.  Every output is
surrounded by guard bytes and prefilled with values the op never writes, so
a case also proves that each element was written exactly where it belongs.
"""
from __future__ import annotations

import json
import os

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests import gpu_util as U

pytestmark = pytest.mark.gpu

_STATS = {}


def _check(w: W.Workload):
    x, gy = W.make_inputs(w)
    got = U.run_cuda(x, gy)
    ref = oracle.silu_dot_fwd_bwd_quant_fuse(x, gy, w.group_size)
    st = U.compare(got, ref, w.name)
    _STATS[w.name] = st
    return got, ref, st


@pytest.fixture(scope="module", autouse=True)
def _report():
    yield
    path = os.environ.get("SDQ_PARITY_REPORT")
    if path:
        with open(path, "w") as f:
            json.dump(_STATS, f, indent=1)


# The four configurations the oracle finishes in seconds run in full.
@pytest.mark.parametrize("idx", [0, 1, 2, 3])
def test_workload_full(idx):
    _check(W.WORKLOADS[idx])


@pytest.mark.parametrize("M", [1, 4, 16, 31, 32, 33, 100, 127, 128, 129, 200, 257, 1000])
@pytest.mark.parametrize("K", [128, 384])
def test_odd_and_tail_shapes(M, K):
    _check(W.small_workload(M, K, seed=M * 7 + K))


def test_saturated_and_tiny_values():
    # |gate| up to ~150 (sigma saturates to 0 / 1), tiny grad_y
    _check(W.small_workload(300, 256, seed=17, sigma_x=30.0, sigma_grad_y=1e-6))
    _check(W.small_workload(300, 256, seed=18, sigma_x=1.0, sigma_grad_y=3.0,
                            outlier_frac=0.02, outlier_mult=50.0))


def test_zero_groups_on_both_axes():
    M, K = 300, 384
    x, gy = W.make_inputs(W.small_workload(M, K, seed=21))
    x[:128, 128:256] = 0           # gate = 0 -> y = 0 for tokens 0..127, channels 128..255
    x[200, :] = 0                  # token 200: gate = up = 0 -> both row halves all-zero
    x[:, K + 300] = 0              # up = 0 in one channel: y = 0 and d_gate = 0 there
    got = U.run_cuda(x, gy)
    ref = oracle.silu_dot_fwd_bwd_quant_fuse(x, gy)
    U.compare(got, ref, "zero groups")
    giq, gis, yqt, yst = got
    assert np.all(yst[128:256, 0] == 1.0) and not yqt[128:256, :128].any()
    assert np.all(gis[200] == 1.0) and not giq[200].any()


def test_outlier_workload_zero_row_groups():
    w = W.WORKLOADS[3]
    x, gy = W.make_inputs(w)
    giq, gis, yqt, yst = U.run_cuda(x, gy)
    for r, j in W.zero_group_positions(w):
        assert gis[r, j] == 1.0 and gis[r, w.Kg + j] == 1.0
        assert not giq[r, j * 128:(j + 1) * 128].any()
        assert not giq[r, w.K + j * 128:w.K + (j + 1) * 128].any()


def test_deterministic_and_on_a_side_stream():
    w = W.small_workload(515, 256, seed=5)
    x, gy = W.make_inputs(w)
    a = U.run_cuda(x, gy)
    s = torch.cuda.Stream()
    b = U.run_cuda(x, gy, stream=s)
    for u, v in zip(a, b):
        assert np.array_equal(u, v)


def test_m_zero_is_a_noop():
    import swiglu_backward_int8_b200 as sdq
    x = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    gy = torch.empty((0, 128), dtype=torch.bfloat16, device="cuda")
    outs = sdq.allocate_outputs(0, 128, "cuda")
    sdq.silu_dot_fwd_bwd_quant_fuse(x, gy, *outs)
    torch.cuda.synchronize()


def test_misaligned_input_is_rejected_and_nothing_written():
    import swiglu_backward_int8_b200 as sdq
    M, K = 128, 128
    base = torch.zeros(M * 2 * K + 8, dtype=torch.bfloat16, device="cuda")
    x = base[1:1 + M * 2 * K].view(M, 2 * K)          # 2-byte offset
    gy = torch.zeros(M, K, dtype=torch.bfloat16, device="cuda")
    outs = [torch.full(s, -128 if i % 2 == 0 else -1, dtype=dt, device="cuda")
            for i, (s, dt) in enumerate(zip(sdq.output_shapes(M, K),
                                            (torch.int8, torch.float32, torch.int8, torch.float32)))]
    with pytest.raises(sdq.SdqError) as ei:
        sdq.silu_dot_fwd_bwd_quant_fuse(x, gy, *outs)
    assert ei.value.status == sdq.Status.ERR_ALIGN
    torch.cuda.synchronize()
    assert (outs[0] == -128).all() and (outs[1] == -1).all()


@pytest.mark.parametrize("M,K,chunk", [(4096, 1408, 0), (4000, 2048, 1024), (1000, 256, 256),
                                       (77, 128, 0)])
def test_host_buffer_entry_matches_device_entry(M, K, chunk):
    import swiglu_backward_int8_b200 as sdq
    x, gy = W.make_inputs(W.small_workload(M, K, seed=M + K))
    dev = U.run_cuda(x, gy)
    xh = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory()
    gyh = torch.from_numpy(gy.view(np.int16)).view(torch.bfloat16).pin_memory()
    outs = [t.pin_memory() for t in sdq.allocate_outputs(M, K, "cpu")]
    for t in outs:
        t.fill_(-128 if t.dtype == torch.int8 else float("nan"))
    ws = torch.empty(sdq.sdq_fuse_host_workspace_bytes(M, K, chunk), dtype=torch.uint8, device="cuda")
    sdq.silu_dot_fwd_bwd_quant_fuse_host(xh, gyh, *outs, workspace=ws, chunk_rows=chunk)
    for a, b in zip(dev, outs):
        assert np.array_equal(a, b.numpy())
    # pageable host memory works too
    outs2 = sdq.allocate_outputs(M, K, "cpu")
    sdq.silu_dot_fwd_bwd_quant_fuse_host(torch.from_numpy(x.view(np.int16)).view(torch.bfloat16),
                                         torch.from_numpy(gy.view(np.int16)).view(torch.bfloat16),
                                         *outs2, workspace=ws, chunk_rows=chunk)
    for a, b in zip(dev, outs2):
        assert np.array_equal(a, b.numpy())


def test_host_entry_rejects_small_workspace():
    import swiglu_backward_int8_b200 as sdq
    M, K = 256, 256
    x = torch.zeros(M, 2 * K, dtype=torch.bfloat16)
    gy = torch.zeros(M, K, dtype=torch.bfloat16)
    outs = sdq.allocate_outputs(M, K, "cpu")
    ws = torch.empty(1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(sdq.SdqError) as ei:
        sdq.silu_dot_fwd_bwd_quant_fuse_host(x, gy, *outs, workspace=ws)
    assert ei.value.status == sdq.Status.ERR_WORKSPACE


def _tiles_to_sample(Mg, Kg, n, seed):
    rng = np.random.default_rng(seed)
    picks = {(0, 0), (Mg - 1, Kg - 1), (0, Kg - 1), (Mg - 1, 0)}
    while len(picks) < n:
        picks.add((int(rng.integers(Mg)), int(rng.integers(Kg))))
    return sorted(picks)


@pytest.mark.slow
def test_largest_workload_in_full_and_invariants():
    """M=16384 K=7168 (the bandwidth-roofline workload, 1.07 GB a call) in the
    bench's launch configuration: every element of all four outputs against
    the oracle on the whole op (about 8 s of one CPU core), every element
    written and nothing outside, and properties that hold at any size: each
    group's largest |q| is 127 unless the group is all zero (scale 1, q 0)."""
    w = W.WORKLOADS[4]
    M, K, G = w.M, w.K, 128
    x, gy = W.make_inputs(w)
    got = U.run_cuda(x, gy)          # guard bytes, sentinels, device status
    giq, gis, yqt, yst = got
    assert (gis > 0).all() and (yst > 0).all()
    rmax = np.abs(giq.reshape(M, 2 * w.Kg, G).astype(np.int16)).max(axis=2)
    assert ((rmax == 127) | ((rmax == 0) & (gis == 1))).all()
    cmax = np.abs(yqt.reshape(K, M // G, G).astype(np.int16)).max(axis=2)
    assert ((cmax == 127) | ((cmax == 0) & (yst == 1))).all()
    ref = oracle.silu_dot_fwd_bwd_quant_fuse(x, gy, w.group_size)
    _STATS[w.name] = U.compare(got, ref, w.name)


def test_scales_exact_over_the_whole_exponent_range():
    """Closed form, no oracle: gate = 32 makes sigma(32) round to 1 in fp32
    (and silu(32), silu'(32) round to 32 and 1 in bf16 from fp64), so with
    grad_y = 1 and up = a_i on every channel of token group i:
        y = 32 a_i,  d_gate = a_i,  d_up = 32.
    a_i sweeps one bf16 value per exponent field, subnormals included, so every
    scale must equal the IEEE fp32 quotient amax / 127 and every code is 127."""
    G = 128
    pats = [0x0005, 0x0041, 0x007F] + [(e << 7) | ((e * 37) % 128) for e in range(1, 249)]
    a = np.array(pats, dtype=np.uint16)
    M, K = G * len(pats), 128
    x = np.empty((M, 2 * K), np.uint16)
    x[:, :K] = 0x4200                                   # 32.0
    x[:, K:] = np.repeat(a, G)[:, None]
    gy = np.full((M, K), 0x3F80, np.uint16)             # 1.0
    giq, gis, yqt, yst = U.run_cuda(x, gy)
    af = W.bf16_bits_to_f32(a)
    f32 = np.float32
    want_dg = af / f32(127)
    want_y = (af * f32(32)) / f32(127)
    assert np.array_equal(gis[:, 0], np.repeat(want_dg, G))
    assert np.all(gis[:, 1] == f32(32) / f32(127))
    assert np.array_equal(yst[0], want_y) and np.all(yst == yst[0:1])
    assert np.all(giq == 127) and np.all(yqt == 127)


def test_bounded_wait_runs_out_and_is_reported():
    """Failure detection without a fault: the test hook withholds the first
    load, every CTA's first wait runs out after 20 ms, the kernel stops early,
    the status word reports the timeout, and the next call is correct."""
    import swiglu_backward_int8_b200 as sdq
    from swiglu_backward_int8_b200 import _lib
    w = W.small_workload(1024, 256, seed=31)
    x, gy = W.make_inputs(w)
    xd, gyd = U.to_device_bf16(x), U.to_device_bf16(gy)
    outs = sdq.allocate_outputs(w.M, w.K, "cuda")
    stream = torch.cuda.current_stream().cuda_stream
    assert sdq.sdq_device_status(stream) == sdq.Status.OK
    _lib.sdq_fuse_test_stall(xd.data_ptr(), gyd.data_ptr(), *(o.data_ptr() for o in outs),
                             w.M, w.K, 128, 20_000_000, stream)
    assert sdq.sdq_device_status(stream) == sdq.Status.ERR_TIMEOUT
    assert sdq.sdq_device_status(stream) == sdq.Status.OK      # read-and-clear
    got = U.run_cuda(x, gy)                                     # the context is still usable
    U.compare(got, oracle.silu_dot_fwd_bwd_quant_fuse(x, gy), "after a timeout")


@pytest.mark.slow
@pytest.mark.parametrize("M,K", [(129, 1048576), (1 << 20, 128)])
def test_maximum_sizes_sampled_tiles(M, K):
    """The largest K the library accepts (2^20 channels) with a ragged tail
    token group, and a million tokens: sampled tiles against the oracle on
    each tile, every element written."""
    import swiglu_backward_int8_b200 as sdq
    w = W.small_workload(M, K, seed=99)
    x, gy = W.make_inputs(w)
    xd, gyd = U.to_device_bf16(x), U.to_device_bf16(gy)
    outs = sdq.allocate_outputs(M, K, "cuda")
    for t in outs:
        t.fill_(U.SENTINEL_Q if t.dtype == torch.int8 else float("nan"))
    sdq.silu_dot_fwd_bwd_quant_fuse(xd, gyd, *outs)
    torch.cuda.synchronize()
    assert sdq.sdq_device_status() == 0
    giq, gis, yqt, yst = outs
    assert not (giq == U.SENTINEL_Q).any() and not (yqt == U.SENTINEL_Q).any()
    assert torch.isfinite(gis).all() and torch.isfinite(yst).all()
    host = [t.cpu().numpy() for t in outs]
    Mg, Kg = (M + 127) // 128, K // 128
    n_diff = n_all = 0
    for (i, j) in _tiles_to_sample(Mg, Kg, 16, seed=M + K):
        got, ref = U.tile_of(host, M, K, i, j), U.oracle_tile(x, gy, i, j)
        st = U.compare(got, ref, f"M={M} K={K} tile ({i},{j})", max_frac=1.0)   # bound over the sample
        n_diff += st["grad_input_q"]["n_diff"] + st["y_q_t"]["n_diff"]
        n_all += ref[0].size + ref[2].size
    assert n_diff <= U.INT8_MAX_FRAC * n_all, f"{n_diff} of {n_all} sampled codes differ"


def test_concurrent_streams_and_graph_replay_are_bit_identical():
    """The device entry keeps no per-call state: calls on three streams at
    once, and calls captured in a CUDA graph and replayed twice, give the
    same bytes as single calls."""
    import swiglu_backward_int8_b200 as sdq
    shapes = [(515, 256, 1), (1000, 384, 2), (300, 1408, 3)]
    ins, want = [], []
    for M, K, seed in shapes:
        x, gy = W.make_inputs(W.small_workload(M, K, seed=seed))
        xd, gyd = U.to_device_bf16(x), U.to_device_bf16(gy)
        ins.append((xd, gyd))
        want.append([t.cpu() for t in sdq.run(xd, gyd)])
    # concurrent: each call on its own stream, all enqueued before any sync
    streams = [torch.cuda.Stream() for _ in shapes]
    outs = [sdq.allocate_outputs(M, K, "cuda") for M, K, _ in shapes]
    torch.cuda.synchronize()
    for (xd, gyd), o, s in zip(ins, outs, streams):
        with torch.cuda.stream(s):
            sdq.silu_dot_fwd_bwd_quant_fuse(xd, gyd, *o)
    torch.cuda.synchronize()
    for o, w in zip(outs, want):
        for a, b in zip(o, w):
            assert torch.equal(a.cpu(), b)
    # graph capture and replay
    gouts = [sdq.allocate_outputs(M, K, "cuda") for M, K, _ in shapes]
    for o in gouts:
        for t in o:
            t.zero_()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=torch.cuda.Stream()):
        for (xd, gyd), o in zip(ins, gouts):
            sdq.silu_dot_fwd_bwd_quant_fuse(xd, gyd, *o)
    for _ in range(2):
        g.replay()
        torch.cuda.synchronize()
        for o, w in zip(gouts, want):
            for a, b in zip(o, w):
                assert torch.equal(a.cpu(), b)
    assert sdq.sdq_device_status() == 0
    del g


def test_back_to_back_bursts_are_bit_identical():
    """Stress for the shared-memory ring: 25 bursts of 8 back-to-back calls
    (each into its own outputs, so consecutive launches overlap their start
    and end) on M=8192 K=4096, every call's four outputs compared byte for
    byte with a single call's, and that call with the oracle.  A stage read
    before its copy had landed would show as a difference."""
    import swiglu_backward_int8_b200 as sdq
    w = W.WORKLOADS[2]
    x, gy = W.make_inputs(w)
    xd, gyd = U.to_device_bf16(x), U.to_device_bf16(gy)
    ref = sdq.allocate_outputs(w.M, w.K, "cuda")
    sdq.silu_dot_fwd_bwd_quant_fuse(xd, gyd, *ref)
    torch.cuda.synchronize()
    U.compare([t.cpu().numpy() for t in ref], oracle.silu_dot_fwd_bwd_quant_fuse(x, gy), w.name)
    sets = [sdq.allocate_outputs(w.M, w.K, "cuda") for _ in range(8)]
    bad = 0
    for _ in range(25):
        for o in sets:
            for t in o:
                t.zero_()
        for o in sets:
            sdq.silu_dot_fwd_bwd_quant_fuse(xd, gyd, *o)
        for o in sets:
            bad += sum(int(not torch.equal(a, b)) for a, b in zip(o, ref))
    torch.cuda.synchronize()
    assert sdq.sdq_device_status() == 0
    assert bad == 0, f"{bad} outputs differ from a single call's"

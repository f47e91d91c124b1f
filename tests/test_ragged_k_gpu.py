"""K not a multiple of the group size (K a multiple of 16): the last channel
tile is partial, and each half of [d_gate | d_up] ends in a shorter group.
Every output is written into a buffer with padded rows and, for the
channel-major outputs (y_q_t, y_s_t), extra rows past K, all filled with
sentinels: the logical outputs must equal the oracle's within the tolerances
of tests/gpu_util.py, and no byte outside them may change.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests import gpu_util as U

pytestmark = pytest.mark.gpu

EXTRA = 48   # sentinel rows past K in y_q_t / y_s_t ([K, Mg] layout) and columns past K ([Mg, K])


def _run(x_u16, gy_u16, G, fmt, with_y=False, int8_grad_y=None):
    """sdq_fuse_strided (or sdq_fuse_int8_grad_y) with every output padded;
    returns numpy outputs like the format oracle (+ y) after checking that
    nothing outside them changed."""
    import swiglu_backward_int8_b200 as sdq
    codes, scales, layout = fmt
    M = x_u16.shape[0]
    K = x_u16.shape[1] // 2
    Kgs, Mg = (K + G - 1) // G, (M + G - 1) // G
    sq = U.SENTINEL_CODE[codes]
    sdt, sfill = (torch.uint8, U.SENTINEL_E8M0) if scales else (torch.float32, float("nan"))
    # (buffer rows, buffer cols, logical rows, logical cols, dtype, fill)
    specs = [(M, 2 * K + 16, M, 2 * K, torch.uint8, sq),
             (M, 2 * Kgs + 3, M, 2 * Kgs, sdt, sfill),
             (K + EXTRA, M + 16, K, M, torch.uint8, sq),
             ((Mg, K + EXTRA, Mg, K) if layout else (K + EXTRA, Mg + 2, K, Mg)) + (sdt, sfill)]
    bufs = [torch.full((r, c), f, dtype=dt, device="cuda") for r, c, _, _, dt, f in specs]
    views = [b[:lr, :lc] for b, (_, _, lr, lc, _, _) in zip(bufs, specs)]
    xd = U.to_device_bf16(x_u16)
    ybuf = torch.full((M, K + 8), 0x7FC1, dtype=torch.int16, device="cuda") if with_y else None
    bits = (sdq.FMT_E4M3 if codes else 0) | (sdq.FMT_E8M0 if scales else 0) | \
        (sdq.FMT_YS_MG_K if layout else 0)
    outs = [v for b, t in zip(bufs, views) for v in (t.data_ptr(), b.stride(0))]
    yargs = (ybuf.data_ptr(), ybuf.stride(0)) if with_y else (None, 0)
    stream = torch.cuda.current_stream().cuda_stream
    if int8_grad_y is None:
        gyd = U.to_device_bf16(gy_u16)
        sdq.sdq_fuse_strided(xd.data_ptr(), 2 * K, xd.data_ptr() + 2 * K, 2 * K, gyd.data_ptr(), K,
                             *outs, *yargs, M, K, G, bits, stream)
    else:
        q, s = (torch.from_numpy(a).cuda() for a in int8_grad_y)
        sdq.sdq_fuse_int8_grad_y(xd.data_ptr(), 2 * K, xd.data_ptr() + 2 * K, 2 * K, q.data_ptr(), K,
                                 s.data_ptr(), s.shape[1], *outs, *yargs, M, K, G, bits, stream)
    torch.cuda.synchronize()
    assert sdq.sdq_device_status() == 0
    got = []
    for b, (_, _, lr, lc, dt, f), name in zip(bufs, specs, ("grad_input_q", "grad_input_s", "y_q_t", "y_s_t")):
        h = b.cpu().numpy()
        mask = np.ones(h.shape, bool)
        mask[:lr, :lc] = False
        outside = h[mask]
        if dt == torch.float32:
            assert np.isnan(outside).all(), f"{name}: written outside its logical shape"
        else:
            assert (outside == f).all(), f"{name}: written outside its logical shape"
        got.append(h[:lr, :lc].copy())
    if with_y:
        h = ybuf.cpu().numpy().view(np.uint16)
        assert (h[:, K:] == 0x7FC1).all(), "y: padding written"
        got.append(h[:, :K].copy())
    return tuple(got)


@pytest.mark.parametrize("K", [16, 144, 208, 400, 1040])
@pytest.mark.parametrize("G,fmt", [(128, (0, 0, 0)), (64, (1, 1, 1)), (32, (0, 1, 0)), (128, (1, 0, 1)),
                                   (256, (0, 0, 0)), (256, (1, 1, 1))])
def test_partial_channel_tile_matches_the_oracle(K, G, fmt):
    M = 300
    x, gy = W.make_inputs(W.small_workload(M, K, seed=K + G, zero_group_every=0))
    got = _run(x, gy, G, fmt)
    ref = oracle.silu_dot_fwd_bwd_quant_fuse_fmt(x, gy, G, *fmt)
    U.compare_fmt(got, ref, *fmt, f"K={K} G={G}", G)


def test_partial_channel_tile_large():
    """M=4096, K=1424 (11 whole channel tiles and one of 16 channels), the
    page's format, in full."""
    M, K = 4096, 1424
    x, gy = W.make_inputs(W.small_workload(M, K, seed=77))
    got = _run(x, gy, 128, (0, 0, 0))
    U.compare_fmt(got, oracle.silu_dot_fwd_bwd_quant_fuse_fmt(x, gy, 128, 0, 0, 0), 0, 0, 0, "K=1424")


@pytest.mark.parametrize("K,G", [(208, 128), (1040, 128), (208, 256), (1040, 256), (400, 256)])
def test_partial_channel_tile_int8_grad_y_with_y(K, G):
    M = 257
    w = W.small_workload(M, K, seed=3 * K, zero_group_every=5)
    x, _ = W.make_inputs(w)
    q, s = W.quantized_grad_y(w)
    assert s.shape == (M, (K + 127) // 128)
    got = _run(x, None, G, (0, 0, 0), with_y=True, int8_grad_y=(q, s))
    U.compare_fmt(got[:4], oracle.silu_dot_fwd_bwd_quant_fuse_qgrad(x, q, s, G, 0, 0, 0), 0, 0, 0,
                  f"int8 grad_y K={K} G={G}", G)
    U.compare_bf16(got[4], oracle.swiglu_bwd_bf16_dy(x, oracle.dequant_grad_y(q, s))[0], "y", f"K={K}")


def test_partial_channel_tile_host_entry_equals_device_entry():
    """sdq_fuse_host (chunked host-buffer path) gives the device path's bytes
    on a K with a partial channel tile."""
    import swiglu_backward_int8_b200 as sdq
    M, K = 700, 208
    x, gy = W.make_inputs(W.small_workload(M, K, seed=19))
    dev = [t.cpu() for t in sdq.run(U.to_device_bf16(x), U.to_device_bf16(gy))]
    xh = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16)
    gh = torch.from_numpy(gy.view(np.int16)).view(torch.bfloat16)
    outs = sdq.allocate_outputs(M, K, "cpu")
    ws = torch.empty(sdq.sdq_fuse_host_workspace_bytes(M, K, 256), dtype=torch.uint8, device="cuda")
    sdq.silu_dot_fwd_bwd_quant_fuse_host(xh, gh, *outs, workspace=ws, chunk_rows=256)
    for a, b in zip(outs, dev):
        assert torch.equal(a, b)

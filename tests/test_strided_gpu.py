"""The strided entry point on the GPU: inputs read through their own row
strides (x as a slice of a wider buffer, gate and up as separate arrays),
outputs written into padded rows.  The logical outputs must equal the
oracle's (tolerances: tests/gpu_util.py), and every padding byte must keep
the sentinel it was filled with.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests import gpu_util as U

pytestmark = pytest.mark.gpu


def _padded(rows, cols, ld, dtype, fill):
    buf = torch.full((rows, ld), fill, dtype=dtype, device="cuda")
    return buf, buf[:, :cols]


Y_SENTINEL = 0x7FC1   # a bf16 NaN the op never writes


def _run_strided(x_u16, gy_u16, G, fmt, pad, split, with_y=False):
    """Run sdq_fuse_strided with every array padded by `pad` (elements);
    returns numpy outputs like the format oracle (and, with_y, the optional
    bf16 y as a fifth array), after checking the pads."""
    import swiglu_backward_int8_b200 as sdq
    codes, scales, layout = fmt
    M, K = gy_u16.shape
    Mg = (M + G - 1) // G
    xd = U.to_device_bf16(x_u16)
    gyd = U.to_device_bf16(gy_u16)
    bf_pad = 8 * pad                                      # bf16 rows stay 16-byte aligned
    if split:   # gate and up in two separate padded buffers
        gbuf, gate = _padded(M, K, K + bf_pad, torch.bfloat16, 0.0)
        ubuf, up = _padded(M, K, K + bf_pad, torch.bfloat16, 0.0)
        gate.copy_(xd[:, :K])
        up.copy_(xd[:, K:])
        g_ptr, ld_g, u_ptr, ld_u = gate.data_ptr(), gbuf.stride(0), up.data_ptr(), ubuf.stride(0)
    else:       # x = [gate | up] inside a wider buffer
        xbuf, xv = _padded(M, 2 * K, 2 * K + bf_pad, torch.bfloat16, 0.0)
        xv.copy_(xd)
        g_ptr, ld_g, u_ptr, ld_u = xv.data_ptr(), xbuf.stride(0), xv.data_ptr() + 2 * K, xbuf.stride(0)
    ybuf, gyv = _padded(M, K, K + bf_pad, torch.bfloat16, 0.0)
    gyv.copy_(gyd)
    sq = U.SENTINEL_CODE[codes]
    sdt, sfill = (torch.uint8, U.SENTINEL_E8M0) if scales else (torch.float32, float("nan"))
    ys_shape = (Mg, K) if layout else (K, Mg)
    q = _padded(M, 2 * K, 2 * K + 16 * pad, torch.uint8, sq)
    s = _padded(M, 2 * K // G, 2 * K // G + pad, sdt, sfill)
    yq = _padded(K, M, M + 13 * pad, torch.uint8, sq)     # often not a multiple of 16: byte stores
    ys = _padded(ys_shape[0], ys_shape[1], ys_shape[1] + pad, sdt, sfill)
    bits = (sdq.FMT_E4M3 if codes else 0) | (sdq.FMT_E8M0 if scales else 0) | (sdq.FMT_YS_MG_K if layout else 0)
    yo = None
    if with_y:   # bf16 y rows padded by 8 * pad elements, filled with a NaN sentinel
        yo = _padded(M, K, K + bf_pad, torch.int16, Y_SENTINEL)
    sdq.sdq_fuse_strided(g_ptr, ld_g, u_ptr, ld_u, gyv.data_ptr(), ybuf.stride(0),
                         q[1].data_ptr(), q[0].stride(0), s[1].data_ptr(), s[0].stride(0),
                         yq[1].data_ptr(), yq[0].stride(0), ys[1].data_ptr(), ys[0].stride(0),
                         yo[1].data_ptr() if with_y else None, yo[0].stride(0) if with_y else 0,
                         M, K, G, bits, torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert sdq.sdq_device_status() == 0
    out = []
    for (buf, view), cols, name in ((q, 2 * K, "grad_input_q"), (s, 2 * K // G, "grad_input_s"),
                                    (yq, M, "y_q_t"), (ys, ys_shape[1], "y_s_t")):
        pad_region = buf[:, cols:].cpu().numpy()
        if buf.dtype == torch.float32:
            assert np.isnan(pad_region).all(), f"{name}: padding written"
        else:
            want = sq if name in ("grad_input_q", "y_q_t") else U.SENTINEL_E8M0
            assert (pad_region == want).all(), f"{name}: padding written"
        out.append(view.cpu().numpy())
    if with_y:
        buf = yo[0].cpu().numpy().view(np.uint16)
        assert (buf[:, K:] == Y_SENTINEL).all(), "y: padding written"
        out.append(buf[:, :K].copy())
    return tuple(out)


@pytest.mark.parametrize("split", [False, True])
@pytest.mark.parametrize("G,fmt", [(128, (0, 0, 0)), (128, (1, 1, 1)), (64, (0, 1, 0)), (32, (1, 0, 1))])
@pytest.mark.parametrize("M,K", [(1000, 256), (129, 384), (4096, 1408)])
def test_strided_arrays_match_the_oracle(M, K, G, fmt, split):
    w = W.small_workload(M, K, seed=M + K + G) if M != 4096 else W.WORKLOADS[1]
    x, gy = W.make_inputs(w)
    got = _run_strided(x, gy, G, fmt, pad=3, split=split)
    ref = oracle.silu_dot_fwd_bwd_quant_fuse_fmt(x, gy, G, *fmt)
    U.compare_fmt(got, ref, *fmt, f"strided M={M} K={K}", G)


def test_strided_equals_packed_bit_for_bit():
    """The same inputs through padded, split arrays and through the packed
    entry point give identical bytes."""
    import swiglu_backward_int8_b200 as sdq
    w = W.small_workload(515, 384, seed=9)
    x, gy = W.make_inputs(w)
    a = _run_strided(x, gy, 128, (0, 0, 0), pad=5, split=True)
    b = U.run_cuda(x, gy)
    assert np.array_equal(a[0].view(np.int8), b[0]) and np.array_equal(a[2].view(np.int8), b[2])
    assert np.array_equal(a[1], b[1]) and np.array_equal(a[3], b[3])
    del sdq


def test_torch_views_of_wider_buffers():
    """The Python wrapper passes each tensor's row stride: views into wider
    buffers and the split-gate/up form give the packed result."""
    import swiglu_backward_int8_b200 as sdq
    w = W.small_workload(300, 256, seed=12)
    x, gy = W.make_inputs(w)
    xd, gyd = U.to_device_bf16(x), U.to_device_bf16(gy)
    ref = [t.cpu() for t in sdq.run(xd, gyd)]
    wide = torch.zeros(300, 2 * 256 + 64, dtype=torch.bfloat16, device="cuda")
    wide[:, :512] = xd
    outs_buf = [torch.zeros(300, 512 + 32, dtype=torch.int8, device="cuda"),
                torch.zeros(300, 4 + 4, dtype=torch.float32, device="cuda"),
                torch.zeros(256, 300 + 20, dtype=torch.int8, device="cuda"),
                torch.zeros(256, 3 + 1, dtype=torch.float32, device="cuda")]
    outs = [outs_buf[0][:, :512], outs_buf[1][:, :4], outs_buf[2][:, :300], outs_buf[3][:, :3]]
    sdq.silu_dot_fwd_bwd_quant_fuse(wide[:, :512], gyd, *outs)
    for a, b in zip(outs, ref):
        assert torch.equal(a.cpu(), b)
    outs2 = sdq.allocate_outputs(300, 256, "cuda")
    sdq.silu_dot_fwd_bwd_quant_fuse_split(xd[:, :256].clone(), xd[:, 256:].clone(), gyd, *outs2)
    for a, b in zip(outs2, ref):
        assert torch.equal(a.cpu(), b)


@pytest.mark.parametrize("G,fmt", [(128, (0, 0, 0)), (64, (1, 1, 1)), (32, (0, 1, 0))])
@pytest.mark.parametrize("M,K,split", [(1000, 256, False), (129, 384, True), (4096, 1408, False)])
def test_optional_y_output(M, K, G, fmt, split):
    """The optional bf16 y: within one bf16 step of the oracle's first-stage y
    (the values y_q_t quantizes), padding untouched, and the four quantized
    outputs bit-identical to the same call without it."""
    w = W.small_workload(M, K, seed=M + 3 * K + G) if M != 4096 else W.WORKLOADS[1]
    x, gy = W.make_inputs(w)
    with_y = _run_strided(x, gy, G, fmt, pad=2, split=split, with_y=True)
    without = _run_strided(x, gy, G, fmt, pad=2, split=split)
    for a, b in zip(with_y[:4], without):
        assert np.array_equal(a, b, equal_nan=True)
    U.compare_bf16(with_y[4], oracle.swiglu_bwd_bf16(x, gy)[0], "y", f"M={M} K={K} G={G}")


def test_optional_y_through_the_wrapper():
    """``y=`` on the Python op (packed and split forms, y a view into a wider
    buffer) gives the same y as the raw entry point and leaves the rest alone."""
    import swiglu_backward_int8_b200 as sdq
    w = W.small_workload(300, 256, seed=31)
    x, gy = W.make_inputs(w)
    xd, gyd = U.to_device_bf16(x), U.to_device_bf16(gy)
    ref = [t.cpu() for t in sdq.run(xd, gyd)]
    raw = _run_strided(x, gy, 128, (0, 0, 0), pad=1, split=False, with_y=True)[4]
    ybuf = torch.zeros(300, 256 + 8, dtype=torch.bfloat16, device="cuda")
    outs = sdq.allocate_outputs(300, 256, "cuda")
    sdq.silu_dot_fwd_bwd_quant_fuse(xd, gyd, *outs, y=ybuf[:, :256])
    for a, b in zip(outs, ref):
        assert torch.equal(a.cpu(), b)
    got = ybuf[:, :256].cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, raw)
    assert (ybuf[:, 256:] == 0).all()
    y2 = torch.empty(300, 256, dtype=torch.bfloat16, device="cuda")
    sdq.silu_dot_fwd_bwd_quant_fuse_split(xd[:, :256].clone(), xd[:, 256:].clone(), gyd,
                                          *sdq.allocate_outputs(300, 256, "cuda"), y=y2)
    assert np.array_equal(y2.cpu().view(torch.int16).numpy().view(np.uint16), raw)
    with pytest.raises(ValueError):   # y must be bf16 [M, K]
        sdq.silu_dot_fwd_bwd_quant_fuse(xd, gyd, *outs, y=torch.empty(300, 256, device="cuda"))

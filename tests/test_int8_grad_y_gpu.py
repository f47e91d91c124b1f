"""grad_y handed over already quantized (INT8 codes [M, K], fp32 scales
[M, K/128]) on the GPU: the outputs must equal the oracle's within the
tolerances of tests/gpu_util.py; with power-of-two scales (every q * s then
a bf16 value, and its fp32 product exact) they must equal, bit for bit, the
kernel's own outputs on that bf16 grad_y; padded rows stay untouched.
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


def _run_int8_grad_y(x_u16, q, s, G, fmt, pad=0, with_y=False):
    """sdq_fuse_int8_grad_y with every array's rows padded by `pad` units;
    returns numpy outputs like the format oracle (plus y with_y), after
    checking that no padding byte changed."""
    import swiglu_backward_int8_b200 as sdq
    codes, scales, layout = fmt
    M, K = q.shape
    Kg, Mg = K // 128, (M + G - 1) // G
    xbuf, xv = _padded(M, 2 * K, 2 * K + 8 * pad, torch.bfloat16, 0.0)
    xv.copy_(U.to_device_bf16(x_u16))
    qbuf, qv = _padded(M, K, K + 16 * pad, torch.int8, 0)
    qv.copy_(torch.from_numpy(q))
    sbuf, sv = _padded(M, Kg, Kg + pad, torch.float32, 0.0)
    sv.copy_(torch.from_numpy(s))
    sq = U.SENTINEL_CODE[codes]
    sdt, sfill = (torch.uint8, U.SENTINEL_E8M0) if scales else (torch.float32, float("nan"))
    ys_shape = (Mg, K) if layout else (K, Mg)
    outs = [_padded(M, 2 * K, 2 * K + 16 * pad, torch.uint8, sq),
            _padded(M, 2 * K // G, 2 * K // G + pad, sdt, sfill),
            _padded(K, M, M + 16 * pad, torch.uint8, sq),
            _padded(ys_shape[0], ys_shape[1], ys_shape[1] + pad, sdt, sfill)]
    yo = _padded(M, K, K + 8 * pad, torch.int16, 0x7FC1) if with_y else None
    bits = (sdq.FMT_E4M3 if codes else 0) | (sdq.FMT_E8M0 if scales else 0) | \
        (sdq.FMT_YS_MG_K if layout else 0)
    sdq.sdq_fuse_int8_grad_y(xv.data_ptr(), xbuf.stride(0), xv.data_ptr() + 2 * K, xbuf.stride(0),
                             qv.data_ptr(), qbuf.stride(0), sv.data_ptr(), sbuf.stride(0),
                             *(v for b, t in outs for v in (t.data_ptr(), b.stride(0))),
                             yo[1].data_ptr() if with_y else None, yo[0].stride(0) if with_y else 0,
                             M, K, G, bits, torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert sdq.sdq_device_status() == 0
    got = []
    for (buf, view), name in zip(outs, ("grad_input_q", "grad_input_s", "y_q_t", "y_s_t")):
        pad_region = buf[:, view.shape[1]:].cpu().numpy()
        if buf.dtype == torch.float32:
            assert np.isnan(pad_region).all(), f"{name}: padding written"
        else:
            want = sq if name in ("grad_input_q", "y_q_t") else U.SENTINEL_E8M0
            assert (pad_region == want).all(), f"{name}: padding written"
        got.append(view.cpu().numpy())
    if with_y:
        buf = yo[0].cpu().numpy().view(np.uint16)
        assert (buf[:, K:] == 0x7FC1).all(), "y: padding written"
        got.append(buf[:, :K].copy())
    return tuple(got)


@pytest.mark.parametrize("G,fmt", [(128, (0, 0, 0)), (128, (1, 1, 1)), (64, (0, 1, 0)), (32, (1, 0, 1))])
@pytest.mark.parametrize("M,K,pad", [(1000, 256, 0), (129, 384, 2), (4096, 1408, 1)])
def test_int8_grad_y_matches_the_oracle(M, K, pad, G, fmt):
    w = W.small_workload(M, K, seed=M + 5 * K + G, zero_group_every=33)
    x, _ = W.make_inputs(w)
    q, s = W.quantized_grad_y(w)
    got = _run_int8_grad_y(x, q, s, G, fmt, pad=pad)
    ref = oracle.silu_dot_fwd_bwd_quant_fuse_qgrad(x, q, s, G, *fmt)
    U.compare_fmt(got, ref, *fmt, f"int8 grad_y M={M} K={K}", G)


@pytest.mark.parametrize("G,fmt", [(128, (0, 0, 0)), (64, (1, 1, 1))])
def test_pow2_scales_equal_the_bf16_path_bit_for_bit(G, fmt):
    M, K = 515, 512
    w = W.small_workload(M, K, seed=17, zero_group_every=9)
    x, _ = W.make_inputs(w)
    q, s = W.quantized_grad_y(w, pow2_scales=True)
    v = (q.astype(np.float32) * np.repeat(s, 128, axis=1)).view(np.uint32)
    assert not (v & 0xFFFF).any()
    gy = (v >> 16).astype(np.uint16)
    a = _run_int8_grad_y(x, q, s, G, fmt, pad=1, with_y=True)
    b = U.run_cuda_fmt(x, gy, *fmt, group_size=G)
    for u, t, name in zip(a[:4], b, ("grad_input_q", "grad_input_s", "y_q_t", "y_s_t")):
        assert np.array_equal(u, t, equal_nan=True), name
    U.compare_bf16(a[4], oracle.swiglu_bwd_bf16(x, gy)[0], "y")


def test_wrapper_takes_int8_grad_y():
    """``grad_y_s=`` on the Python op (packed and split forms) gives the raw
    entry point's bytes; a bf16 grad_y with scales, or scales of the wrong
    shape, are refused."""
    import swiglu_backward_int8_b200 as sdq
    M, K = 300, 256
    w = W.small_workload(M, K, seed=23)
    x, _ = W.make_inputs(w)
    q, s = W.quantized_grad_y(w)
    raw = _run_int8_grad_y(x, q, s, 128, (0, 0, 0))
    xd = U.to_device_bf16(x)
    qd, sd = torch.from_numpy(q).cuda(), torch.from_numpy(s).cuda()
    outs = sdq.allocate_outputs(M, K, "cuda")
    sdq.silu_dot_fwd_bwd_quant_fuse(xd, qd, *outs, grad_y_s=sd)
    for a, b in zip(outs, raw):
        assert np.array_equal(a.cpu().numpy().view(b.dtype), b, equal_nan=True)
    outs2 = sdq.allocate_outputs(M, K, "cuda")
    sdq.silu_dot_fwd_bwd_quant_fuse_split(xd[:, :K].clone(), xd[:, K:].clone(), qd, *outs2, grad_y_s=sd)
    for a, b in zip(outs2, raw):
        assert np.array_equal(a.cpu().numpy().view(b.dtype), b, equal_nan=True)
    with pytest.raises(ValueError):
        sdq.silu_dot_fwd_bwd_quant_fuse(xd, qd.to(torch.bfloat16), *outs, grad_y_s=sd)
    with pytest.raises(ValueError):
        sdq.silu_dot_fwd_bwd_quant_fuse(xd, qd, *outs, grad_y_s=sd[:, :1])


@pytest.mark.slow
def test_int8_grad_y_full_size_sampled_tiles():
    """M=16384, K=7168 in one launch with grad_y as INT8 codes + scales and the
    bf16 y written too: 24 sampled 128x128 tiles against the oracle on each
    tile (every group lies inside one tile, and so does each row's scale of
    the tile's 128 grad_y channels); y on the same tiles."""
    import swiglu_backward_int8_b200 as sdq
    w = W.WORKLOADS[4]
    M, K = w.M, w.K
    x, _ = W.make_inputs(w)
    q, s = W.quantized_grad_y(w)
    outs = sdq.allocate_outputs(M, K, "cuda")
    y = torch.empty(M, K, dtype=torch.bfloat16, device="cuda")
    sdq.silu_dot_fwd_bwd_quant_fuse(U.to_device_bf16(x), torch.from_numpy(q).cuda(), *outs, y=y,
                                    grad_y_s=torch.from_numpy(s).cuda())
    torch.cuda.synchronize()
    assert sdq.sdq_device_status() == 0
    giq, gis, yqt, yst = (t.cpu().numpy() for t in outs)
    yh = y.view(torch.int16).cpu().numpy().view(np.uint16)
    rng = np.random.default_rng(11)
    tiles = {(0, 0), (M // 128 - 1, K // 128 - 1)}
    while len(tiles) < 24:
        tiles.add((int(rng.integers(M // 128)), int(rng.integers(K // 128))))
    n_diff = 0
    for i, j in sorted(tiles):
        r0, c0 = 128 * i, 128 * j
        xt = np.concatenate([x[r0:r0 + 128, c0:c0 + 128], x[r0:r0 + 128, K + c0:K + c0 + 128]], axis=1)
        qt, st_ = q[r0:r0 + 128, c0:c0 + 128], s[r0:r0 + 128, j:j + 1]
        ref = oracle.silu_dot_fwd_bwd_quant_fuse_qgrad(xt, qt, st_, 128, 0, 0, 0)
        got = (np.concatenate([giq[r0:r0 + 128, c0:c0 + 128], giq[r0:r0 + 128, K + c0:K + c0 + 128]],
                              axis=1).view(np.uint8),
               np.stack([gis[r0:r0 + 128, j], gis[r0:r0 + 128, K // 128 + j]], axis=1),
               yqt[c0:c0 + 128, r0:r0 + 128].view(np.uint8), yst[c0:c0 + 128, i:i + 1])
        st = U.compare_fmt(got, ref, 0, 0, 0, f"M16384 INT8 grad_y tile ({i},{j})", 128,
                           max_frac=1.0)                 # the 0.1 % bound applies to the whole sample
        n_diff += st["grad_input_q"]["n_diff"] + st["y_q_t"]["n_diff"]
        ry = oracle.swiglu_bwd_bf16_dy(xt, oracle.dequant_grad_y(qt, st_))[0]
        U.compare_bf16(yh[r0:r0 + 128, c0:c0 + 128], ry, "y", f"tile ({i},{j})")
    total = 24 * 128 * 128 * 3
    assert n_diff <= 1e-3 * total, f"{n_diff} of {total} sampled codes differ"


@pytest.mark.parametrize("G,fmt", [(128, (0, 0, 0)), (64, (1, 0, 1)), (32, (0, 1, 0))])
@pytest.mark.parametrize("M,K", [(1, 128), (31, 128), (127, 256), (257, 128), (640, 640)])
def test_int8_grad_y_odd_shapes_with_y(M, K, G, fmt):
    """Tail token groups of 1..127 tokens, M % 16 != 0 (byte-wise y_q_t
    stores), one channel tile, both variants at once (INT8 grad_y and the
    y output) at three group sizes: outputs against the oracle, y against
    the oracle's first stage."""
    w = W.small_workload(M, K, seed=3 * M + K, zero_group_every=5)
    x, _ = W.make_inputs(w)
    q, s = W.quantized_grad_y(w)
    got = _run_int8_grad_y(x, q, s, G, fmt, pad=1, with_y=True)
    ref = oracle.silu_dot_fwd_bwd_quant_fuse_qgrad(x, q, s, G, *fmt)
    U.compare_fmt(got[:4], ref, *fmt, f"int8 grad_y M={M} K={K} G={G}", G)
    U.compare_bf16(got[4], oracle.swiglu_bwd_bf16_dy(x, oracle.dequant_grad_y(q, s))[0], "y",
                   f"M={M} K={K}")

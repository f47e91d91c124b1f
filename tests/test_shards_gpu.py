"""Token-range shards on one GPU: the op run as several calls, each on a
range of whole token groups, writing into ONE global set of outputs through
the strided entry point, gives the bytes of the single call over all tokens.

This is the layout a data-parallel split of one batch uses: rank r owns
tokens [m0, m1) (swiglu_backward_int8_b200.parallel.shard_rows), writes its
rows of grad_input_q/_s and its columns [m0, m1) of y_q_t and
[m0/G, ceil(m1/G)) of y_s_t, with the global leading dimensions.  Row groups
lie inside a token and column groups inside one token group, so no shard
needs another's data ("kernelgen-challenge-9-task3-silu-quant", outputs
section: row-wise channel groups, transposed token-group quantization).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from swiglu_backward_int8_b200 import parallel
from tests import gpu_util as U

pytestmark = pytest.mark.gpu


def _outputs(M, K, G, fmt):
    codes, scales, layout = fmt
    Kgs, Mg = (K + G - 1) // G, (M + G - 1) // G
    sdt, sfill = (torch.uint8, U.SENTINEL_E8M0) if scales else (torch.float32, float("nan"))
    sq = U.SENTINEL_CODE[codes]
    return [torch.full((M, 2 * K), sq, dtype=torch.uint8, device="cuda"),
            torch.full((M, 2 * Kgs), sfill, dtype=sdt, device="cuda"),
            torch.full((K, M), sq, dtype=torch.uint8, device="cuda"),
            torch.full((Mg, K) if layout else (K, Mg), sfill, dtype=sdt, device="cuda")]


def _call(xd, gyd, outs, m0, m1, K, G, fmt):
    """One call on tokens [m0, m1) into the global outputs."""
    import swiglu_backward_int8_b200 as sdq
    codes, scales, layout = fmt
    giq, gis, yqt, yst = outs
    i0, _ = parallel.group_range(m0, m1, G)
    bits = (sdq.FMT_E4M3 if codes else 0) | (sdq.FMT_E8M0 if scales else 0) | \
        (sdq.FMT_YS_MG_K if layout else 0)
    ss = gis.element_size()
    gate = xd.data_ptr() + m0 * xd.stride(0) * 2
    yst_ptr = yst.data_ptr() + (i0 * yst.stride(0) if layout else i0) * ss
    sdq.sdq_fuse_strided(gate, xd.stride(0), gate + 2 * K, xd.stride(0),
                         gyd.data_ptr() + m0 * gyd.stride(0) * 2, gyd.stride(0),
                         giq.data_ptr() + m0 * giq.stride(0), giq.stride(0),
                         gis.data_ptr() + m0 * gis.stride(0) * ss, gis.stride(0),
                         yqt.data_ptr() + m0, yqt.stride(0),
                         yst_ptr, yst.stride(0),
                         None, 0, m1 - m0, K, G, bits, torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("M,K,G,fmt,world", [
    (1000, 256, 128, (0, 0, 0), 2),     # tail group of 104 tokens in the last shard
    (1000, 256, 128, (0, 0, 0), 3),
    (4096, 1408, 128, (0, 0, 0), 4),
    (300, 208, 128, (0, 0, 1), 2),      # a partial channel tile; y_s_t [Mg, K]
    (777, 384, 64, (1, 1, 0), 3),       # E4M3 codes, E8M0 scales, shards of 64-token groups
    (250, 128, 32, (0, 1, 1), 4),
    (130, 128, 128, (0, 0, 0), 4),      # more ranks than token groups: empty shards
])
def test_shards_write_the_single_call_bytes(M, K, G, fmt, world):
    import swiglu_backward_int8_b200 as sdq
    x, gy = W.make_inputs(W.small_workload(M, K, seed=M + K + world))
    xd, gyd = U.to_device_bf16(x), U.to_device_bf16(gy)
    whole = _outputs(M, K, G, fmt)
    _call(xd, gyd, whole, 0, M, K, G, fmt)
    sharded = _outputs(M, K, G, fmt)
    covered = 0
    for r in range(world):
        m0, m1 = parallel.shard_rows(M, world, r, G)
        assert m0 == covered
        covered = m1
        if m1 > m0:
            _call(xd, gyd, sharded, m0, m1, K, G, fmt)
    assert covered == M
    torch.cuda.synchronize()
    assert sdq.sdq_device_status() == 0
    for a, b, name in zip(whole, sharded, ("grad_input_q", "grad_input_s", "y_q_t", "y_s_t")):
        assert torch.equal(a.view(torch.uint8) if a.dtype != torch.float32 else a.view(torch.int32),
                           b.view(torch.uint8) if b.dtype != torch.float32 else b.view(torch.int32)), name
    got = [t.cpu().numpy() for t in sharded]
    ref = oracle.silu_dot_fwd_bwd_quant_fuse_fmt(x, gy, G, *fmt)
    U.compare_fmt(got, ref, *fmt, f"M={M} K={K} G={G} world={world}", G)

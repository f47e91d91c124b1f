"""The host-buffer entry point that allocates nothing (sdq_fuse_host_noalloc).

It serves callers that cannot allocate device memory -- a host-only C/C++
program with no device allocator, a plugin inside a framework whose caching
allocator owns the GPU's memory, a service that forbids allocation after
start-up -- and so cannot hand sdq_fuse_host its workspace.  It stages through
a fixed array inside the library instead.

This file is collected last on purpose: if it fails, a run that stops at the
first failure has already run every other test.
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads as W
from tests import gpu_util as U


def _host(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


@pytest.mark.gpu
def test_noalloc_matches_existing_entry_on_two_calls_in_a_row():
    import swiglu_backward_int8_b200 as sdq
    # Two different problems back to back: the second must not see the first's
    # leftovers in the shared array.  The first spans two chunks (2560 + 440
    # rows at K=1408, the second ending in a partial token group).  Each result
    # is compared with the existing device entry point and with the oracle.
    cases = [W.small_workload(3000, 1408, seed=101), W.small_workload(777, 384, seed=102)]
    for w in cases:
        x, gy = W.make_inputs(w)
        want = U.run_cuda(x, gy)                 # the existing device entry point
        outs = [t.pin_memory() for t in sdq.allocate_outputs(w.M, w.K, "cpu")]
        for t in outs:
            t.fill_(-128 if t.dtype == torch.int8 else float("nan"))
        xh, gyh = _host(x).pin_memory(), _host(gy).pin_memory()
        stream = torch.cuda.current_stream()
        # straight through the C ABI (ctypes), no torch allocation involved
        sdq.sdq_fuse_host_noalloc(xh.data_ptr(), gyh.data_ptr(), *(t.data_ptr() for t in outs),
                                  w.M, w.K, 128, stream.cuda_stream)
        stream.synchronize()
        got = [t.numpy() for t in outs]
        U.compare(got, want, f"noalloc {w.name}")
        U.compare(got, oracle.silu_dot_fwd_bwd_quant_fuse(x, gy), f"noalloc {w.name} vs oracle")
        assert not (got[0] == -128).any() and not (got[2] == -128).any()
        assert np.isfinite(got[1]).all() and np.isfinite(got[3]).all()


@pytest.mark.gpu
def test_noalloc_with_pageable_host_buffers():
    """Pageable (not page-locked) host buffers: the copies are then staged by
    the CUDA runtime and block the host, but the bytes are the same."""
    import swiglu_backward_int8_b200 as sdq
    w = W.small_workload(1000, 208, seed=103)    # a partial channel tile and a tail token group
    x, gy = W.make_inputs(w)
    want = U.run_cuda(x, gy)
    outs = [t.fill_(-128 if t.dtype == torch.int8 else float("nan"))
            for t in sdq.allocate_outputs(w.M, w.K, "cpu")]
    xh, gyh = _host(x), _host(gy)
    stream = torch.cuda.current_stream()
    sdq.sdq_fuse_host_noalloc(xh.data_ptr(), gyh.data_ptr(), *(t.data_ptr() for t in outs),
                              w.M, w.K, 128, stream.cuda_stream)
    stream.synchronize()
    for a, b in zip(want, outs):
        assert np.array_equal(a, b.numpy())


def test_noalloc_rejects_k_beyond_its_scratch():
    # Answered before any CUDA call, so this needs no GPU.
    import swiglu_backward_int8_b200 as sdq
    A = 1 << 20
    with pytest.raises(sdq.SdqError) as ei:
        sdq.sdq_fuse_host_noalloc(A, A, A, A, A, A, 256, 28800 + 128, 128)
    assert ei.value.status == sdq.Status.ERR_TOO_LARGE
    with pytest.raises(sdq.SdqError) as ei:
        sdq.sdq_fuse_host_noalloc(A, A, A, A, A, A, 256, 200, 128)
    assert ei.value.status == sdq.Status.ERR_SHAPE

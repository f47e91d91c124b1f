"""The C ABI library: builds, loads, exports every symbol include/sdq.h
declares, and its host-side validation answers without a GPU (no compute
calls here)."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sdq.h")


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sdq_[a-z0-9_]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    import __graft_entry__
    path = __graft_entry__._build_module().build()
    return ctypes.CDLL(path)


def test_header_declares_the_entry_points():
    names = _declared_functions()
    for must in ("sdq_fuse", "sdq_validate", "sdq_fuse_host", "sdq_fuse_host_workspace_bytes",
                 "sdq_device_status", "sdq_status_string", "sdq_last_cuda_error", "sdq_version"):
        assert must in names


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in _declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_python_binding_loads():
    import swiglu_backward_int8_b200 as sdq
    assert sdq.version() == "0.1.0"
    assert sdq.status_string(0) == "SDQ_OK"
    assert "group_size" in sdq.status_string(2)


A = 1 << 20  # a 16-byte-aligned fake address: validation never dereferences


@pytest.mark.parametrize("args,status", [
    (dict(), 0),
    (dict(group_size=64), 0),
    (dict(group_size=32), 0),
    (dict(group_size=96), 2),
    (dict(group_size=256), 0),            # 256 x 256 units
    (dict(group_size=512), 2),
    (dict(group_size=64, K=192), 0),      # a shorter last channel tile
    (dict(K=144), 0),                     # 128 + 16: the last channel group holds 16
    (dict(K=16), 0),
    (dict(K=136), 3),                     # K must be a multiple of 16
    (dict(K=100), 3),
    (dict(K=0), 3),
    (dict(M=-1), 3),
    (dict(K=1 << 21), 3),
    (dict(x=0), 1),
    (dict(y_s_t=0), 1),
    (dict(x=A + 2), 4),
    (dict(y_q_t=A + 8), 4),
    (dict(grad_input_s=A + 2), 4),
    (dict(grad_input_s=A + 4), 0),
    (dict(M=0, x=0, grad_y=0), 0),
])
def test_validation_statuses(args, status):
    import swiglu_backward_int8_b200 as sdq
    a = dict(x=A, grad_y=A, grad_input_q=A, grad_input_s=A, y_q_t=A, y_s_t=A, M=256, K=256,
             group_size=128)
    a.update(args)
    assert sdq.sdq_validate(a["x"], a["grad_y"], a["grad_input_q"], a["grad_input_s"], a["y_q_t"],
                            a["y_s_t"], a["M"], a["K"], a["group_size"]) == status


def test_fuse_rejects_before_any_cuda_call():
    # Invalid arguments return their status without touching CUDA (works on a
    # machine with no GPU).
    import swiglu_backward_int8_b200 as sdq
    with pytest.raises(sdq.SdqError) as ei:
        sdq.sdq_fuse(A, A, A, A, A, A, 256, 200, 128)
    assert ei.value.status == sdq.Status.ERR_SHAPE
    with pytest.raises(sdq.SdqError) as ei:
        sdq.sdq_fuse(A, A, A, A, A, A, 256, 256, 16)
    assert ei.value.status == sdq.Status.ERR_GROUP
    sdq.sdq_fuse(0, 0, 0, 0, 0, 0, 0, 256, 128)  # M == 0: nothing to do


def test_host_workspace_sizes():
    import swiglu_backward_int8_b200 as sdq
    assert sdq.sdq_fuse_host_workspace_bytes(4096, 1408, 0) > 0
    assert sdq.sdq_fuse_host_workspace_bytes(4096, 100, 0) == 0
    assert sdq.sdq_fuse_host_workspace_bytes(4096, 1408, 100) == 0
    b128 = sdq.sdq_fuse_host_workspace_bytes(4096, 1408, 128)
    b256 = sdq.sdq_fuse_host_workspace_bytes(4096, 1408, 256)
    # two buffer sets of chunk_rows * (6K input + 3K output bytes + scales)
    assert b128 >= 2 * 128 * 1408 * 9 and b256 >= 2 * b128 - 4096


def test_torch_wrapper_argument_checks():
    import torch
    import swiglu_backward_int8_b200 as sdq
    x = torch.zeros(8, 256, dtype=torch.bfloat16)
    gy = torch.zeros(8, 128, dtype=torch.bfloat16)
    outs = sdq.allocate_outputs(8, 128, "cpu")
    with pytest.raises(ValueError):   # host tensors are not accepted by the device entry
        sdq.silu_dot_fwd_bwd_quant_fuse(x, gy, *outs)
    with pytest.raises(ValueError):
        sdq.silu_dot_fwd_bwd_quant_fuse(x.float(), gy, *outs)
    with pytest.raises(ValueError):
        sdq.silu_dot_fwd_bwd_quant_fuse(x, gy[:, :64], *outs)


@pytest.mark.parametrize("fmt,args,status", [
    (0, dict(), 0),
    (7, dict(), 0),
    (8, dict(), 9),                        # unknown bit
    (1 << 31, dict(), 9),
    (2, dict(grad_input_s=A + 1, y_s_t=A + 3), 0),   # E8M0 scales are bytes: any alignment
    (0, dict(grad_input_s=A + 1), 4),
    (1, dict(y_s_t=A + 2), 4),             # E4M3 codes with fp32 scales: 4-byte scales
    (6, dict(grad_input_q=A + 1), 4),      # code arrays stay 16-byte aligned
    (3, dict(group_size=48), 2),
    (3, dict(group_size=32), 0),
    (5, dict(M=0, x=0), 0),
])
def test_validate_format_statuses(fmt, args, status):
    import swiglu_backward_int8_b200 as sdq
    a = dict(x=A, grad_y=A, grad_input_q=A, grad_input_s=A, y_q_t=A, y_s_t=A, M=256, K=256,
             group_size=128)
    a.update(args)
    assert sdq.sdq_validate_format(a["x"], a["grad_y"], a["grad_input_q"], a["grad_input_s"],
                                   a["y_q_t"], a["y_s_t"], a["M"], a["K"], a["group_size"],
                                   fmt) == status


def test_format_names_shapes_and_dtypes():
    import torch
    import swiglu_backward_int8_b200 as sdq
    assert sdq.output_format() == 0
    assert sdq.output_format("e4m3", "e8m0", "mg_k") == 7
    assert sdq.output_format(scales="e8m0") == sdq.FMT_E8M0
    with pytest.raises(ValueError):
        sdq.output_format("fp4")
    q, s, yq, ys = sdq.allocate_outputs(300, 256, "cpu", codes="e4m3", scales="e8m0",
                                        y_scale_layout="mg_k")
    assert q.dtype == torch.float8_e4m3fn and yq.dtype == torch.float8_e4m3fn
    assert s.dtype == torch.uint8 and ys.dtype == torch.uint8
    assert tuple(q.shape) == (300, 512) and tuple(s.shape) == (300, 4)
    assert tuple(yq.shape) == (256, 300) and tuple(ys.shape) == (3, 256)
    x = torch.zeros(300, 512, dtype=torch.bfloat16)
    gy = torch.zeros(300, 256, dtype=torch.bfloat16)
    with pytest.raises(ValueError):     # host tensors: the device entry refuses before any call
        sdq.silu_dot_fwd_bwd_quant_fuse(x, gy, q, s, yq, ys, y_scale_layout="mg_k")
    with pytest.raises(ValueError):     # [K, Mg] scales where [Mg, K] was asked for
        sdq.silu_dot_fwd_bwd_quant_fuse(x, gy, q, s, yq, ys.T.contiguous(), y_scale_layout="mg_k")
    with pytest.raises(ValueError):     # E4M3 codes with INT8 asked for
        sdq.silu_dot_fwd_bwd_quant_fuse(x, gy, q, s, yq, ys, codes="int8", y_scale_layout="mg_k")


def _strided_args(**kw):
    M, K = 256, 256
    a = dict(gate=A, ld_gate=2 * K, up=A + 2 * K, ld_up=2 * K, grad_y=A, ld_grad_y=K,
             grad_input_q=A, ld_grad_input_q=2 * K, grad_input_s=A, ld_grad_input_s=4,
             y_q_t=A, ld_y_q_t=M, y_s_t=A, ld_y_s_t=2, y=None, ld_y=0, M=M, K=K, group_size=128,
             format=0)
    a.update(kw)
    return a


@pytest.mark.parametrize("kw,status", [
    (dict(), 0),
    (dict(ld_gate=1024, ld_up=520, ld_grad_y=264, ld_grad_input_q=528, ld_grad_input_s=7,
          ld_y_q_t=259, ld_y_s_t=9), 0),                  # padded rows; y_q_t ld not a multiple of 16
    (dict(up=A + (1 << 20)), 0),                         # gate and up apart
    (dict(ld_gate=255), 10),                             # shorter than a row
    (dict(ld_grad_input_s=3), 10),
    (dict(ld_y_q_t=255), 10),
    (dict(ld_y_s_t=1), 10),
    (dict(format=4, ld_y_s_t=255), 10),                  # [Mg, K] layout needs ld >= K
    (dict(format=4, ld_y_s_t=256), 0),
    (dict(ld_gate=1 << 37), 10),                         # above SDQ_MAX_LD
    (dict(ld_grad_input_q=(1 << 24) + 16), 10),          # above SDQ_MAX_LD_ROWS
    (dict(ld_grad_input_s=(1 << 24) + 1), 10),
    (dict(ld_up=516), 4),                                # bf16 rows must start on 16 bytes
    (dict(ld_grad_input_q=520), 4),                      # grad_input_q rows on 16 bytes
    (dict(up=A + 8), 4),
    (dict(group_size=64, ld_grad_input_s=8, ld_y_s_t=4), 0),
    (dict(group_size=64, ld_grad_input_s=7), 10),
    (dict(M=0, gate=0, up=0), 0),
    (dict(up=0), 1),
    (dict(y=A, ld_y=256), 0),                            # the optional bf16 y
    (dict(y=A, ld_y=264), 0),
    (dict(y=A, ld_y=255), 10),                           # shorter than a row
    (dict(y=A, ld_y=(1 << 36) + 8), 10),                 # above SDQ_MAX_LD
    (dict(y=A, ld_y=260), 4),                            # rows must start on 16 bytes
    (dict(y=A + 8, ld_y=256), 4),
    (dict(y=None, ld_y=3), 0),                           # no y: its ld is not looked at
])
def test_validate_strided_statuses(kw, status):
    import swiglu_backward_int8_b200 as sdq
    a = _strided_args(**kw)
    assert sdq.sdq_validate_strided(*a.values()) == status


def test_wrapper_takes_row_strides_and_refuses_other_layouts():
    import torch
    import swiglu_backward_int8_b200 as sdq
    from swiglu_backward_int8_b200 import _rows
    wide = torch.zeros(8, 600, dtype=torch.bfloat16)
    assert _rows("x", wide, (8, 600), (torch.bfloat16,), False, None) == 600
    with pytest.raises(ValueError):          # transposed: rows are not unit-stride
        _rows("x", torch.zeros(512, 8, dtype=torch.bfloat16).t(), (8, 512), (torch.bfloat16,), True,
              torch.device("cpu"))
    with pytest.raises(ValueError):          # expanded: rows overlap
        _rows("x", torch.zeros(1, 512, dtype=torch.bfloat16).expand(8, 512), (8, 512),
              (torch.bfloat16,), True, torch.device("cpu"))
    with pytest.raises(ValueError):          # the host entry points need contiguous tensors
        _rows("x", wide[:, :512], (8, 512), (torch.bfloat16,), False, torch.device("cpu"))


def test_fwd_rejects_bad_arguments_without_launching():
    import swiglu_backward_int8_b200 as sdq
    A = 1 << 20
    assert sdq.sdq_validate_swiglu_q8_1(A, 64, A, 64, None, A, 64, A, 4, 48) == sdq.Status.ERR_SHAPE
    assert sdq.sdq_validate_swiglu_q8_1(A, 60, A, 64, None, A, 64, A, 4, 64) == sdq.Status.ERR_STRIDE
    assert sdq.sdq_validate_swiglu_q8_1(A + 2, 64, A, 64, None, A, 64, A, 4, 64) == sdq.Status.ERR_ALIGN
    assert sdq.sdq_validate_swiglu_q8_1(A, 64, A, 64, None, A, 64, A + 2, 4, 64) == sdq.Status.ERR_ALIGN
    assert sdq.sdq_validate_swiglu_q8_1(0, 64, 0, 64, None, 0, 64, 0, 0, 64) == sdq.Status.OK


def _int8_gy_args(**kw):
    M, K = 256, 256
    a = dict(gate=A, ld_gate=2 * K, up=A + 2 * K, ld_up=2 * K, grad_y_q=A, ld_grad_y_q=K,
             grad_y_s=A, ld_grad_y_s=2, grad_input_q=A, ld_grad_input_q=2 * K, grad_input_s=A,
             ld_grad_input_s=4, y_q_t=A, ld_y_q_t=M, y_s_t=A, ld_y_s_t=2, y=None, ld_y=0, M=M, K=K,
             group_size=128, format=0)
    a.update(kw)
    return a


@pytest.mark.parametrize("kw,status", [
    (dict(), 0),
    (dict(ld_grad_y_q=272, ld_grad_y_s=5), 0),          # padded rows
    (dict(ld_grad_y_q=264), 4),                          # code rows must start on 16 bytes
    (dict(ld_grad_y_q=255), 10),
    (dict(grad_y_q=A + 8), 4),
    (dict(grad_y_s=None), 1),
    (dict(grad_y_q=None), 1),
    (dict(ld_grad_y_s=1), 10),                           # fewer than K/128 scales a row
    (dict(ld_grad_y_s=(1 << 36) + 1), 10),
    (dict(grad_y_s=A + 2), 4),                           # fp32 scales on 4 bytes
    (dict(grad_y_s=A + 4), 0),
    (dict(y=A, ld_y=256, format=7, ld_y_s_t=256), 0),    # with y, another format
    (dict(M=0, gate=None, up=None, grad_y_q=None, grad_y_s=None), 0),
    (dict(group_size=96), 2),
])
def test_validate_int8_grad_y_statuses(kw, status):
    import swiglu_backward_int8_b200 as sdq
    a = _int8_gy_args(**kw)
    assert sdq.sdq_validate_int8_grad_y(*a.values()) == status

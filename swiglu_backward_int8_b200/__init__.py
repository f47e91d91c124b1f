"""B200-native silu_dot_fwd_bwd_quant_fuse: fused SwiGLU forward recompute,
backward and dual-axis INT8 quantization ("kernelgen-challenge-9-task3-silu-quant",
entry point and outputs sections).

    silu_dot_fwd_bwd_quant_fuse(x, grad_y, grad_input_q, grad_input_s, y_q_t, y_s_t,
                                group_size=128)

takes CUDA tensors x = [gate | up] (bf16 [M, 2K]) and grad_y (bf16 [M, K]) and
writes, in place, grad_input_q (int8 [M, 2K]), grad_input_s (fp32 [M, 2 ceil(K/128)]),
y_q_t (int8 [K, M]) and y_s_t (fp32 [K, ceil(M/128)]).  PyTorch supplies only
the device memory and the current stream; the work runs in libsdq.so.

Other output formats (include/sdq.h, SDQ_FMT_*) follow from the output
tensors' dtypes: float8_e4m3fn codes (OCP FP8 E4M3), uint8 or float8_e8m0fnu
scales (E8M0 powers of two); ``y_scale_layout="mg_k"`` gives y_s_t as
[ceil(M/128), K].
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch

from ._lib import (FMT_E4M3, FMT_E8M0, FMT_YS_MG_K, LIB_PATH, SdqError, Status, last_cuda_error,
                   sdq_device_status, sdq_fuse, sdq_fuse_format, sdq_fuse_host,
                   sdq_fuse_host_noalloc, sdq_fuse_host_workspace_bytes, sdq_fuse_int8_grad_y,
                   sdq_fuse_strided, sdq_validate_int8_grad_y,
                   sdq_swiglu_q8_1, sdq_validate, sdq_validate_format, sdq_validate_strided,
                   sdq_validate_swiglu_q8_1, status_string, version)

__all__ = [
    "silu_dot_fwd_bwd_quant_fuse", "silu_dot_fwd_bwd_quant_fuse_split",
    "silu_dot_fwd_bwd_quant_fuse_host", "allocate_outputs", "sdq_fuse_strided", "sdq_validate_strided",
    "sdq_fuse_int8_grad_y", "sdq_validate_int8_grad_y",
    "swiglu_q8_1", "sdq_swiglu_q8_1", "sdq_validate_swiglu_q8_1", "Q8_1_BLOCK_BYTES",
    "output_shapes", "output_format", "sdq_fuse", "sdq_fuse_format", "sdq_validate_format",
    "FMT_E4M3", "FMT_E8M0", "FMT_YS_MG_K", "sdq_fuse_host", "sdq_fuse_host_noalloc",
    "sdq_fuse_host_workspace_bytes", "sdq_validate",
    "sdq_device_status", "SdqError", "Status", "status_string", "last_cuda_error", "version",
    "LIB_PATH", "GROUP_SIZE", "GROUP_SIZES", "K_MULTIPLE",
]

GROUP_SIZE = 128
GROUP_SIZES = (32, 64, 128, 256)   # 128 x 128 tiles hold whole groups of 32..128; 256: 256 x 256 units
K_MULTIPLE = 16               # K must be a multiple of this (a shorter last channel group otherwise)


_E8M0_DTYPES = tuple(d for d in (torch.uint8, getattr(torch, "float8_e8m0fnu", None)) if d is not None)
_CODE_DTYPES = {"int8": (torch.int8,), "e4m3": (torch.float8_e4m3fn, torch.uint8)}
_SCALE_DTYPES = {"fp32": (torch.float32,), "e8m0": _E8M0_DTYPES}
_LAYOUTS = ("k_mg", "mg_k")


def output_format(codes: str = "int8", scales: str = "fp32", y_scale_layout: str = "k_mg") -> int:
    """FMT_* bits for the named output format."""
    if codes not in _CODE_DTYPES or scales not in _SCALE_DTYPES or y_scale_layout not in _LAYOUTS:
        raise ValueError(f"unknown format codes={codes!r} scales={scales!r} "
                         f"y_scale_layout={y_scale_layout!r}")
    return ((FMT_E4M3 if codes == "e4m3" else 0) | (FMT_E8M0 if scales == "e8m0" else 0) |
            (FMT_YS_MG_K if y_scale_layout == "mg_k" else 0))


def output_shapes(M: int, K: int, group_size: int = GROUP_SIZE, y_scale_layout: str = "k_mg"):
    """Shapes of (grad_input_q, grad_input_s, y_q_t, y_s_t)."""
    G = group_size
    Mg = (M + G - 1) // G
    Kg = (K + G - 1) // G   # channel groups per half of [d_gate | d_up]; the last may be short
    return (M, 2 * K), (M, 2 * Kg), (K, M), ((Mg, K) if y_scale_layout == "mg_k" else (K, Mg))


def allocate_outputs(M: int, K: int, device, group_size: int = GROUP_SIZE, codes: str = "int8",
                     scales: str = "fp32", y_scale_layout: str = "k_mg"):
    """Uninitialised output tensors for one call (the op writes every element)."""
    output_format(codes, scales, y_scale_layout)
    s = output_shapes(M, K, group_size, y_scale_layout)
    cdt, sdt = _CODE_DTYPES[codes][0], _SCALE_DTYPES[scales][0]
    return (torch.empty(s[0], dtype=cdt, device=device),
            torch.empty(s[1], dtype=sdt, device=device),
            torch.empty(s[2], dtype=cdt, device=device),
            torch.empty(s[3], dtype=sdt, device=device))


def _infer(kind: str, given: Optional[str], t: torch.Tensor, table) -> str:
    if given is None:
        for name, dts in table.items():
            if t.dtype in dts:
                return name
        raise ValueError(f"cannot tell the {kind} format from dtype {t.dtype}; pass {kind}=...")
    if given not in table:
        raise ValueError(f"unknown {kind} format {given!r}")
    return given


def _rows(name: str, t: torch.Tensor, shape, dtypes, want_cuda: bool, device) -> int:
    """Check a 2-D row-major operand (rows may be padded: stride(0) >= its
    row); returns its leading dimension in elements."""
    if t.dim() != 2 or tuple(t.shape) != tuple(shape) or t.dtype not in dtypes:
        raise ValueError(f"{name}: expected {' or '.join(map(str, dtypes))} {tuple(shape)}, "
                         f"got {t.dtype} {tuple(t.shape)}")
    if t.shape[1] > 1 and t.stride(1) != 1:
        raise ValueError(f"{name} must have unit stride along its rows")
    if t.shape[0] > 1 and t.stride(0) < t.shape[1]:
        raise ValueError(f"{name}: rows overlap (stride {t.stride(0)} < row length {t.shape[1]})")
    if not want_cuda and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous for the host-buffer entry points")
    if want_cuda and (not t.is_cuda or t.device != device):
        raise ValueError(f"{name} must be a CUDA tensor on {device}")
    if not want_cuda and t.is_cuda:
        raise ValueError(f"{name} must be a host tensor")
    return int(t.stride(0)) if t.shape[0] > 1 else int(t.shape[1])


def _check_group(K: int, group_size: int, want_cuda: bool):
    if group_size not in GROUP_SIZES or K % K_MULTIPLE or K < 1:
        raise ValueError(f"group_size must be one of {GROUP_SIZES} and K={K} a positive multiple "
                         f"of {K_MULTIPLE}")
    if not want_cuda and group_size != GROUP_SIZE:
        raise ValueError("the host-buffer entry points take group_size 128 only")


def _check_outputs(M, K, outs, group_size, want_cuda, codes, scales, y_scale_layout, device):
    names = ("grad_input_q", "grad_input_s", "y_q_t", "y_s_t")
    dtypes = (_CODE_DTYPES[codes], _SCALE_DTYPES[scales]) * 2
    return [_rows(n, t, shp, dts, want_cuda, device)
            for n, t, shp, dts in zip(names, outs, output_shapes(M, K, group_size, y_scale_layout), dtypes)]


def _check_tensors(x, grad_y, outs, group_size, want_cuda: bool, codes="int8", scales="fp32",
                   y_scale_layout="k_mg", grad_y_s=None):
    if x.dim() != 2 or grad_y.dim() != 2:
        raise ValueError("x and grad_y must be 2-D")
    M, K2 = x.shape
    if K2 % 2:
        raise ValueError(f"x has an odd channel count {K2}; expected [gate | up]")
    K = K2 // 2
    _check_group(K, group_size, want_cuda)
    bf16 = (torch.bfloat16,)
    ld_x = _rows("x", x, (M, 2 * K), bf16, want_cuda, x.device)
    if grad_y_s is None:
        ld_gy, gys = _rows("grad_y", grad_y, (M, K), bf16, want_cuda, x.device), (None, 0)
    else:
        ld_gy, *gys = _grad_y(grad_y, grad_y_s, M, K, x.device)
    lds = _check_outputs(M, K, outs, group_size, want_cuda, codes, scales, y_scale_layout, x.device)
    return M, K, ld_x, ld_gy, lds, tuple(gys)


def _check_y(y, M, K, device):
    """The optional bf16 y output: (pointer or None, leading dimension)."""
    if y is None:
        return None, 0
    return y.data_ptr(), _rows("y", y, (M, K), (torch.bfloat16,), True, device)


def _grad_y(grad_y, grad_y_s, M, K, device):
    """grad_y in bf16 [M, K], or INT8 codes [M, K] with fp32 scales
    ``grad_y_s`` [M, ceil(K/128)]: (its leading dimension, the scales' pointer or
    None, their leading dimension)."""
    if grad_y_s is None:
        return _rows("grad_y", grad_y, (M, K), (torch.bfloat16,), True, device), None, 0
    ld_q = _rows("grad_y", grad_y, (M, K), (torch.int8,), True, device)
    ld_s = _rows("grad_y_s", grad_y_s, (M, (K + GROUP_SIZE - 1) // GROUP_SIZE), (torch.float32,), True,
                 device)
    return ld_q, grad_y_s.data_ptr(), ld_s


def _call_strided(gate, ld_gate, up, ld_up, grad_y, ld_gy, outs, lds, M, K, group_size, fmt, device,
                  y=None, gys=None, ld_gys=0):
    yp, ld_y = _check_y(y, M, K, device)
    with torch.cuda.device(device):
        stream = torch.cuda.current_stream(device).cuda_stream
        q, s, yq, ys = outs
        if gys is None:
            sdq_fuse_strided(gate, ld_gate, up, ld_up, grad_y.data_ptr(), ld_gy, q.data_ptr(),
                             lds[0], s.data_ptr(), lds[1], yq.data_ptr(), lds[2], ys.data_ptr(),
                             lds[3], yp, ld_y, M, K, group_size, fmt, stream)
        else:
            sdq_fuse_int8_grad_y(gate, ld_gate, up, ld_up, grad_y.data_ptr(), ld_gy, gys, ld_gys,
                                 q.data_ptr(), lds[0], s.data_ptr(), lds[1], yq.data_ptr(), lds[2],
                                 ys.data_ptr(), lds[3], yp, ld_y, M, K, group_size, fmt, stream)


def silu_dot_fwd_bwd_quant_fuse(x: torch.Tensor, grad_y: torch.Tensor, grad_input_q: torch.Tensor,
                                grad_input_s: torch.Tensor, y_q_t: torch.Tensor,
                                y_s_t: torch.Tensor, group_size: int = GROUP_SIZE, *,
                                codes: Optional[str] = None, scales: Optional[str] = None,
                                y_scale_layout: str = "k_mg", y: Optional[torch.Tensor] = None,
                                grad_y_s: Optional[torch.Tensor] = None) -> None:
    """Fused SwiGLU backward + dual-axis quantization, in place, on the
    current CUDA stream of x's device.  The code format ("int8" or "e4m3")
    and the scale format ("fp32" or "e8m0") follow the dtypes of
    grad_input_q and grad_input_s unless given; ``y_scale_layout`` is "k_mg"
    (y_s_t [K, ceil(M/G)]) or "mg_k"; ``group_size`` is 128, 64, 32 or 256.  Every
    tensor is 2-D row-major; rows may be padded (a slice of a wider buffer):
    the library takes each tensor's row stride.  ``y`` (bf16 [M, K], optional)
    also receives the recomputed y itself, the values y_q_t quantizes.  With
    ``grad_y_s`` (fp32 [M, ceil(K/128)]) grad_y is INT8 codes [M, K] standing for
    grad_y * grad_y_s[m, k // 128] (grad_y handed over already quantized).
    Raises ValueError on bad arguments and SdqError on a library status."""
    outs = (grad_input_q, grad_input_s, y_q_t, y_s_t)
    codes = _infer("codes", codes, grad_input_q, _CODE_DTYPES)
    scales = _infer("scales", scales, grad_input_s, _SCALE_DTYPES)
    fmt = output_format(codes, scales, y_scale_layout)
    M, K, ld_x, ld_gy, lds, gys = _check_tensors(x, grad_y, outs, group_size, True, codes, scales,
                                                 y_scale_layout, grad_y_s)
    _call_strided(x.data_ptr(), ld_x, x.data_ptr() + 2 * K, ld_x, grad_y, ld_gy, outs, lds, M, K,
                  group_size, fmt, x.device, y, *gys)


def silu_dot_fwd_bwd_quant_fuse_split(gate: torch.Tensor, up: torch.Tensor, grad_y: torch.Tensor,
                                      grad_input_q: torch.Tensor, grad_input_s: torch.Tensor,
                                      y_q_t: torch.Tensor, y_s_t: torch.Tensor,
                                      group_size: int = GROUP_SIZE, *, codes: Optional[str] = None,
                                      scales: Optional[str] = None,
                                      y_scale_layout: str = "k_mg",
                                      y: Optional[torch.Tensor] = None,
                                      grad_y_s: Optional[torch.Tensor] = None) -> None:
    """The op with gate and up as two [M, K] bf16 tensors instead of one
    x = [gate | up] (e.g. the two halves of a fused projection kept apart);
    otherwise as silu_dot_fwd_bwd_quant_fuse."""
    outs = (grad_input_q, grad_input_s, y_q_t, y_s_t)
    codes = _infer("codes", codes, grad_input_q, _CODE_DTYPES)
    scales = _infer("scales", scales, grad_input_s, _SCALE_DTYPES)
    fmt = output_format(codes, scales, y_scale_layout)
    if gate.dim() != 2:
        raise ValueError("gate must be 2-D")
    M, K = gate.shape
    _check_group(K, group_size, True)
    bf16 = (torch.bfloat16,)
    ld_g = _rows("gate", gate, (M, K), bf16, True, gate.device)
    ld_u = _rows("up", up, (M, K), bf16, True, gate.device)
    ld_gy, gys, ld_gys = _grad_y(grad_y, grad_y_s, M, K, gate.device)
    lds = _check_outputs(M, K, outs, group_size, True, codes, scales, y_scale_layout, gate.device)
    _call_strided(gate.data_ptr(), ld_g, up.data_ptr(), ld_u, grad_y, ld_gy, outs, lds, M, K,
                  group_size, fmt, gate.device, y, gys, ld_gys)


def silu_dot_fwd_bwd_quant_fuse_host(x: torch.Tensor, grad_y: torch.Tensor,
                                     grad_input_q: torch.Tensor, grad_input_s: torch.Tensor,
                                     y_q_t: torch.Tensor, y_s_t: torch.Tensor,
                                     workspace: torch.Tensor, group_size: int = GROUP_SIZE,
                                     chunk_rows: int = 0, device: Optional[torch.device] = None,
                                     synchronize: bool = True) -> None:
    """The op on HOST tensors (pinned for overlapped copies), staged through a
    device ``workspace`` (uint8 CUDA tensor of at least
    ``sdq_fuse_host_workspace_bytes(M, K, chunk_rows)`` bytes)."""
    outs = (grad_input_q, grad_input_s, y_q_t, y_s_t)
    M, K, _, _, _, _ = _check_tensors(x, grad_y, outs, group_size, want_cuda=False)
    if not workspace.is_cuda:
        raise ValueError("workspace must be a CUDA tensor")
    dev = device or workspace.device
    with torch.cuda.device(dev):
        stream = torch.cuda.current_stream(dev).cuda_stream
        sdq_fuse_host(x.data_ptr(), grad_y.data_ptr(), grad_input_q.data_ptr(),
                      grad_input_s.data_ptr(), y_q_t.data_ptr(), y_s_t.data_ptr(), M, K,
                      group_size, workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                      chunk_rows, stream)
        if synchronize:
            torch.cuda.current_stream(dev).synchronize()


Q8_1_BLOCK_BYTES = 36


def swiglu_q8_1(gate: torch.Tensor, up: torch.Tensor, w: Optional[torch.Tensor] = None,
                limit: float = 0.0, h: Optional[torch.Tensor] = None,
                q8: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """The forward-side neighbour: h = bf16(silu(gate) * up * w[row]) (gate and
    up clamped when limit > 0) and its q8_1 blocks, on the current CUDA stream.
    gate, up: bf16 [rows, inter] (row-major, rows may be padded); w: fp32
    [rows] or None.  Returns (h bf16 [rows, inter], q8 uint8 [rows, inter/32, 36]),
    allocating whichever is not given."""
    if gate.dim() != 2:
        raise ValueError("gate must be 2-D")
    rows, inter = gate.shape
    if inter % 32 or inter < 32:
        raise ValueError(f"inter={inter} must be a positive multiple of 32")
    bf16 = (torch.bfloat16,)
    ld_g = _rows("gate", gate, (rows, inter), bf16, True, gate.device)
    ld_u = _rows("up", up, (rows, inter), bf16, True, gate.device)
    if h is None:
        h = torch.empty((rows, inter), dtype=torch.bfloat16, device=gate.device)
    ld_h = _rows("h", h, (rows, inter), bf16, True, gate.device)
    if q8 is None:
        q8 = torch.empty((rows, inter // 32, Q8_1_BLOCK_BYTES), dtype=torch.uint8, device=gate.device)
    if tuple(q8.shape) != (rows, inter // 32, Q8_1_BLOCK_BYTES) or q8.dtype != torch.uint8 or \
            not q8.is_contiguous() or q8.device != gate.device:
        raise ValueError(f"q8 must be a contiguous uint8 CUDA tensor [{rows}, {inter // 32}, 36]")
    wp = None
    if w is not None:
        if tuple(w.shape) != (rows,) or w.dtype != torch.float32 or not w.is_contiguous() or \
                w.device != gate.device:
            raise ValueError(f"w must be a contiguous float32 CUDA tensor [{rows}]")
        wp = w.data_ptr()
    with torch.cuda.device(gate.device):
        stream = torch.cuda.current_stream(gate.device).cuda_stream
        sdq_swiglu_q8_1(gate.data_ptr(), ld_g, up.data_ptr(), ld_u, wp, h.data_ptr(), ld_h,
                        q8.data_ptr(), rows, inter, limit, stream)
    return h, q8


def run(x: torch.Tensor, grad_y: torch.Tensor, group_size: int = GROUP_SIZE, codes: str = "int8",
        scales: str = "fp32", y_scale_layout: str = "k_mg"
        ) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor, torch.Tensor]:
    """Allocate the outputs and run the op; returns (grad_input_q, grad_input_s, y_q_t, y_s_t)."""
    M, K2 = x.shape
    outs = allocate_outputs(M, K2 // 2, x.device, group_size, codes, scales, y_scale_layout)
    silu_dot_fwd_bwd_quant_fuse(x, grad_y, *outs, group_size=group_size, codes=codes,
                                scales=scales, y_scale_layout=y_scale_layout)
    return outs

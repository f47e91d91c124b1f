"""B200-native silu_dot_fwd_bwd_quant_fuse: fused SwiGLU forward recompute,
backward and dual-axis INT8 quantization ("kernelgen-challenge-9-task3-silu-quant",
entry point and outputs sections).

    silu_dot_fwd_bwd_quant_fuse(x, grad_y, grad_input_q, grad_input_s, y_q_t, y_s_t,
                                group_size=128)

takes CUDA tensors x = [gate | up] (bf16 [M, 2K]) and grad_y (bf16 [M, K]) and
writes, in place, grad_input_q (int8 [M, 2K]), grad_input_s (fp32 [M, 2K/128]),
y_q_t (int8 [K, M]) and y_s_t (fp32 [K, ceil(M/128)]).  PyTorch supplies only
the device memory and the current stream; the work runs in libsdq.so.
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch

from ._lib import (LIB_PATH, SdqError, Status, last_cuda_error, sdq_device_status, sdq_fuse,
                   sdq_fuse_host, sdq_fuse_host_noalloc, sdq_fuse_host_workspace_bytes,
                   sdq_validate, status_string, version)

__all__ = [
    "silu_dot_fwd_bwd_quant_fuse", "silu_dot_fwd_bwd_quant_fuse_host", "allocate_outputs",
    "output_shapes", "sdq_fuse", "sdq_fuse_host", "sdq_fuse_host_noalloc",
    "sdq_fuse_host_workspace_bytes", "sdq_validate",
    "sdq_device_status", "SdqError", "Status", "status_string", "last_cuda_error", "version",
    "LIB_PATH", "GROUP_SIZE",
]

GROUP_SIZE = 128


def output_shapes(M: int, K: int, group_size: int = GROUP_SIZE):
    """Shapes of (grad_input_q, grad_input_s, y_q_t, y_s_t)."""
    G = group_size
    return (M, 2 * K), (M, 2 * (K // G)), (K, M), (K, (M + G - 1) // G)


def allocate_outputs(M: int, K: int, device, group_size: int = GROUP_SIZE):
    """Uninitialised output tensors for one call (the op writes every element)."""
    s = output_shapes(M, K, group_size)
    return (torch.empty(s[0], dtype=torch.int8, device=device),
            torch.empty(s[1], dtype=torch.float32, device=device),
            torch.empty(s[2], dtype=torch.int8, device=device),
            torch.empty(s[3], dtype=torch.float32, device=device))


def _check_tensors(x, grad_y, outs, group_size, want_cuda: bool):
    if x.dim() != 2 or grad_y.dim() != 2:
        raise ValueError("x and grad_y must be 2-D")
    M, K2 = x.shape
    if K2 % 2:
        raise ValueError(f"x has an odd channel count {K2}; expected [gate | up]")
    K = K2 // 2
    if tuple(grad_y.shape) != (M, K):
        raise ValueError(f"grad_y shape {tuple(grad_y.shape)} != {(M, K)}")
    if x.dtype != torch.bfloat16 or grad_y.dtype != torch.bfloat16:
        raise ValueError("x and grad_y must be bfloat16")
    if group_size != GROUP_SIZE or K % group_size:
        raise ValueError(f"group_size must be 128 and K={K} a multiple of it")
    names = ("grad_input_q", "grad_input_s", "y_q_t", "y_s_t")
    dtypes = (torch.int8, torch.float32, torch.int8, torch.float32)
    for name, t, shape, dt in zip(names, outs, output_shapes(M, K, group_size), dtypes):
        if tuple(t.shape) != shape or t.dtype != dt:
            raise ValueError(f"{name}: expected {dt} {shape}, got {t.dtype} {tuple(t.shape)}")
    for name, t in zip(("x", "grad_y") + names, (x, grad_y) + tuple(outs)):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        if want_cuda and (not t.is_cuda or t.device != x.device):
            raise ValueError(f"{name} must be a CUDA tensor on {x.device}")
        if not want_cuda and t.is_cuda:
            raise ValueError(f"{name} must be a host tensor")
    return M, K


def silu_dot_fwd_bwd_quant_fuse(x: torch.Tensor, grad_y: torch.Tensor, grad_input_q: torch.Tensor,
                                grad_input_s: torch.Tensor, y_q_t: torch.Tensor,
                                y_s_t: torch.Tensor, group_size: int = GROUP_SIZE) -> None:
    """Fused SwiGLU backward + dual-axis INT8 quantization, in place, on the
    current CUDA stream of x's device.  Raises ValueError on bad arguments and
    SdqError on a library status."""
    outs = (grad_input_q, grad_input_s, y_q_t, y_s_t)
    M, K = _check_tensors(x, grad_y, outs, group_size, want_cuda=True)
    with torch.cuda.device(x.device):
        stream = torch.cuda.current_stream(x.device).cuda_stream
        sdq_fuse(x.data_ptr(), grad_y.data_ptr(), grad_input_q.data_ptr(), grad_input_s.data_ptr(),
                 y_q_t.data_ptr(), y_s_t.data_ptr(), M, K, group_size, stream)


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
    M, K = _check_tensors(x, grad_y, outs, group_size, want_cuda=False)
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


def run(x: torch.Tensor, grad_y: torch.Tensor, group_size: int = GROUP_SIZE
        ) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor, torch.Tensor]:
    """Allocate the outputs and run the op; returns (grad_input_q, grad_input_s, y_q_t, y_s_t)."""
    M, K2 = x.shape
    outs = allocate_outputs(M, K2 // 2, x.device, group_size)
    silu_dot_fwd_bwd_quant_fuse(x, grad_y, *outs, group_size=group_size)
    return outs

"""ctypes binding of libsdq.so (the C ABI in include/sdq.h).

Argument marshalling only: every step of the op runs in the CUDA library.
There is no CPU path; if the library is missing, importing this module raises.
"""
from __future__ import annotations

import ctypes
import enum
import os
from typing import Optional

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsdq.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m swiglu_backward_int8_b200.build` "
        "(or __graft_entry__.build()); there is no fallback implementation")

_lib = ctypes.CDLL(LIB_PATH)

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I32 = ctypes.c_int32

_lib.sdq_fuse.argtypes = [_P, _P, _P, _P, _P, _P, _I64, _I64, _I32, _P]
_lib.sdq_fuse.restype = ctypes.c_int
_lib.sdq_validate.argtypes = [_P, _P, _P, _P, _P, _P, _I64, _I64, _I32]
_lib.sdq_validate.restype = ctypes.c_int
_lib.sdq_fuse_format.argtypes = [_P, _P, _P, _P, _P, _P, _I64, _I64, _I32, ctypes.c_uint32, _P]
_lib.sdq_fuse_format.restype = ctypes.c_int
_lib.sdq_validate_format.argtypes = [_P, _P, _P, _P, _P, _P, _I64, _I64, _I32, ctypes.c_uint32]
_lib.sdq_validate_format.restype = ctypes.c_int
_STRIDED = [_P, _I64] * 8 + [_I64, _I64, _I32, ctypes.c_uint32]
_lib.sdq_fuse_strided.argtypes = _STRIDED + [_P]
_lib.sdq_fuse_strided.restype = ctypes.c_int
_lib.sdq_validate_strided.argtypes = _STRIDED
_lib.sdq_validate_strided.restype = ctypes.c_int
_INT8_GY = [_P, _I64] * 9 + [_I64, _I64, _I32, ctypes.c_uint32]
_lib.sdq_fuse_int8_grad_y.argtypes = _INT8_GY + [_P]
_lib.sdq_fuse_int8_grad_y.restype = ctypes.c_int
_lib.sdq_validate_int8_grad_y.argtypes = _INT8_GY
_lib.sdq_validate_int8_grad_y.restype = ctypes.c_int
_lib.sdq_swiglu_q8_1.argtypes = [_P, _I64, _P, _I64, _P, _P, _I64, _P, _I64, _I64, ctypes.c_float, _P]
_lib.sdq_swiglu_q8_1.restype = ctypes.c_int
_lib.sdq_validate_swiglu_q8_1.argtypes = [_P, _I64, _P, _I64, _P, _P, _I64, _P, _I64, _I64]
_lib.sdq_validate_swiglu_q8_1.restype = ctypes.c_int
_lib.sdq_fuse_host.argtypes = [_P, _P, _P, _P, _P, _P, _I64, _I64, _I32, _P, ctypes.c_size_t, _I64, _P]
_lib.sdq_fuse_host.restype = ctypes.c_int
_lib.sdq_fuse_host_workspace_bytes.argtypes = [_I64, _I64, _I64]
_lib.sdq_fuse_host_workspace_bytes.restype = ctypes.c_size_t
_lib.sdq_fuse_host_noalloc.argtypes = [_P, _P, _P, _P, _P, _P, _I64, _I64, _I32, _P]
_lib.sdq_fuse_host_noalloc.restype = ctypes.c_int
_lib.sdq_fuse_test_stall.argtypes = [_P, _P, _P, _P, _P, _P, _I64, _I64, _I32, _I64, _P]
_lib.sdq_fuse_test_stall.restype = ctypes.c_int
_lib.sdq_device_status.argtypes = [_P]
_lib.sdq_device_status.restype = ctypes.c_int
_lib.sdq_status_string.argtypes = [ctypes.c_int]
_lib.sdq_status_string.restype = ctypes.c_char_p
_lib.sdq_last_cuda_error.argtypes = []
_lib.sdq_last_cuda_error.restype = ctypes.c_int
_lib.sdq_version.argtypes = []
_lib.sdq_version.restype = ctypes.c_char_p


class Status(enum.IntEnum):
    OK = 0
    ERR_NULL = 1
    ERR_GROUP = 2
    ERR_SHAPE = 3
    ERR_ALIGN = 4
    ERR_CUDA = 5
    ERR_TIMEOUT = 6
    ERR_WORKSPACE = 7
    ERR_TOO_LARGE = 8
    ERR_FORMAT = 9
    ERR_STRIDE = 10


# Output-format bits of sdq_fuse_format (include/sdq.h): 0 = INT8 codes, fp32
# scales, y_s_t [K, ceil(M/128)].
FMT_E4M3 = 1       # codes are OCP FP8 E4M3 bytes
FMT_E8M0 = 2       # scales are E8M0 bytes (powers of two)
FMT_YS_MG_K = 4    # y_s_t is [ceil(M/128), K]


class SdqError(RuntimeError):
    """A non-OK status from the library."""

    def __init__(self, status: int, where: str):
        self.status = Status(status) if status in Status._value2member_map_ else status
        msg = f"{where}: {status_string(status)}"
        if status == Status.ERR_CUDA:
            msg += f" (cudaError {last_cuda_error()})"
        super().__init__(msg)


def status_string(status: int) -> str:
    return _lib.sdq_status_string(int(status)).decode()


def last_cuda_error() -> int:
    return int(_lib.sdq_last_cuda_error())


def version() -> str:
    return _lib.sdq_version().decode()


def _check(status: int, where: str) -> None:
    if status != Status.OK:
        raise SdqError(status, where)


def sdq_fuse(x: int, grad_y: int, grad_input_q: int, grad_input_s: int, y_q_t: int, y_s_t: int,
             M: int, K: int, group_size: int = 128, stream: Optional[int] = None) -> None:
    """Raw-pointer form of the device entry point (device addresses as ints)."""
    _check(_lib.sdq_fuse(x, grad_y, grad_input_q, grad_input_s, y_q_t, y_s_t, M, K,
                         group_size, stream or 0), "sdq_fuse")


def sdq_fuse_format(x: int, grad_y: int, grad_input_q: int, grad_input_s: int, y_q_t: int,
                    y_s_t: int, M: int, K: int, group_size: int = 128, format: int = 0,
                    stream: Optional[int] = None) -> None:
    """Raw-pointer form of the device entry point with an output format (FMT_* bits)."""
    _check(_lib.sdq_fuse_format(x, grad_y, grad_input_q, grad_input_s, y_q_t, y_s_t, M, K,
                                group_size, format, stream or 0), "sdq_fuse_format")


def sdq_fuse_strided(gate: int, ld_gate: int, up: int, ld_up: int, grad_y: int, ld_grad_y: int,
                     grad_input_q: int, ld_grad_input_q: int, grad_input_s: int, ld_grad_input_s: int,
                     y_q_t: int, ld_y_q_t: int, y_s_t: int, ld_y_s_t: int, y: Optional[int],
                     ld_y: int, M: int, K: int, group_size: int = 128, format: int = 0,
                     stream: Optional[int] = None) -> None:
    """Raw-pointer form of the strided entry point (leading dimensions in
    elements; y, the optional bf16 y output, may be None)."""
    _check(_lib.sdq_fuse_strided(gate, ld_gate, up, ld_up, grad_y, ld_grad_y, grad_input_q,
                                 ld_grad_input_q, grad_input_s, ld_grad_input_s, y_q_t, ld_y_q_t,
                                 y_s_t, ld_y_s_t, y, ld_y, M, K, group_size, format, stream or 0),
           "sdq_fuse_strided")


def sdq_validate_strided(gate: int, ld_gate: int, up: int, ld_up: int, grad_y: int, ld_grad_y: int,
                         grad_input_q: int, ld_grad_input_q: int, grad_input_s: int,
                         ld_grad_input_s: int, y_q_t: int, ld_y_q_t: int, y_s_t: int, ld_y_s_t: int,
                         y: Optional[int], ld_y: int, M: int, K: int, group_size: int = 128,
                         format: int = 0) -> int:
    """Argument checks of sdq_fuse_strided only (no CUDA call); returns the status code."""
    return int(_lib.sdq_validate_strided(gate, ld_gate, up, ld_up, grad_y, ld_grad_y, grad_input_q,
                                         ld_grad_input_q, grad_input_s, ld_grad_input_s, y_q_t,
                                         ld_y_q_t, y_s_t, ld_y_s_t, y, ld_y, M, K, group_size,
                                         format))


def sdq_fuse_int8_grad_y(gate: int, ld_gate: int, up: int, ld_up: int, grad_y_q: int,
                         ld_grad_y_q: int, grad_y_s: int, ld_grad_y_s: int, grad_input_q: int,
                         ld_grad_input_q: int, grad_input_s: int, ld_grad_input_s: int, y_q_t: int,
                         ld_y_q_t: int, y_s_t: int, ld_y_s_t: int, y: Optional[int], ld_y: int,
                         M: int, K: int, group_size: int = 128, format: int = 0,
                         stream: Optional[int] = None) -> None:
    """Raw-pointer form of the entry point taking grad_y as INT8 codes and
    fp32 scales (leading dimensions in elements)."""
    _check(_lib.sdq_fuse_int8_grad_y(gate, ld_gate, up, ld_up, grad_y_q, ld_grad_y_q, grad_y_s,
                                     ld_grad_y_s, grad_input_q, ld_grad_input_q, grad_input_s,
                                     ld_grad_input_s, y_q_t, ld_y_q_t, y_s_t, ld_y_s_t, y, ld_y, M,
                                     K, group_size, format, stream or 0),
           "sdq_fuse_int8_grad_y")


def sdq_validate_int8_grad_y(gate: int, ld_gate: int, up: int, ld_up: int, grad_y_q: int,
                             ld_grad_y_q: int, grad_y_s: int, ld_grad_y_s: int, grad_input_q: int,
                             ld_grad_input_q: int, grad_input_s: int, ld_grad_input_s: int,
                             y_q_t: int, ld_y_q_t: int, y_s_t: int, ld_y_s_t: int,
                             y: Optional[int], ld_y: int, M: int, K: int, group_size: int = 128,
                             format: int = 0) -> int:
    """Argument checks of sdq_fuse_int8_grad_y only (no CUDA call); returns the status code."""
    return int(_lib.sdq_validate_int8_grad_y(gate, ld_gate, up, ld_up, grad_y_q, ld_grad_y_q,
                                             grad_y_s, ld_grad_y_s, grad_input_q, ld_grad_input_q,
                                             grad_input_s, ld_grad_input_s, y_q_t, ld_y_q_t, y_s_t,
                                             ld_y_s_t, y, ld_y, M, K, group_size, format))


def sdq_swiglu_q8_1(gate: int, ld_gate: int, up: int, ld_up: int, w: Optional[int], h: int, ld_h: int,
                    q8: int, rows: int, inter: int, limit: float = 0.0,
                    stream: Optional[int] = None) -> None:
    """Raw-pointer form of the forward SwiGLU + q8_1 entry point (w may be None)."""
    _check(_lib.sdq_swiglu_q8_1(gate, ld_gate, up, ld_up, w or None, h, ld_h, q8, rows, inter,
                                float(limit), stream or 0), "sdq_swiglu_q8_1")


def sdq_validate_swiglu_q8_1(gate: int, ld_gate: int, up: int, ld_up: int, w: Optional[int], h: int,
                             ld_h: int, q8: int, rows: int, inter: int) -> int:
    """Argument checks of sdq_swiglu_q8_1 only (no CUDA call); returns the status code."""
    return int(_lib.sdq_validate_swiglu_q8_1(gate, ld_gate, up, ld_up, w or None, h, ld_h, q8, rows,
                                             inter))


def sdq_validate_format(x: int, grad_y: int, grad_input_q: int, grad_input_s: int, y_q_t: int,
                        y_s_t: int, M: int, K: int, group_size: int = 128, format: int = 0) -> int:
    """Argument checks of sdq_fuse_format only (no CUDA call); returns the status code."""
    return int(_lib.sdq_validate_format(x, grad_y, grad_input_q, grad_input_s, y_q_t, y_s_t, M, K,
                                        group_size, format))


def sdq_validate(x: int, grad_y: int, grad_input_q: int, grad_input_s: int, y_q_t: int,
                 y_s_t: int, M: int, K: int, group_size: int = 128) -> int:
    """Argument checks only (no CUDA call); returns the status code."""
    return int(_lib.sdq_validate(x, grad_y, grad_input_q, grad_input_s, y_q_t, y_s_t, M, K,
                                 group_size))


def sdq_fuse_host(x: int, grad_y: int, grad_input_q: int, grad_input_s: int, y_q_t: int,
                  y_s_t: int, M: int, K: int, group_size: int, workspace: int,
                  workspace_bytes: int, chunk_rows: int = 0, stream: Optional[int] = None) -> None:
    """Raw-pointer form of the host-buffer entry point."""
    _check(_lib.sdq_fuse_host(x, grad_y, grad_input_q, grad_input_s, y_q_t, y_s_t, M, K,
                              group_size, workspace, workspace_bytes, chunk_rows, stream or 0),
           "sdq_fuse_host")


def sdq_fuse_host_noalloc(x: int, grad_y: int, grad_input_q: int, grad_input_s: int, y_q_t: int,
                          y_s_t: int, M: int, K: int, group_size: int = 128,
                          stream: Optional[int] = None) -> None:
    """Host-buffer entry point for callers that cannot allocate device
    memory: it stages through a fixed array inside the library instead of a
    caller workspace (K up to SDQ_NOALLOC_MAX_K = 28800).  Host addresses as
    ints; the outputs are complete once `stream` is synchronized."""
    _check(_lib.sdq_fuse_host_noalloc(x, grad_y, grad_input_q, grad_input_s, y_q_t, y_s_t, M, K,
                                      group_size, stream or 0), "sdq_fuse_host_noalloc")


def sdq_fuse_test_stall(x: int, grad_y: int, grad_input_q: int, grad_input_s: int, y_q_t: int,
                        y_s_t: int, M: int, K: int, group_size: int, wait_limit_ns: int,
                        stream: Optional[int] = None) -> None:
    """Failure-path test hook: the kernel withholds its first load, so its
    first bounded wait runs out; sdq_device_status then reports ERR_TIMEOUT."""
    _check(_lib.sdq_fuse_test_stall(x, grad_y, grad_input_q, grad_input_s, y_q_t, y_s_t, M, K,
                                    group_size, wait_limit_ns, stream or 0), "sdq_fuse_test_stall")


def sdq_fuse_host_workspace_bytes(M: int, K: int, chunk_rows: int = 0) -> int:
    return int(_lib.sdq_fuse_host_workspace_bytes(M, K, chunk_rows))


def sdq_device_status(stream: Optional[int] = None) -> int:
    """Synchronize `stream`, read and clear the device status word."""
    return int(_lib.sdq_device_status(stream or 0))

"""CPU oracle for silu_dot_fwd_bwd_quant_fuse -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding) never imports it and never falls back to it.

The arithmetic lives in ``sdq_oracle.cpp`` (plain single-threaded C++, fp64);
this module only compiles it with g++ and marshals numpy arrays through
ctypes.  Every function's pin is listed in the C++ file's header.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sdq_oracle.cpp")
_LIB = os.path.join(_HERE, "liboracle.so")
# No fast-math and no FMA contraction: every fp64/fp32 operation rounds once,
# in the order written.
CXXFLAGS = ["-O2", "-std=c++17", "-fPIC", "-shared", "-fno-fast-math",
            "-ffp-contract=off", "-fno-strict-aliasing"]

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/liboracle.so`` (g++; a second or two)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["g++", *CXXFLAGS, _SRC, "-o", tmp], check=True)
        os.replace(tmp, _LIB)
    return _LIB


def lib() -> ctypes.CDLL:
    """The compiled oracle.  ``SDQ_ORACLE_LIB`` names another build of the same
    source (the mutation test plants mistakes in copies and points here)."""
    global _lib
    if _lib is None:
        path = os.environ.get("SDQ_ORACLE_LIB") or build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i64 = ctypes.c_int64
        dbl = ctypes.c_double
        L.oracle_bf16_rne.argtypes = [dbl]
        L.oracle_bf16_rne.restype = ctypes.c_uint16
        for f in (L.oracle_sigmoid, L.oracle_silu, L.oracle_silu_grad):
            f.argtypes = [dbl]
            f.restype = dbl
        L.oracle_swiglu_bwd_fp64.argtypes = [dbl, dbl, dbl, P, P, P]
        L.oracle_swiglu_bwd_fp64.restype = None
        L.oracle_quant_group.argtypes = [P, i64, i64, P, i64, P]
        L.oracle_quant_group.restype = None
        L.oracle_swiglu_bwd_bf16.argtypes = [P, P, i64, i64, P, P, P]
        L.oracle_swiglu_bwd_bf16.restype = None
        L.oracle_silu_dot_fwd_bwd_quant_fuse.argtypes = [P, P, P, P, P, P, i64, i64, i64]
        L.oracle_silu_dot_fwd_bwd_quant_fuse.restype = ctypes.c_int
        L.oracle_e4m3_rne.argtypes = [dbl]
        L.oracle_e4m3_rne.restype = ctypes.c_uint8
        L.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_value.restype = dbl
        L.oracle_e8m0_ceil.argtypes = [ctypes.c_float]
        L.oracle_e8m0_ceil.restype = ctypes.c_uint8
        L.oracle_e8m0_value.argtypes = [ctypes.c_uint8]
        L.oracle_e8m0_value.restype = dbl
        L.oracle_quant_group_fmt.argtypes = [P, i64, i64, P, i64, P, ctypes.c_int, ctypes.c_int]
        L.oracle_quant_group_fmt.restype = None
        L.oracle_silu_dot_fwd_bwd_quant_fuse_fmt.argtypes = [P, P, P, P, P, P, i64, i64, i64,
                                                             ctypes.c_int, ctypes.c_int, ctypes.c_int]
        L.oracle_silu_dot_fwd_bwd_quant_fuse_fmt.restype = ctypes.c_int
        L.oracle_swiglu_bwd_bf16_dy.argtypes = [P, P, i64, i64, P, P, P]
        L.oracle_swiglu_bwd_bf16_dy.restype = None
        L.oracle_dequant_grad_y.argtypes = [P, P, i64, i64, P]
        L.oracle_dequant_grad_y.restype = None
        L.oracle_silu_dot_fwd_bwd_quant_fuse_qgrad.argtypes = [P, P, P, P, P, P, P, i64, i64, i64,
                                                               ctypes.c_int, ctypes.c_int,
                                                               ctypes.c_int]
        L.oracle_silu_dot_fwd_bwd_quant_fuse_qgrad.restype = ctypes.c_int
        L.oracle_fp16_rne.argtypes = [dbl]
        L.oracle_fp16_rne.restype = ctypes.c_uint16
        L.oracle_q8_1_block.argtypes = [P, P]
        L.oracle_q8_1_block.restype = None
        L.oracle_swiglu_q8_1_rows.argtypes = [P, P, P, P, P, i64, i64, ctypes.c_float]
        L.oracle_swiglu_q8_1_rows.restype = ctypes.c_int
        _lib = L
    return _lib


def _ptr(a: np.ndarray) -> ctypes.c_void_p:
    return ctypes.c_void_p(a.ctypes.data)


def bf16_rne(v: float) -> int:
    """Nearest bf16 bit pattern of a double, ties to even."""
    return int(lib().oracle_bf16_rne(float(v)))


def sigmoid(g: float) -> float:
    return float(lib().oracle_sigmoid(float(g)))


def silu(g: float) -> float:
    return float(lib().oracle_silu(float(g)))


def silu_grad(g: float) -> float:
    return float(lib().oracle_silu_grad(float(g)))


def swiglu_bwd_fp64(g: float, u: float, dy: float) -> Tuple[float, float, float]:
    """(y, d_gate, d_up) of one element in fp64, before rounding."""
    out = [ctypes.c_double() for _ in range(3)]
    lib().oracle_swiglu_bwd_fp64(float(g), float(u), float(dy),
                                 *(ctypes.byref(o) for o in out))
    return tuple(o.value for o in out)  # type: ignore[return-value]


def quant_group(v_bf16: np.ndarray) -> Tuple[np.ndarray, float]:
    """Quantize one group of bf16 bit patterns -> (int8 q, fp32 scale)."""
    v = np.ascontiguousarray(v_bf16, dtype=np.uint16)
    q = np.zeros(v.size, dtype=np.int8)
    s = np.zeros(1, dtype=np.float32)
    lib().oracle_quant_group(_ptr(v), v.size, 1, _ptr(q), 1, _ptr(s))
    return q, float(s[0])


def swiglu_bwd_bf16(x: np.ndarray, grad_y: np.ndarray):
    """First stage: bf16 bit arrays (y, d_gate, d_up), each [M, K]."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    gy = np.ascontiguousarray(grad_y, dtype=np.uint16)
    M, K = gy.shape
    assert x.shape == (M, 2 * K)
    y = np.empty((M, K), np.uint16)
    dg = np.empty((M, K), np.uint16)
    du = np.empty((M, K), np.uint16)
    lib().oracle_swiglu_bwd_bf16(_ptr(x), _ptr(gy), M, K, _ptr(y), _ptr(dg), _ptr(du))
    return y, dg, du


def silu_dot_fwd_bwd_quant_fuse(x: np.ndarray, grad_y: np.ndarray, group_size: int = 128):
    """The whole op on uint16 (bf16 bit) arrays, in the page's format.

    Returns ``(grad_input_q [M,2K] int8, grad_input_s [M,2 ceil(K/G)] f32,
    y_q_t [K,M] int8, y_s_t [K,ceil(M/G)] f32)``; when G does not divide K
    the last channel group of each half of [d_gate | d_up] is shorter.
    """
    x = np.ascontiguousarray(x, dtype=np.uint16)
    gy = np.ascontiguousarray(grad_y, dtype=np.uint16)
    M, K = gy.shape
    assert x.shape == (M, 2 * K), (x.shape, gy.shape)
    G = int(group_size)
    if G < 1:
        raise ValueError(f"group_size={G} must be positive")
    Kg, Mg = (K + G - 1) // G, (M + G - 1) // G
    giq = np.zeros((M, 2 * K), np.int8)
    gis = np.zeros((M, 2 * Kg), np.float32)
    yqt = np.zeros((K, M), np.int8)
    yst = np.zeros((K, Mg), np.float32)
    rc = lib().oracle_silu_dot_fwd_bwd_quant_fuse(_ptr(x), _ptr(gy), _ptr(giq), _ptr(gis),
                                                  _ptr(yqt), _ptr(yst), M, K, G)
    if rc != 0:
        raise ValueError(f"oracle rejected M={M} K={K} group_size={G}")
    return giq, gis, yqt, yst


# ---- output formats (codes: 0 INT8, 1 E4M3; scales: 0 fp32, 1 E8M0;
# ys_layout: 0 y_s_t [K, Mg], 1 [Mg, K]) -------------------------------------

CODES_INT8, CODES_E4M3 = 0, 1
SCALES_FP32, SCALES_E8M0 = 0, 1
YS_K_MG, YS_MG_K = 0, 1


def e4m3_rne(v: float) -> int:
    """Nearest OCP E4M3 code (byte) of a double, ties to even, saturating at 448."""
    return int(lib().oracle_e4m3_rne(float(v)))


def e4m3_value(code: int) -> float:
    return float(lib().oracle_e4m3_value(int(code)))


def e8m0_ceil(s: float) -> int:
    """E8M0 byte of the smallest power of two >= s (s a positive float32)."""
    return int(lib().oracle_e8m0_ceil(float(s)))


def e8m0_value(e: int) -> float:
    return float(lib().oracle_e8m0_value(int(e)))


def quant_group_fmt(v_bf16: np.ndarray, codes: int = 0, scales: int = 0):
    """One group of bf16 bit patterns -> (code bytes uint8, scale) where the
    scale is a float (fp32 scales) or an int byte (E8M0)."""
    v = np.ascontiguousarray(v_bf16, dtype=np.uint16)
    q = np.zeros(v.size, dtype=np.uint8)
    s = np.zeros(4, dtype=np.uint8)
    lib().oracle_quant_group_fmt(_ptr(v), v.size, 1, _ptr(q), 1, _ptr(s), int(codes), int(scales))
    return q, (int(s[0]) if scales else float(s.view(np.float32)[0]))


def output_shapes_fmt(M: int, K: int, group_size: int = 128, ys_layout: int = 0):
    """Output shapes; with G not dividing K each half of a row ends in a
    shorter group, so grad_input_s has 2 * ceil(K/G) columns."""
    G = int(group_size)
    Kg, Mg = (K + G - 1) // G, (M + G - 1) // G
    return (M, 2 * K), (M, 2 * Kg), (K, M), ((Mg, K) if ys_layout else (K, Mg))


def silu_dot_fwd_bwd_quant_fuse_fmt(x: np.ndarray, grad_y: np.ndarray, group_size: int = 128,
                                    codes: int = 0, scales: int = 0, ys_layout: int = 0):
    """The whole op in a chosen output format, on uint16 (bf16 bit) arrays.

    Returns ``(grad_input_q [M,2K] uint8 code bytes, grad_input_s
    [M,2*ceil(K/G)], y_q_t [K,M] uint8, y_s_t [K,Mg] or [Mg,K])``; scale
    arrays are float32 (fp32 scales) or uint8 (E8M0 bytes).  When G does not
    divide K, each half of [d_gate | d_up] ends in a shorter group.
    """
    x = np.ascontiguousarray(x, dtype=np.uint16)
    gy = np.ascontiguousarray(grad_y, dtype=np.uint16)
    M, K = gy.shape
    assert x.shape == (M, 2 * K), (x.shape, gy.shape)
    G = int(group_size)
    if G < 1:
        raise ValueError(f"group_size={G}")
    sq, ss, yq, ys = output_shapes_fmt(M, K, G, ys_layout)
    sdt = np.uint8 if scales else np.float32
    giq = np.zeros(sq, np.uint8)
    gis = np.zeros(ss, sdt)
    yqt = np.zeros(yq, np.uint8)
    yst = np.zeros(ys, sdt)
    rc = lib().oracle_silu_dot_fwd_bwd_quant_fuse_fmt(_ptr(x), _ptr(gy), _ptr(giq), _ptr(gis),
                                                      _ptr(yqt), _ptr(yst), M, K, G,
                                                      int(codes), int(scales), int(ys_layout))
    if rc != 0:
        raise ValueError(f"oracle rejected M={M} K={K} group_size={G} format "
                         f"({codes}, {scales}, {ys_layout})")
    return giq, gis, yqt, yst


# ---- grad_y handed over already quantized ------------------------------------

def dequant_grad_y(grad_y_q: np.ndarray, grad_y_s: np.ndarray) -> np.ndarray:
    """dy = q * s as float64 [M, K]: codes int8 [M, K], scales float32
    [M, K/128], one per token and 128 consecutive channels."""
    q = np.ascontiguousarray(grad_y_q, dtype=np.int8)
    sc = np.ascontiguousarray(grad_y_s, dtype=np.float32)
    M, K = q.shape
    assert sc.shape == (M, (K + 127) // 128), (q.shape, sc.shape)
    dy = np.empty((M, K), np.float64)
    lib().oracle_dequant_grad_y(_ptr(q), _ptr(sc), M, K, _ptr(dy))
    return dy


def swiglu_bwd_bf16_dy(x: np.ndarray, dy: np.ndarray):
    """First stage on an fp64 grad_y: bf16 bit arrays (y, d_gate, d_up)."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    dy = np.ascontiguousarray(dy, dtype=np.float64)
    M, K = dy.shape
    assert x.shape == (M, 2 * K)
    y = np.empty((M, K), np.uint16)
    dg = np.empty((M, K), np.uint16)
    du = np.empty((M, K), np.uint16)
    lib().oracle_swiglu_bwd_bf16_dy(_ptr(x), _ptr(dy), M, K, _ptr(y), _ptr(dg), _ptr(du))
    return y, dg, du


def silu_dot_fwd_bwd_quant_fuse_qgrad(x: np.ndarray, grad_y_q: np.ndarray, grad_y_s: np.ndarray,
                                      group_size: int = 128, codes: int = 0, scales: int = 0,
                                      ys_layout: int = 0):
    """The whole op with grad_y given quantized (INT8 codes [M, K], fp32
    scales [M, K/128]); outputs as silu_dot_fwd_bwd_quant_fuse_fmt."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    q = np.ascontiguousarray(grad_y_q, dtype=np.int8)
    sc = np.ascontiguousarray(grad_y_s, dtype=np.float32)
    M, K = q.shape
    assert x.shape == (M, 2 * K) and sc.shape == (M, (K + 127) // 128), (x.shape, q.shape, sc.shape)
    G = int(group_size)
    sq, ss, yq, ys = output_shapes_fmt(M, K, G, ys_layout)
    sdt = np.uint8 if scales else np.float32
    giq = np.zeros(sq, np.uint8)
    gis = np.zeros(ss, sdt)
    yqt = np.zeros(yq, np.uint8)
    yst = np.zeros(ys, sdt)
    rc = lib().oracle_silu_dot_fwd_bwd_quant_fuse_qgrad(_ptr(x), _ptr(q), _ptr(sc), _ptr(giq),
                                                        _ptr(gis), _ptr(yqt), _ptr(yst), M, K, G,
                                                        int(codes), int(scales), int(ys_layout))
    if rc != 0:
        raise ValueError(f"oracle rejected M={M} K={K} group_size={G}")
    return giq, gis, yqt, yst


# ---- forward-side neighbour: SwiGLU forward + q8_1 rows ----------------------

Q8_1_BLOCK_BYTES = 36


def fp16_rne(v: float) -> int:
    """Nearest IEEE binary16 bit pattern of a double, ties to even."""
    return int(lib().oracle_fp16_rne(float(v)))


def q8_1_block(h_bf16: np.ndarray) -> np.ndarray:
    """One 36-byte q8_1 block (fp16 d, fp16 sum, 32 int8) of 32 bf16 values."""
    h = np.ascontiguousarray(h_bf16, dtype=np.uint16)
    assert h.size == 32
    out = np.zeros(Q8_1_BLOCK_BYTES, np.uint8)
    lib().oracle_q8_1_block(_ptr(h), _ptr(out))
    return out


def swiglu_q8_1_rows(gate: np.ndarray, up: np.ndarray, w=None, limit: float = 0.0):
    """The forward op on uint16 (bf16 bit) arrays [rows, inter]; w float32 [rows]
    or None.  Returns (h [rows, inter] uint16 bf16 bits, q8 [rows, inter/32, 36] uint8)."""
    g = np.ascontiguousarray(gate, dtype=np.uint16)
    u = np.ascontiguousarray(up, dtype=np.uint16)
    rows, inter = g.shape
    assert u.shape == g.shape
    h = np.zeros((rows, inter), np.uint16)
    q8 = np.zeros((rows, inter // 32, Q8_1_BLOCK_BYTES), np.uint8)
    wp = None
    if w is not None:
        w = np.ascontiguousarray(w, dtype=np.float32)
        assert w.shape == (rows,)
        wp = _ptr(w)
    rc = lib().oracle_swiglu_q8_1_rows(_ptr(g), _ptr(u), wp, _ptr(h), _ptr(q8), rows, inter,
                                       float(limit))
    if rc != 0:
        raise ValueError(f"oracle rejected rows={rows} inter={inter}")
    return h, q8

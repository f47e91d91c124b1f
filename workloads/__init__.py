"""Seeded synthetic inputs for silu_dot_fwd_bwd_quant_fuse.

This module is the one piece of code that both sides of the parity check use:
the CUDA path (through ``bench.py`` and the tests) and the CPU oracle (through
the tests). It holds none of the method's arithmetic -- no sigmoid, no
gradients, no quantization -- only the construction of the inputs ``x`` and
``grad_y`` as bf16 bit patterns (``numpy.uint16``).

Random numbers come from splitmix64 (Steele, Lea and Flood, "Fast splittable
pseudorandom number generators", OOPSLA 2014), used counter-style: draw ``n``
of a stream with key ``k`` is ``mix64(k + (n + 1) * GOLDEN)``, so any element
can be produced on its own and chunking never changes the values.  Normal
samples use the Box-Muller transform: element ``2p`` takes the cosine branch
and element ``2p + 1`` the sine branch of the pair built from draws ``2p`` and
``2p + 1``.  A sample is scaled by sigma in float64, rounded to float32, then
to bf16 with round-to-nearest-even.

Streams: 0 = x, 1 = grad_y, 2 = outlier mask over x, 3 = zero-group choice.

The workloads are those of the fused SwiGLU backward + dual-axis INT8
quantization op described on "kernelgen-challenge-9-task3-silu-quant"
(entry point and outputs sections): ``x = [gate | up]`` is ``[M, 2K]`` and
``grad_y`` is ``[M, K]``, both bf16, with ``group_size = 128``.
"""
from __future__ import annotations

import concurrent.futures
import dataclasses
import math
import os
from typing import Dict, List, Tuple

import numpy as np

GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_CHUNK = 1 << 22

ZERO_GROUP_WIDTH = 128   # channels zeroed (in gate and up) per zero-group row, whatever the group size

STREAM_X = 0
STREAM_GRAD_Y = 1
STREAM_OUTLIER = 2
STREAM_ZERO_GROUP = 3


def _mix64(z: np.ndarray) -> np.ndarray:
    """splitmix64 finaliser on a uint64 array (wrapping arithmetic)."""
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def _mix64_scalar(v: int) -> int:
    with np.errstate(over="ignore"):
        return int(_mix64(np.array([v & 0xFFFFFFFFFFFFFFFF], dtype=np.uint64))[0])


def stream_key(seed: int, stream: int) -> int:
    """Key of one named stream of one seed."""
    return _mix64_scalar(_mix64_scalar(seed) ^ (((stream + 1) * 0x9E3779B97F4A7C15) & 0xFFFFFFFFFFFFFFFF))


def draws(key: int, start: int, count: int) -> np.ndarray:
    """Raw 64-bit draws ``start .. start+count-1`` of the stream ``key``."""
    n = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix64(np.uint64(key) + n * GOLDEN)


def uniforms(key: int, start: int, count: int) -> np.ndarray:
    """Uniform float64 in [0, 1): the top 53 bits of each draw."""
    return (draws(key, start, count) >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def normals(key: int, start: int, count: int) -> np.ndarray:
    """Standard normal float64 samples ``start .. start+count-1`` (Box-Muller)."""
    p0 = start // 2
    p1 = (start + count + 1) // 2
    npair = p1 - p0
    d = draws(key, 2 * p0, 2 * npair)
    u1 = ((d[0::2] >> np.uint64(11)).astype(np.float64) + 1.0) * (2.0 ** -53)  # (0, 1]
    u2 = (d[1::2] >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)          # [0, 1)
    r = np.sqrt(-2.0 * np.log(u1))
    t = 2.0 * math.pi * u2
    z = np.empty(2 * npair, dtype=np.float64)
    z[0::2] = r * np.cos(t)
    z[1::2] = r * np.sin(t)
    off = start - 2 * p0
    return z[off:off + count]


def f32_to_bf16_bits(f: np.ndarray) -> np.ndarray:
    """float32 array -> bf16 bit patterns (uint16), round-to-nearest-even.

    Input construction only (the method's own bf16 rounding lives on each
    side of the check separately).  NaN is not expected here.
    """
    u = np.ascontiguousarray(f, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float32 (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _threads() -> int:
    return max(1, min(16, os.cpu_count() or 1))


def normal_bf16(seed: int, stream: int, count: int, sigma: float) -> np.ndarray:
    """``count`` samples of N(0, sigma) as bf16 bits, generated in chunks
    (on several threads; the values do not depend on the chunking)."""
    key = stream_key(seed, stream)
    out = np.empty(count, dtype=np.uint16)

    def fill(s: int) -> None:
        n = min(_CHUNK, count - s)
        z = normals(key, s, n) * float(sigma)
        out[s:s + n] = f32_to_bf16_bits(z.astype(np.float32))

    starts = range(0, count, _CHUNK)
    if count > _CHUNK and _threads() > 1:
        with concurrent.futures.ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(fill, starts))
    else:
        for s in starts:
            fill(s)
    return out


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic problem: shapes, value distributions and structure."""

    name: str
    M: int
    K: int
    sigma_x: float
    sigma_grad_y: float
    seed: int
    group_size: int = 128
    outlier_frac: float = 0.0      # fraction of x entries multiplied by outlier_mult
    outlier_mult: float = 50.0
    zero_group_every: int = 0      # one all-zero 128-channel group of gate and up per this many rows
    note: str = ""

    @property
    def Mg(self) -> int:
        return (self.M + self.group_size - 1) // self.group_size

    @property
    def Kg(self) -> int:
        return self.K // self.group_size

    def algorithmic_bytes(self, scale_bytes: int = 4) -> int:
        """Bytes any fused implementation must move: read x and grad_y (6 B per
        (m, k)), write grad_input_q (2 B) and y_q_t (1 B) codes, plus the
        scales (fp32: 4 B each; E8M0: 1 B)."""
        mk = self.M * self.K
        kgs = (self.K + self.group_size - 1) // self.group_size   # row groups per half (last may be short)
        return 6 * mk + 3 * mk + scale_bytes * (self.M * 2 * kgs + self.K * self.Mg)

    def describe(self) -> Dict[str, object]:
        return {"workload": self.name, "M": self.M, "K": self.K,
                "group_size": self.group_size, "sigma_x": self.sigma_x,
                "sigma_grad_y": self.sigma_grad_y, "seed": self.seed,
                "outlier_frac": self.outlier_frac,
                "zero_group_every": self.zero_group_every}


WORKLOADS: List[Workload] = [
    Workload("swiglu_bwd_int8_M256_K256", 256, 256, 1.0, 0.02, 0,
             note="small case; several tiles"),
    Workload("swiglu_bwd_int8_M4096_K1408", 4096, 1408, 1.0, 0.02, 1,
             note="MoE-expert-sized FFN"),
    Workload("swiglu_bwd_int8_M8192_K4096", 8192, 4096, 1.5, 1e-3, 2),
    Workload("swiglu_bwd_int8_M4000_K2048_outliers", 4000, 2048, 1.0, 0.02, 3,
             outlier_frac=1e-3, outlier_mult=50.0, zero_group_every=64,
             note="tail token group of 32 rows; 0.1% x50 outliers; zero groups"),
    Workload("swiglu_bwd_int8_M16384_K7168", 16384, 7168, 1.0, 0.01, 4,
             note="bandwidth-roofline case"),
]

BY_NAME: Dict[str, Workload] = {w.name: w for w in WORKLOADS}


def make_inputs(w: Workload) -> Tuple[np.ndarray, np.ndarray]:
    """Return ``(x, grad_y)`` as uint16 bf16 bit arrays of shapes [M, 2K], [M, K]."""
    M, K = w.M, w.K
    x = normal_bf16(w.seed, STREAM_X, M * 2 * K, w.sigma_x).reshape(M, 2 * K)
    gy = normal_bf16(w.seed, STREAM_GRAD_Y, M * K, w.sigma_grad_y).reshape(M, K)
    if w.outlier_frac > 0.0:
        key = stream_key(w.seed, STREAM_OUTLIER)
        flat = x.reshape(-1)
        for s in range(0, flat.size, _CHUNK):
            n = min(_CHUNK, flat.size - s)
            hit = np.nonzero(uniforms(key, s, n) < w.outlier_frac)[0] + s
            if hit.size:
                v = bf16_bits_to_f32(flat[hit]) * np.float32(w.outlier_mult)
                flat[hit] = f32_to_bf16_bits(v)
    nz = K // ZERO_GROUP_WIDTH
    if w.zero_group_every > 0 and nz > 0:
        key = stream_key(w.seed, STREAM_ZERO_GROUP)
        rows = np.arange(0, M, w.zero_group_every)
        groups = (draws(key, 0, rows.size) % np.uint64(nz)).astype(np.int64)
        G = ZERO_GROUP_WIDTH
        for r, j in zip(rows.tolist(), groups.tolist()):
            x[r, j * G:(j + 1) * G] = 0          # gate
            x[r, K + j * G:K + (j + 1) * G] = 0  # up
    return x, gy


def zero_group_positions(w: Workload) -> List[Tuple[int, int]]:
    """(row, group) pairs zeroed by ``make_inputs`` (for tests of the all-zero case)."""
    nz = w.K // ZERO_GROUP_WIDTH
    if w.zero_group_every <= 0 or nz == 0:
        return []
    key = stream_key(w.seed, STREAM_ZERO_GROUP)
    rows = np.arange(0, w.M, w.zero_group_every)
    groups = (draws(key, 0, rows.size) % np.uint64(nz)).astype(np.int64)
    return list(zip(rows.tolist(), groups.tolist()))


def small_workload(M: int, K: int, seed: int = 7, sigma_x: float = 1.0,
                   sigma_grad_y: float = 0.02, **kw) -> Workload:
    """An ad-hoc shape with the same recipe (tests of odd and tiny shapes)."""
    return Workload(f"swiglu_bwd_int8_M{M}_K{K}_s{seed}", M, K, sigma_x,
                    sigma_grad_y, seed, **kw)


# ---- the forward-side neighbour (SwiGLU forward + q8_1 rows) ------------------

STREAM_ROW_WEIGHT = 7


def row_weights(seed: int, rows: int) -> np.ndarray:
    """Per-row weights (e.g. MoE router weights) uniform in (0, 1], float32,
    from the seed's own stream."""
    u = uniforms(stream_key(seed, STREAM_ROW_WEIGHT), 0, rows)
    return (1.0 - u).astype(np.float32)


def fwd_inputs(w: Workload):
    """(gate, up, row weights) of a workload for the forward op: gate and up
    are the two halves of the workload's x ([rows, K] bf16 bits each, as views
    of x with row stride 2K), rows = M, inter = K."""
    x, _ = make_inputs(w)
    return x[:, :w.K], x[:, w.K:], row_weights(w.seed, w.M)


# ---- grad_y handed over already quantized ---------------------------------------

STREAM_GRAD_Y_CODES = 8
STREAM_GRAD_Y_SCALES = 9


def quantized_grad_y(w: Workload, pow2_scales: bool = False):
    """A grad_y already in the row-group INT8 format: (codes int8 [M, K],
    scales float32 [M, ceil(K/128)]).  Codes are a normal of spread 42 rounded and
    clipped to [-127, 127] (one value per channel); scales are
    sigma_grad_y / 42 times a log-normal factor exp(N(0, 1/4)) per token and
    128-channel group, so the values have about the bf16 grad_y's spread;
    with ``pow2_scales`` each scale is the nearest power of two of that.
    Every ``zero_group_every``-th token has one all-zero code group."""
    M, K = w.M, w.K
    Kg = (K + 127) // 128   # the last scale of a row covers what is left of it
    z = normals(stream_key(w.seed, STREAM_GRAD_Y_CODES), 0, M * K)
    q = np.clip(np.rint(z * 42.0), -127, 127).astype(np.int8).reshape(M, K)
    e = normals(stream_key(w.seed, STREAM_GRAD_Y_SCALES), 0, M * Kg).reshape(M, Kg)
    s = (w.sigma_grad_y / 42.0) * np.exp(0.5 * e)
    if pow2_scales:
        s = np.exp2(np.rint(np.log2(s)))
    s = s.astype(np.float32)
    if w.zero_group_every > 0 and Kg > 0:
        for r in range(0, M, w.zero_group_every):
            j = (r // w.zero_group_every) % Kg
            q[r, j * 128:(j + 1) * 128] = 0
    return q, s

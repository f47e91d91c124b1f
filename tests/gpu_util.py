"""Helpers for the GPU tests: run the CUDA path with guarded, sentinel-filled
outputs, run the oracle on the same inputs, and compare within the stated
tolerances.

Tolerances (from the arithmetic: the kernel computes in fp32 with the
hardware exp2/reciprocal approximations, the oracle in fp64; a value within a
few fp32 ulps of a bf16 rounding boundary can round the other way, and a
quotient within an ulp of a half-integer can round the other way):
  int8 outputs: |q_gpu - q_oracle| <= 1 everywhere, and != on at most 0.1 %
  of the elements;
  scales: relative difference <= 2^-7.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

INT8_MAX_DIFF = 1
INT8_MAX_FRAC = 1e-3
SCALE_MAX_REL = 2.0 ** -7
GUARD = 256
SENTINEL_Q = -128          # never produced by the op (q is in [-127, 127])


def to_device_bf16(a_u16: np.ndarray, device="cuda") -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(a_u16).view(np.int16)).view(torch.bfloat16)
    return t.to(device)


class Guarded:
    """An output tensor with guard bytes on both sides, prefilled."""

    def __init__(self, shape, dtype, fill, device="cuda"):
        n = int(np.prod(shape)) if len(shape) else 1
        esz = torch.empty((), dtype=dtype).element_size()
        g = GUARD // esz
        self.buf = torch.full((n + 2 * g,), fill, dtype=dtype, device=device)
        self.g = g
        self.n = n
        self.fill = fill
        self.guard_before = self.buf[:g].clone()
        self.guard_after = self.buf[g + n:].clone()
        self.t = self.buf[g:g + n].view(shape)

    def guards_intact(self) -> bool:
        b = self.buf
        same = lambda a, c: bool(torch.equal(a, c) or (torch.isnan(a).all() and torch.isnan(c).all()))
        return same(b[:self.g], self.guard_before) and same(b[self.g + self.n:], self.guard_after)


def run_cuda(x_u16: np.ndarray, gy_u16: np.ndarray, stream=None):
    """Run the device entry point; returns numpy outputs after checking that
    the guard bytes are intact and every element was written."""
    import swiglu_backward_int8_b200 as sdq
    M, K = gy_u16.shape
    x = to_device_bf16(x_u16)
    gy = to_device_bf16(gy_u16)
    shp = sdq.output_shapes(M, K)
    outs = [Guarded(shp[0], torch.int8, SENTINEL_Q), Guarded(shp[1], torch.float32, float("nan")),
            Guarded(shp[2], torch.int8, SENTINEL_Q), Guarded(shp[3], torch.float32, float("nan"))]
    if stream is None:
        sdq.silu_dot_fwd_bwd_quant_fuse(x, gy, *(o.t for o in outs))
    else:
        with torch.cuda.stream(stream):
            sdq.silu_dot_fwd_bwd_quant_fuse(x, gy, *(o.t for o in outs))
    torch.cuda.synchronize()
    assert sdq.sdq_device_status() == 0
    for o, name in zip(outs, ("grad_input_q", "grad_input_s", "y_q_t", "y_s_t")):
        assert o.guards_intact(), f"{name}: guard bytes overwritten"
    giq, gis, yqt, yst = (o.t.cpu().numpy() for o in outs)
    assert not (giq == SENTINEL_Q).any(), "grad_input_q: elements left unwritten"
    assert not (yqt == SENTINEL_Q).any(), "y_q_t: elements left unwritten"
    assert np.isfinite(gis).all() and np.isfinite(yst).all(), "scales left unwritten"
    return giq, gis, yqt, yst


def compare(got, ref, where=""):
    """Assert the tolerances; returns mismatch statistics."""
    giq, gis, yqt, yst = got
    rq, rs, ryq, rys = ref
    stats = {}
    for name, a, b in (("grad_input_q", giq, rq), ("y_q_t", yqt, ryq)):
        assert a.shape == b.shape, (name, a.shape, b.shape)
        d = np.abs(a.astype(np.int16) - b.astype(np.int16))
        nd = int((d != 0).sum())
        stats[name] = {"max_abs_diff": int(d.max()) if d.size else 0, "n_diff": nd,
                       "frac_diff": nd / max(1, d.size)}
        assert d.max(initial=0) <= INT8_MAX_DIFF, f"{where} {name}: max |dq| = {d.max()}"
        assert nd <= INT8_MAX_FRAC * d.size, f"{where} {name}: {nd} of {d.size} differ"
    for name, a, b in (("grad_input_s", gis, rs), ("y_s_t", yst, rys)):
        assert a.shape == b.shape, (name, a.shape, b.shape)
        rel = np.abs(a.astype(np.float64) - b.astype(np.float64)) / np.abs(b.astype(np.float64))
        stats[name] = {"max_rel_diff": float(rel.max()) if rel.size else 0.0,
                       "n_diff": int((a != b).sum())}
        assert rel.max(initial=0) <= SCALE_MAX_REL, f"{where} {name}: max rel = {rel.max()}"
    return stats


def oracle_tile(x_u16, gy_u16, i, j, G=128):
    """The oracle on one 128x128 tile (token group i, channel group j): every
    group lies inside one tile, so this is the op's definition restricted to
    the tile.  Returns the tile's pieces of the four outputs."""
    M, K = gy_u16.shape
    r0, r1 = i * G, min(M, i * G + G)
    xt = np.concatenate([x_u16[r0:r1, j * G:(j + 1) * G], x_u16[r0:r1, K + j * G:K + (j + 1) * G]],
                        axis=1)
    gyt = gy_u16[r0:r1, j * G:(j + 1) * G]
    return oracle.silu_dot_fwd_bwd_quant_fuse(xt, gyt, G)


def tile_of(outputs, M, K, i, j, G=128):
    """The same pieces cut out of full-size outputs (numpy or torch)."""
    giq, gis, yqt, yst = outputs
    Kg = K // G
    r0, r1 = i * G, min(M, i * G + G)
    c = slice(j * G, (j + 1) * G)
    q = giq[r0:r1]
    tq = np.concatenate([np.asarray(q[:, c]), np.asarray(q[:, K + j * G:K + (j + 1) * G])], axis=1)
    ts = np.stack([np.asarray(gis[r0:r1, j]), np.asarray(gis[r0:r1, Kg + j])], axis=1)
    return tq, ts, np.asarray(yqt[c, r0:r1]), np.asarray(yst[c, i:i + 1])

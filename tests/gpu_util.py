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


def compare(got, ref, where="", max_frac=INT8_MAX_FRAC):
    """Assert the tolerances; returns mismatch statistics.  max_frac: the
    bound on the fraction of differing codes (a sampled test applies it to
    the whole sample instead)."""
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
        assert nd <= max_frac * d.size, f"{where} {name}: {nd} of {d.size} differ"
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


# ---- output formats (codes: 0 INT8, 1 E4M3; scales: 0 fp32, 1 E8M0;
# ys_layout: 0 y_s_t [K, Mg], 1 [Mg, K]) -------------------------------------
#
# Tolerances for the formats, from the same arithmetic as above: a value that
# rounds to the other bf16 neighbour, or a quotient next to a rounding
# boundary of the code, moves a code to the adjacent one; with E8M0 scales a
# flipped amax can also move the group's power of two by one step.  So:
# codes equal on all but 0.1 % of the elements, and every dequantized value
# (code x scale) within one code step (of either side) of the oracle's;
# fp32 scales within 2^-7 relative, E8M0 bytes within 1 and equal on all but
# 0.1 %.  E4M3 has two zero codes of one value, +0 (0x00) and -0 (0x80); where
# sigma(g) underflows to 0 in fp32 (g < -88) but not in fp64, the kernel's
# product is an exact zero signed by the other factors while the oracle's
# tiny value rounds to the zero of its own sign, so the two zeros count as
# equal (and are reported as n_signed_zero).

SENTINEL_CODE = {0: 0x80, 1: 0x7F}     # INT8 -128; E4M3 NaN: neither is ever written
SENTINEL_E8M0 = 0xFF                   # E8M0 NaN: scales stop at 2^127 (byte 254)


def _e4m3_values():
    from tests.exact import e4m3_table
    v = np.full(256, np.nan)
    for val, c in e4m3_table():
        v[c] = float(val)
        v[c | 0x80] = -float(val)
    return v


E4M3_VALUE = _e4m3_values()


def run_cuda_fmt(x_u16: np.ndarray, gy_u16: np.ndarray, codes: int, scales: int, ys_layout: int,
                 group_size: int = 128):
    """The device entry point in a chosen format, on guarded outputs; returns
    numpy (code bytes, scales, code bytes, scales) like the format oracle."""
    import swiglu_backward_int8_b200 as sdq
    M, K = gy_u16.shape
    x = to_device_bf16(x_u16)
    gy = to_device_bf16(gy_u16)
    shp = oracle.output_shapes_fmt(M, K, group_size, ys_layout)
    sq = SENTINEL_CODE[codes]
    mk_s = (lambda s: Guarded(s, torch.uint8, SENTINEL_E8M0)) if scales else \
        (lambda s: Guarded(s, torch.float32, float("nan")))
    outs = [Guarded(shp[0], torch.uint8, sq), mk_s(shp[1]), Guarded(shp[2], torch.uint8, sq), mk_s(shp[3])]
    fmt = (sdq.FMT_E4M3 if codes else 0) | (sdq.FMT_E8M0 if scales else 0) | \
        (sdq.FMT_YS_MG_K if ys_layout else 0)
    sdq.sdq_fuse_format(x.data_ptr(), gy.data_ptr(), *(o.t.data_ptr() for o in outs), M, K, group_size, fmt,
                        torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert sdq.sdq_device_status() == 0
    for o, name in zip(outs, ("grad_input_q", "grad_input_s", "y_q_t", "y_s_t")):
        assert o.guards_intact(), f"{name}: guard bytes overwritten"
    giq, gis, yqt, yst = (o.t.cpu().numpy() for o in outs)
    assert not (giq == sq).any() and not (yqt == sq).any(), "codes left unwritten"
    if scales:
        assert not (gis == SENTINEL_E8M0).any() and not (yst == SENTINEL_E8M0).any(), "scales left unwritten"
    else:
        assert np.isfinite(gis).all() and np.isfinite(yst).all(), "scales left unwritten"
    return giq, gis, yqt, yst


def _code_values(q, codes):
    return E4M3_VALUE[q] if codes else q.view(np.int8).astype(np.float64)


def _code_step(vals, codes):
    if not codes:
        return np.ones_like(vals)
    e = np.floor(np.log2(np.maximum(np.abs(vals), 2.0 ** -6)))
    return 2.0 ** (e - 3)       # E4M3 spacing at |v| (2^-9 below the normal range)


def _scale_values(s, scales):
    return np.ldexp(1.0, s.astype(np.int64) - 127) if scales else s.astype(np.float64)


def compare_fmt(got, ref, codes: int, scales: int, ys_layout: int, where="", group_size: int = 128,
                max_frac: float = 1e-3):
    """Assert the format tolerances; returns mismatch statistics."""
    giq, gis, yqt, yst = got
    rq, rs, ryq, rys = ref
    if ys_layout:
        yst, rys = yst.T, rys.T
    stats = {}
    for name, a, b in (("grad_input_s", gis, rs), ("y_s_t", yst, rys)):
        assert a.shape == b.shape, (name, a.shape, b.shape)
        nd = int((a != b).sum())
        stats[name] = {"n_diff": nd}
        if scales:
            d = np.abs(a.astype(np.int16) - b.astype(np.int16))
            assert d.max(initial=0) <= 1, f"{where} {name}: E8M0 bytes differ by {d.max()}"
            assert nd <= 1e-3 * a.size, f"{where} {name}: {nd} of {a.size} E8M0 scales differ"
        else:
            rel = np.abs(a.astype(np.float64) - b.astype(np.float64)) / np.abs(b.astype(np.float64))
            assert rel.max(initial=0) <= SCALE_MAX_REL, f"{where} {name}: max rel = {rel.max()}"
    G = group_size
    M = giq.shape[0]
    K = giq.shape[1] // 2
    # each code's row scale: channel c of [d_gate | d_up] is in group
    # half * ceil(K/G) + (c mod K) // G (a half may end in a shorter group)
    Kgs = (K + G - 1) // G
    c = np.arange(2 * K)
    col = (c // K) * Kgs + (c % K) // G
    for name, a, b, sa, sb in (("grad_input_q", giq, rq, gis[:, col], rs[:, col]),
                               ("y_q_t", yqt, ryq, np.repeat(yst, G, axis=1)[:, :M],
                                np.repeat(rys, G, axis=1)[:, :M])):
        assert a.shape == b.shape, (name, a.shape, b.shape)
        differ = a != b
        signed_zero = np.zeros_like(differ)
        if codes:
            signed_zero = differ & ((a & 0x7F) == 0) & ((b & 0x7F) == 0)
            differ &= ~signed_zero
        nd = int(differ.sum())
        va, vb = _code_values(a, codes), _code_values(b, codes)
        fa, fb = _scale_values(sa, scales), _scale_values(sb, scales)
        tol = _code_step(va, codes) * fa + _code_step(vb, codes) * fb
        err = np.abs(va * fa - vb * fb)
        bad = err > tol
        stats[name] = {"n_diff": nd, "frac_diff": nd / max(1, a.size), "n_out_of_step": int(bad.sum()),
                       "n_signed_zero": int(signed_zero.sum())}
        assert not bad.any(), f"{where} {name}: {int(bad.sum())} values more than a step apart"
        assert nd <= max_frac * a.size, f"{where} {name}: {nd} of {a.size} codes differ"
    return stats


# ---- the forward-side neighbour (SwiGLU forward + q8_1 rows) -----------------
#
# Tolerances, from the same arithmetic as the backward op: h = bf16 of an fp32
# computation (hardware exp2/reciprocal approximations, two roundings before
# bf16) against the oracle's fp64 value rounded once, so an h next to a bf16
# rounding boundary can round the other way: h within one bf16 step, and equal
# on all but 0.1 %; the codes within 1 (the kernel multiplies by 1/d32, the
# oracle divides), equal on all but 0.1 %; d (fp16) within a relative 2^-7
# (only a flipped amax moves it).  sum = fp16(d32 * sum(q)) is a function of
# the block's d32 and codes, which the two checks above compare with the
# oracle (a flipped amax moves d32 and, with it, up to every code of the
# block by one), so the kernel's sum is checked against its own block:
# |sum - d * sum(q)| within the fp16 rounding of d and of the product.

def run_cuda_fwd(gate_u16, up_u16, w, limit=0.0, ld_pad=0):
    """The forward entry on the device; gate/up may be views (row stride kept
    if ld_pad is 0, else copied into rows padded by ld_pad elements); h and
    q8 are guarded and prefilled.  Returns numpy (h uint16 [rows, inter],
    q8 uint8 [rows, inter/32, 36])."""
    import swiglu_backward_int8_b200 as sdq
    rows, inter = gate_u16.shape

    def dev(a):
        t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
        if ld_pad:
            buf = torch.zeros((rows, inter + ld_pad), dtype=torch.bfloat16, device="cuda")
            buf[:, :inter] = t
            return buf[:, :inter]
        return t

    g, u = dev(gate_u16), dev(up_u16)
    wd = torch.from_numpy(np.ascontiguousarray(w, np.float32)).cuda() if w is not None else None
    hb = Guarded((rows, inter), torch.int16, -1)              # 0xFFFF: a NaN bf16, never written
    qb = Guarded((rows, inter // 32, 36), torch.uint8, 0xA5)
    sdq.swiglu_q8_1(g, u, wd, limit, hb.t.view(torch.bfloat16), qb.t)
    torch.cuda.synchronize()
    assert hb.guards_intact() and qb.guards_intact(), "guard bytes overwritten"
    h = hb.t.cpu().numpy().view(np.uint16)
    q8 = qb.t.cpu().numpy()
    assert not (h == 0xFFFF).any(), "h left unwritten"
    return h, q8


def _bf16_ordinal(b):
    """bf16 bits as signed-magnitude ordinals (adjacent values one apart)."""
    b = b.astype(np.int64)
    return np.where(b & 0x8000, -(b & 0x7FFF), b)


def compare_bf16(got, ref, name, where=""):
    """bf16 bit arrays: at most one bf16 step apart everywhere, and apart on
    at most 0.1 % of the elements (the same rounding-boundary argument as the
    int8 codes; +0 and -0 count as equal)."""
    assert got.shape == ref.shape
    d = np.abs(_bf16_ordinal(got) - _bf16_ordinal(ref))
    n = int((d != 0).sum())
    assert d.max(initial=0) <= 1, f"{where} {name}: {d.max()} bf16 steps apart"
    assert n <= 1e-3 * got.size, f"{where} {name}: {n} of {got.size} differ"
    return n


def compare_fwd(got, ref, where=""):
    h, q8 = got
    rh, rq8 = ref
    assert h.shape == rh.shape and q8.shape == rq8.shape
    nh = compare_bf16(h, rh, "h", where)
    q, rq = q8[..., 4:].view(np.int8).astype(np.int16), rq8[..., 4:].view(np.int8).astype(np.int16)
    dq = np.abs(q - rq)
    nq = int((dq != 0).sum())
    assert dq.max(initial=0) <= 1, f"{where} codes: {dq.max()} apart"
    assert nq <= 1e-3 * q.size, f"{where} codes: {nq} of {q.size} differ"
    d = q8[..., 0:2].copy().view(np.float16)[..., 0].astype(np.float64)
    rd = rq8[..., 0:2].copy().view(np.float16)[..., 0].astype(np.float64)
    s = q8[..., 2:4].copy().view(np.float16)[..., 0].astype(np.float64)
    rs = rq8[..., 2:4].copy().view(np.float16)[..., 0].astype(np.float64)
    both_zero = (d == 0) & (rd == 0)
    rel = np.where(both_zero, 0.0, np.abs(d - rd) / np.maximum(np.abs(rd), 1e-300))
    assert rel.max(initial=0) <= 2.0 ** -7, f"{where} d: rel {rel.max()}"
    ulp = lambda v: np.ldexp(1.0, np.floor(np.log2(np.maximum(np.abs(v), 2.0 ** -14))).astype(int) - 10)
    ds = np.abs(s - rs)
    qsum = q.sum(axis=-1)
    own = d * qsum                            # fp16 d is within half its spacing of d32
    tol = np.abs(qsum) * ulp(d) / 2 + ulp(s) / 2 + np.abs(own) * 2.0 ** -40
    bad = np.abs(s - own) > tol
    assert not bad.any(), f"{where} sum: {int(bad.sum())} blocks off their own d * sum(q)"
    same = (q == rq).all(axis=-1) & (d == rd)  # where the block agrees, the sum must too
    assert np.array_equal(s[same], rs[same]), f"{where} sum differs on blocks that agree"
    del ds
    return {"h_n_diff": nh, "q_n_diff": nq, "d_n_diff": int((d != rd).sum()), "s_n_diff": int((s != rs).sum())}

// The forward-side neighbour of the backward op, for sm_100a: SwiGLU forward
// plus q8_1 row quantization of its output (the activation path whose
// launcher is kquant_swiglu_q8_1_rows on the page with the K-quant kernels:
// h = bf16(swiglu(gate, up) * w[row]), then the q8_1 blocks of those bf16
// rows; a block is 32 int8 + half2 (d, sum), 36 bytes).
//
//   h[m, k]  = bf16( silu(g') * u' * w[m] )      g', u': gate and up, clamped when limit > 0
//                                                (g' <= limit, |u'| <= limit)
//   per block of 32 consecutive h of a row:
//     d32 = fl32(amax / 127), q = round-half-even(h * (1/d32)) in [-127, 127],
//     d = fp16(d32), sum = fp16(d32 * sum(q)); an all-zero block is all zero.
//
// A pure streaming kernel (4 bytes read, 3.125 written per element): no
// shared memory and no tensor cores.  A warp takes 256 consecutive elements
// of one row (8 blocks); a lane holds 8 of them (one 16-byte load of gate and
// of up, one 16-byte store of h), so a block is 4 neighbouring lanes and its
// amax and code sum take two shuffles.  A persistent grid walks the
// (row, 256-element chunk) units, two per warp iteration (both units' loads
// in flight before either is computed).
#pragma once

#include <cuda_fp16.h>

#include <cstdint>

#include "sdq_ptx.cuh"

namespace sdq {
namespace fwd {

constexpr int kThreads = 256;
constexpr int kUnit = 256;          // elements per warp unit
constexpr int kBlock = 32;          // q8_1 block
constexpr int kBlockBytes = 36;

struct Params {
  const uint8_t* gate;   // bf16 rows, ld_gate elements apart
  const uint8_t* up;
  const float* w;        // [rows] or null
  uint8_t* h;            // bf16 rows, ld_h elements apart
  uint8_t* q8;           // [rows, inter/32] blocks, contiguous
  int64_t rows;
  int64_t ld_gate, ld_up, ld_h;
  int32_t inter;
  int32_t units_per_row;
  float limit;           // clamp when > 0
  int32_t clamp;         // limit > 0 (false for NaN)
};

__device__ __forceinline__ float2 bf2(uint32_t v) { return make_float2(bf16_lo(v), bf16_hi(v)); }

// silu(g) * u * w for g < -80, where sigma(g) = 1 / (1 + e^-g) leaves the
// normal fp32 range (e^-g overflows, or the approximate reciprocal flushes a
// subnormal sigma to zero) although the product can still be a normal bf16:
// sigma is computed at a 2^64 scale (e^-g * 2^-64 is finite up to g = -132,
// and 1 is negligible beside it) and the scale comes off in the last IEEE
// product, which keeps subnormal results.
__device__ __noinline__ float silu_mul_deep_negative(float g, float u, float w) {
  constexpr float kNegLog2e = -1.4426950408889634f;
  constexpr float kTwoM64 = 5.42101086242752217e-20f;   // 2^-64
  const float s64 = rcp_approx(ex2_approx(fmaf(g, kNegLog2e, -64.0f)));   // sigma(g) * 2^64
  return __fmul_rn(__fmul_rn(__fmul_rn(g * s64, u), w), kTwoM64);
}

// Eight h values (4 bf16 pairs) from 8 gate and up values and the row weight.
__device__ __forceinline__ void swiglu8(const uint4& g, const uint4& u, float w, const Params& p,
                                        uint32_t (&h)[4]) {
  constexpr float kNegLog2e = -1.4426950408889634f;
  const uint32_t gw[4] = {g.x, g.y, g.z, g.w};
  const uint32_t uw[4] = {u.x, u.y, u.z, u.w};
  const float2 one = make_float2(1.0f, 1.0f);
  const float2 ww = make_float2(w, w);
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    float2 gg = bf2(gw[c]), uu = bf2(uw[c]);
    if (p.clamp) {
      gg = make_float2(fminf(gg.x, p.limit), fminf(gg.y, p.limit));
      uu = make_float2(fminf(fmaxf(uu.x, -p.limit), p.limit), fminf(fmaxf(uu.y, -p.limit), p.limit));
    }
    const float2 xl = __fmul2_rn(gg, make_float2(kNegLog2e, kNegLog2e));
    const float2 d = __fadd2_rn(make_float2(ex2_approx(xl.x), ex2_approx(xl.y)), one);
    const float2 sg = make_float2(rcp_approx(d.x), rcp_approx(d.y));
    float2 y = __fmul2_rn(__fmul2_rn(__fmul2_rn(gg, sg), uu), ww);
    if (fminf(gg.x, gg.y) < -80.0f) {   // rare: sigma below the normal fp32 range
      if (gg.x < -80.0f) y.x = silu_mul_deep_negative(gg.x, uu.x, w);
      if (gg.y < -80.0f) y.y = silu_mul_deep_negative(gg.y, uu.y, w);
    }
    h[c] = pack_bf16x2(y.x, y.y);
  }
}

// One warp unit after its loads: h, its store, and the unit's 8 q8_1 blocks.
// tab: per bf16 mantissa m, (fl((1 + m/128)/127), its reciprocal); for a
// block amax (1 + m/128) * 2^e with a bf16 exponent field >= 10 the scale
// fl(amax/127) and 1/scale are those entries with 2^e moved into the
// exponent fields, exactly (both stay normal floats).
__device__ __forceinline__ void finish_unit(const Params& p, const float2* tab, const uint4& g,
                                            const uint4& u, float w, int64_t m, int k0, bool active,
                                            int lane) {
  constexpr unsigned kFull = 0xffffffffu;
  uint32_t h[4] = {0u, 0u, 0u, 0u};
  if (active) {
    swiglu8(g, u, w, p, h);
    st_cs_v4(reinterpret_cast<int8_t*>(p.h + 2 * (m * p.ld_h + k0)), make_uint4(h[0], h[1], h[2], h[3]));
  }
  // block amax over the 4 lanes of the block (bf16, exact)
  uint32_t a = absmax_bf16x2(absmax_bf16x2(h[0], h[1]), absmax_bf16x2(h[2], h[3]));
  a = absmax_bf16x2(a, __shfl_xor_sync(kFull, a, 1));
  a = absmax_bf16x2(a, __shfl_xor_sync(kFull, a, 2));
  const uint32_t ab = (a & 0x7FFFu) > ((a >> 16) & 0x7FFFu) ? (a & 0x7FFFu) : ((a >> 16) & 0x7FFFu);
  float d = 0.0f;
  uint32_t qw[2] = {0u, 0u};
  int qs = 0;
  if (ab >= 0x0500u) {   // amax >= 2^-117: the table path, then multiply by 1/d32
    const float2 t = tab[ab & 127u];
    const int sh = (static_cast<int>(ab >> 7) - 127) << 23;
    d = __int_as_float(__float_as_int(t.x) + sh);
    const float inv = __int_as_float(__float_as_int(t.y) - sh);
    const float2 iv = make_float2(inv, inv);
    const float2 magic = make_float2(12582912.0f, 12582912.0f);
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      const float2 q0 = __ffma2_rn(bf2(h[2 * c]), iv, magic);
      const float2 q1 = __ffma2_rn(bf2(h[2 * c + 1]), iv, magic);
      qw[c] = pack_low_bytes(__float_as_uint(q0.x), __float_as_uint(q0.y), __float_as_uint(q1.x),
                             __float_as_uint(q1.y));
      qs += (static_cast<int>(__float_as_uint(q0.x)) - 0x4B400000) +
            (static_cast<int>(__float_as_uint(q0.y)) - 0x4B400000) +
            (static_cast<int>(__float_as_uint(q1.x)) - 0x4B400000) +
            (static_cast<int>(__float_as_uint(q1.y)) - 0x4B400000);
    }
  } else if (ab != 0u) {  // tiny block (1/d32 may overflow): divide, as the definition reads
    d = __fdiv_rn(__uint_as_float(ab << 16), 127.0f);
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      int qb[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t pr = h[2 * c + (e >> 1)];
        const float v = (e & 1) ? bf16_hi(pr) : bf16_lo(pr);
        qb[e] = static_cast<int>(fminf(fmaxf(rintf(__fdiv_rn(v, d)), -127.0f), 127.0f));
        qs += qb[e];
      }
      qw[c] = (qb[0] & 0xFF) | ((qb[1] & 0xFF) << 8) | ((qb[2] & 0xFF) << 16) |
              (static_cast<uint32_t>(qb[3] & 0xFF) << 24);
    }
  }
  qs += __shfl_xor_sync(kFull, qs, 1);
  qs += __shfl_xor_sync(kFull, qs, 2);
  if (active) {
    uint8_t* b = p.q8 + (m * (p.inter / kBlock) + k0 / kBlock) * kBlockBytes;
    const int part = lane & 3;                          // 8 codes at bytes 4 + 8 * part
    *reinterpret_cast<uint32_t*>(b + 4 + 8 * part) = qw[0];
    *reinterpret_cast<uint32_t*>(b + 8 + 8 * part) = qw[1];
    if (part == 0) {   // an all-zero block has d = 0 and qs = 0: both halves 0
      const __half dh = __float2half_rn(d);
      const __half sh = __double2half(static_cast<double>(d) * static_cast<double>(qs));
      *reinterpret_cast<uint32_t*>(b) = static_cast<uint32_t>(__half_as_ushort(dh)) |
                                        (static_cast<uint32_t>(__half_as_ushort(sh)) << 16);
    }
  }
}

__global__ void __launch_bounds__(kThreads)
    swiglu_q8_1_kernel(const Params p) {
  __shared__ float2 tab[128];
  const int lane = threadIdx.x & 31;
  if (threadIdx.x < 128) {
    const float t = __fdiv_rn(1.0f + static_cast<float>(threadIdx.x) * (1.0f / 128.0f), 127.0f);
    tab[threadIdx.x] = make_float2(t, __frcp_rn(t));
  }
  __syncthreads();
  const int64_t warp0 = (static_cast<int64_t>(blockIdx.x) * kThreads + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * kThreads) >> 5;
  const int64_t units = p.rows * p.units_per_row;
  // The warp's units are warp0, warp0 + nwarps, ...; (row, chunk) of the next
  // one is (row, chunk) + (dm, dc) with a carry, so no division per unit.
  const int upr = p.units_per_row;
  int64_t m = warp0 / upr;
  int c = static_cast<int>(warp0 - m * upr);
  const int64_t dm = nwarps / upr;
  const int dc = static_cast<int>(nwarps - dm * upr);
  grid_dependency_wait();   // inputs may come from the previous kernel in the stream
  grid_launch_dependents();
  // two units per iteration: both units' loads are in flight before either is computed
  for (int64_t unit = warp0; unit < units; unit += 2 * nwarps) {
    int64_t m1 = m + dm;
    int c1 = c + dc;
    if (c1 >= upr) { c1 -= upr; ++m1; }
    const bool has1 = unit + nwarps < units;            // warp-uniform
    const int k0 = c * kUnit + lane * 8, k1 = c1 * kUnit + lane * 8;
    const bool act0 = k0 < p.inter, act1 = has1 && k1 < p.inter;   // whole blocks: inter % 32 == 0
    uint4 g0 = make_uint4(0, 0, 0, 0), u0 = g0, g1 = g0, u1 = g0;
    float w0 = 1.0f, w1 = 1.0f;
    if (act0) {
      g0 = *reinterpret_cast<const uint4*>(p.gate + 2 * (m * p.ld_gate + k0));
      u0 = *reinterpret_cast<const uint4*>(p.up + 2 * (m * p.ld_up + k0));
      if (p.w) w0 = p.w[m];
    }
    if (act1) {
      g1 = *reinterpret_cast<const uint4*>(p.gate + 2 * (m1 * p.ld_gate + k1));
      u1 = *reinterpret_cast<const uint4*>(p.up + 2 * (m1 * p.ld_up + k1));
      if (p.w) w1 = p.w[m1];
    }
    finish_unit(p, tab, g0, u0, w0, m, k0, act0, lane);
    if (has1) finish_unit(p, tab, g1, u1, w1, m1, k1, act1, lane);
    m = m1 + dm;
    c = c1 + dc;
    if (c >= upr) { c -= upr; ++m; }
  }
}

}  // namespace fwd
}  // namespace sdq

// CPU oracle for silu_dot_fwd_bwd_quant_fuse -- TEST INFRASTRUCTURE ONLY.
//
// Only the tests, the smoke check and the CPU-baseline leg of the bench may
// load this code.  It is a plain, slow, single-threaded restatement of what the
// op computes, written to be checked by eye; it shares no code, header, table
// or constant with the CUDA library.
//
// What it follows ("kernelgen-challenge-9-task3-silu-quant"):
//   * entry point section: the op takes x, grad_y and four preallocated
//     outputs grad_input_q, grad_input_s, y_q_t, y_s_t, with group_size = 128
//     by default;
//   * outputs section: it recomputes the SwiGLU forward value
//     y = silu(gate) * up, computes the backward gradients, and writes
//     [d_gate, d_up] quantized row-wise in 128-channel groups and y transposed
//     and quantized in 128-token groups;
//   * constraints list, third item: every value takes a bf16 round-trip
//     before it is quantized.
// Readings where the page is silent (each one is listed with its reason in
// the design notes): x = [gate | up] along channels; d_gate =
// grad_y*up*silu'(gate), d_up = grad_y*silu(gate) (the derivatives of
// y = silu(gate)*up); math in fp64, each of y, d_gate, d_up rounded to bf16
// once, to nearest even; scale = amax/127 in fp32; q = round-half-even of the
// fp32 quotient v/scale, clamped to [-127, 127]; an all-zero group gets
// scale 1 and q 0; a tail token group (M % G != 0) is quantized over the
// tokens it holds, and likewise a channel group cut short by the end of its
// half of [d_gate | d_up] when G does not divide K; grad_input_s is
// [M, 2 ceil(K/G)] (d_gate groups first) and y_s_t is [K, ceil(M/G)].
//
// How each function is pinned (tests/test_oracle_pins.py):
//   oracle_bf16_rne        brute force over the neighbouring bf16 values with
//                          exact rational arithmetic; float32 inputs against
//                          torch's float32->bfloat16 conversion.
//   oracle_sigmoid/silu    library expit, closed forms (sigma(0)=1/2,
//                          sigma(-g)=1-sigma(g), silu(g)-silu(-g)=g).
//   oracle_silu_grad       central finite difference of oracle_silu.
//   oracle_swiglu_bwd_fp64 torch float64 autograd of sum(grad_y*silu(g)*u);
//                          finite differences of y in g and u.
//   oracle_quant_group     (the page's format of oracle_quant_group_fmt, the
//                          one quantizer) exact-rational check that scale is
//                          amax/127 rounded once, nearest-integer brute
//                          force, exact ties to even, symmetry, monotonicity.
//   whole op               closed-form hand-derived cases (gate = 0, gate
//                          large), layout/transposition patterns, tail and
//                          zero groups, and a hand-derived golden fixture.
//
// Output formats beyond the page's (INT8 codes, fp32 scales, y_s_t [K, Mg]);
// the page only says the outputs feed quantized GEMMs, so these follow public
// format definitions, each reading listed in the design notes:
//   * FP8 codes: OCP 8-bit floating point, E4M3 variant (sign, 4 exponent
//     bits with bias 7, 3 mantissa bits; no infinities; S.1111.111 is NaN, so
//     the largest finite magnitude is 448).  scale = fl32(amax / 448); a code
//     is the nearest E4M3 value of the fp32 quotient v / scale, ties to an
//     even mantissa, magnitudes above 448 saturated to 448.
//   * E8M0 scales: OCP Microscaling (MX) scale format, an unsigned biased
//     exponent byte e with value 2^(e - 127).  The scale is the smallest
//     power of two not below fl32(amax / Qmax) (Qmax = 127 for INT8 codes,
//     448 for E4M3), so no element exceeds the code range, clamped to
//     [2^-127, 2^127]; an all-zero group gets 2^0 (byte 127).
//   * In every format an all-zero group has scale 1 and each code is that of
//     v / 1: zero, with v's sign in E4M3 (0x80 for -0.0).
//   * y_s_t [Mg, K]: token group i, channel k at i * K + k.
// The forward-side neighbour (the q8_1 activation path on the page whose
// launcher is kquant_swiglu_q8_1_rows: "h = bf16(swiglu(gate, up) * w[row]),
// then the q8_1 blocks of those bf16 rows"; a block_q8_1 is "32 int8 + half2
// (d, sum)", 36 bytes).  Readings where that page is silent: swiglu(g, u) =
// silu(g) * u as in the backward op, with `limit` > 0 clamping gate to at
// most limit and up to [-limit, limit] first (limit <= 0 or NaN: no clamp);
// h in fp64 rounded once to bf16; per block of 32 consecutive h values of a
// row, d32 = fl32(amax / 127), q = round-half-even(fl32(h / d32)) in
// [-127, 127], stored d = fp16(d32) and sum = fp16(d32 * sum(q)) (the exact
// product rounded once: the sum of the block's dequantized values), both
// nearest-even; an all-zero block has d = sum = 0 and q = 0; the block is
// half2 (d, sum) first, then the 32 codes.  Pins: tests/test_oracle_fwd.py.
//
// A quantized grad_y (oracle_dequant_grad_y, oracle_swiglu_bwd_bf16_dy,
// oracle_silu_dot_fwd_bwd_quant_fuse_qgrad; the reading is stated above
// them).  Pins (tests/test_oracle_qgrad.py): with power-of-two scales every
// q * s is a bf16 value, so the whole op must equal the pinned bf16-grad_y op
// on that bf16 grad_y bit for bit; with any scales the first stage must equal
// torch's float64 autograd of sum(q*s * silu(g) * u) rounded by the pinned
// bf16 rounding.
//
// Pins (tests/test_oracle_formats.py): oracle_e4m3_rne against torch's
// float8_e4m3fn conversion inside the finite range and against brute force
// over all 127 finite magnitudes with exact rationals; oracle_e8m0_ceil
// against brute force over the 255 powers of two; oracle_quant_group_fmt
// against exact-rational brute force of each definition and its invariants
// (scale/2 < amax/Qmax <= scale, |code| <= Qmax, the amax element reaches
// the top binade); the whole op against the pinned INT8 whole op (default
// format), a transposition identity between the two y_s_t layouts, and
// closed-form cases.

#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

namespace {

// bf16 bit pattern -> float (exact: bf16 is the upper half of a float32).
float bf16_to_float(uint16_t b) {
  uint32_t u = static_cast<uint32_t>(b) << 16;
  float f;
  std::memcpy(&f, &u, sizeof f);
  return f;
}

uint16_t float_bits_hi(float f) {
  uint32_t u;
  std::memcpy(&u, &f, sizeof u);
  return static_cast<uint16_t>(u >> 16);
}

}  // namespace

extern "C" {

// Round a double to the nearest bf16 (8 significant bits, float32's exponent
// range, subnormals kept), ties to even, in ONE rounding step.
uint16_t oracle_bf16_rne(double v) {
  if (std::isnan(v)) return 0x7FC0;
  const uint16_t sign = std::signbit(v) ? 0x8000 : 0x0000;
  const double a = std::fabs(v);
  if (a == 0.0) return sign;
  if (std::isinf(a)) return sign | 0x7F80;
  int e = std::ilogb(a);            // 2^e <= a < 2^(e+1)
  if (e < -126) e = -126;           // below the normal range the spacing stays 2^-133
  const double ulp = std::ldexp(1.0, e - 7);
  const double r = std::nearbyint(a / ulp) * ulp;  // a/ulp is exact; nearbyint ties to even
  if (r >= std::ldexp(1.0, 128)) return sign | 0x7F80;  // rounds past the largest finite bf16
  return sign | float_bits_hi(static_cast<float>(r));  // r is a bf16 value: exact in float
}

double oracle_sigmoid(double g) { return 1.0 / (1.0 + std::exp(-g)); }

double oracle_silu(double g) { return g * oracle_sigmoid(g); }

// d/dg [g * sigma(g)] = sigma(g) * (1 + g * (1 - sigma(g))).
double oracle_silu_grad(double g) {
  const double s = oracle_sigmoid(g);
  return s * (1.0 + g * (1.0 - s));
}

// One element of the forward recompute and the backward, in fp64, before any
// rounding:  y = silu(g)*u,  d_gate = dy*u*silu'(g),  d_up = dy*silu(g).
void oracle_swiglu_bwd_fp64(double g, double u, double dy, double* y,
                            double* d_gate, double* d_up) {
  const double silu = oracle_silu(g);
  *y = silu * u;
  *d_gate = dy * u * oracle_silu_grad(g);
  *d_up = dy * silu;
}

// First stage on grad_y given as fp64 values dy [M, K]: the bf16 values y,
// d_gate, d_up ([M, K] each, bf16 bits) from x = [gate | up] ([M, 2K]).
void oracle_swiglu_bwd_bf16_dy(const uint16_t* x, const double* dy, int64_t M, int64_t K,
                               uint16_t* y, uint16_t* d_gate, uint16_t* d_up) {
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t k = 0; k < K; ++k) {
      const double g = bf16_to_float(x[m * 2 * K + k]);
      const double u = bf16_to_float(x[m * 2 * K + K + k]);
      double yv, dg, du;
      oracle_swiglu_bwd_fp64(g, u, dy[m * K + k], &yv, &dg, &du);
      y[m * K + k] = oracle_bf16_rne(yv);
      d_gate[m * K + k] = oracle_bf16_rne(dg);
      d_up[m * K + k] = oracle_bf16_rne(du);
    }
  }
}

// First stage on a bf16 grad_y ([M, K] bf16 bits): its exact values.
void oracle_swiglu_bwd_bf16(const uint16_t* x, const uint16_t* grad_y,
                            int64_t M, int64_t K, uint16_t* y,
                            uint16_t* d_gate, uint16_t* d_up) {
  std::vector<double> dy(M * K);
  for (int64_t i = 0; i < M * K; ++i) dy[i] = bf16_to_float(grad_y[i]);
  oracle_swiglu_bwd_bf16_dy(x, dy.data(), M, K, y, d_gate, d_up);
}

// ---- output formats ---------------------------------------------------------

// Nearest OCP E4M3 code of a double, ties to an even mantissa, in one rounding
// step; magnitudes above 448 saturate to 448 (code 0x7E); NaN gives 0x7F.
uint8_t oracle_e4m3_rne(double v) {
  if (std::isnan(v)) return 0x7F;
  const uint8_t sign = std::signbit(v) ? 0x80 : 0x00;
  const double a = std::fabs(v);
  if (a > 448.0) return sign | 0x7E;
  if (a == 0.0) return sign;
  int e = std::ilogb(a);            // 2^e <= a < 2^(e+1)
  if (e < -6) e = -6;               // below the normal range the spacing stays 2^-9
  const double ulp = std::ldexp(1.0, e - 3);
  const double r = std::nearbyint(a / ulp) * ulp;  // a/ulp is exact; nearbyint ties to even
  if (r < std::ldexp(1.0, -6))      // subnormal: exponent field 0, mantissa r / 2^-9
    return sign | static_cast<uint8_t>(r / std::ldexp(1.0, -9));
  const int re = std::ilogb(r);     // r may have rounded up into the next binade
  const int mant = static_cast<int>(r / std::ldexp(1.0, re - 3)) - 8;
  return sign | static_cast<uint8_t>(((re + 7) << 3) | mant);
}

// Value of an E4M3 code (NaN for S.1111.111).
double oracle_e4m3_value(uint8_t c) {
  const double sign = (c & 0x80) ? -1.0 : 1.0;
  const int ef = (c >> 3) & 0xF;
  const int mf = c & 0x7;
  if (ef == 0xF && mf == 0x7) return std::nan("");
  if (ef == 0) return sign * std::ldexp(static_cast<double>(mf), -9);
  return sign * std::ldexp(1.0 + mf / 8.0, ef - 7);
}

// E8M0 byte of the smallest power of two >= s (s > 0), clamped to
// [2^-127, 2^127]: value 2^(e - 127).
uint8_t oracle_e8m0_ceil(float s) {
  const double d = static_cast<double>(s);
  int k = std::ilogb(d);                    // 2^k <= d < 2^(k+1)
  if (std::ldexp(1.0, k) < d) k += 1;       // not a power of two: round up
  if (k < -127) k = -127;
  if (k > 127) k = 127;
  return static_cast<uint8_t>(k + 127);
}

double oracle_e8m0_value(uint8_t e) { return std::ldexp(1.0, static_cast<int>(e) - 127); }

// Quantize one group of n bf16 values (element i at v[i*stride]) in a chosen
// format.  codes: 0 INT8 (q as int8 bits), 1 E4M3; scales: 0 fp32 (*scale is
// a float), 1 E8M0 (*scale is one byte).  All-zero group: codes 0, scale 1.
void oracle_quant_group_fmt(const uint16_t* v, int64_t n, int64_t stride, uint8_t* q,
                            int64_t qstride, void* scale, int codes, int scales) {
  const float qmax = codes ? 448.0f : 127.0f;
  float amax = 0.0f;
  for (int64_t i = 0; i < n; ++i) {
    const float a = std::fabs(bf16_to_float(v[i * stride]));
    if (a > amax) amax = a;
  }
  double s;   // the scale's value
  if (amax == 0.0f) {
    s = 1.0;
  } else {
    const float s32 = amax / qmax;   // fp32 division, rounded once
    s = scales ? oracle_e8m0_value(oracle_e8m0_ceil(s32)) : static_cast<double>(s32);
  }
  if (scales) *static_cast<uint8_t*>(scale) = oracle_e8m0_ceil(static_cast<float>(s));
  else *static_cast<float*>(scale) = static_cast<float>(s);
  // Every group, the all-zero one included (scale 1), codes v / scale: a
  // -0.0 element therefore gets the E4M3 negative zero, as a cast of the
  // quotient would give.
  for (int64_t i = 0; i < n; ++i) {
    // the quotient rounded once to fp32 (exact for a power-of-two scale)
    const float t = static_cast<float>(static_cast<double>(bf16_to_float(v[i * stride])) / s);
    uint8_t c;
    if (codes) {
      c = oracle_e4m3_rne(t);
    } else {
      float r = std::nearbyint(t);
      if (r > 127.0f) r = 127.0f;
      if (r < -127.0f) r = -127.0f;
      c = static_cast<uint8_t>(static_cast<int8_t>(r));
    }
    q[i * qstride] = c;
  }
}

// The page's format of oracle_quant_group_fmt: INT8 codes (q as int8),
// fp32 scale.  amax = max |v|; all-zero -> scale 1, q 0; else scale =
// amax/127 (fp32 division) and q = clamp(round-half-even(v/scale), -127, 127)
// with the quotient taken in fp32.  Writes q[i*qstride] and *scale.
void oracle_quant_group(const uint16_t* v, int64_t n, int64_t stride,
                        int8_t* q, int64_t qstride, float* scale) {
  oracle_quant_group_fmt(v, n, stride, reinterpret_cast<uint8_t*>(q), qstride, scale, 0, 0);
}

// The whole op in a chosen format.  codes / scales as in
// oracle_quant_group_fmt; ys_layout: 0 y_s_t [K, Mg], 1 [Mg, K].  Code
// arrays are bytes; scale arrays are fp32 or one byte per scale.
static void quantize_outputs_fmt(const uint16_t* y, const uint16_t* dg, const uint16_t* du,
                                 uint8_t* grad_input_q, void* grad_input_s, uint8_t* y_q_t,
                                 void* y_s_t, int64_t M, int64_t K, int64_t G, int codes,
                                 int scales, int ys_layout);

int oracle_silu_dot_fwd_bwd_quant_fuse_fmt(const uint16_t* x, const uint16_t* grad_y,
                                           uint8_t* grad_input_q, void* grad_input_s,
                                           uint8_t* y_q_t, void* y_s_t, int64_t M, int64_t K,
                                           int64_t group_size, int codes, int scales,
                                           int ys_layout) {
  const int64_t G = group_size;
  if (G < 1 || M < 0 || K < 0) return -1;
  if (codes < 0 || codes > 1 || scales < 0 || scales > 1 || ys_layout < 0 || ys_layout > 1) return -1;
  if (M == 0 || K == 0) return 0;
  std::vector<uint16_t> y(M * K), dg(M * K), du(M * K);
  oracle_swiglu_bwd_bf16(x, grad_y, M, K, y.data(), dg.data(), du.data());
  quantize_outputs_fmt(y.data(), dg.data(), du.data(), grad_input_q, grad_input_s, y_q_t, y_s_t,
                       M, K, G, codes, scales, ys_layout);
  return 0;
}

// The whole op in the page's format (INT8 codes, fp32 scales, y_s_t
// [K, ceil(M/G)]): the format op above with codes 0, scales 0, layout 0.
// Returns 0, or -1 for arguments the definition does not cover
// (group_size < 1, negative sizes).
//   grad_input_q [M, 2K] int8     grad_input_s [M, 2 ceil(K/G)] fp32
//   y_q_t        [K, M]  int8     y_s_t        [K, ceil(M/G)] fp32
int oracle_silu_dot_fwd_bwd_quant_fuse(const uint16_t* x, const uint16_t* grad_y,
                                       int8_t* grad_input_q, float* grad_input_s,
                                       int8_t* y_q_t, float* y_s_t, int64_t M,
                                       int64_t K, int64_t group_size) {
  return oracle_silu_dot_fwd_bwd_quant_fuse_fmt(x, grad_y, reinterpret_cast<uint8_t*>(grad_input_q),
                                                grad_input_s, reinterpret_cast<uint8_t*>(y_q_t), y_s_t,
                                                M, K, group_size, 0, 0, 0);
}

// ---- grad_y handed over already quantized (the chained backward) -------------
//
// Reading: the upstream step hands grad_y over in the row-group format this
// op itself writes for grad_input: INT8 codes q [M, K] and fp32 scales
// s [M, ceil(K/128)], one per token and 128 consecutive channels (the last
// group of a row holds what is left); the value it stands for is q * s
// (exact in fp64: 8 x 24 significant bits).

// dy[m, k] = q[m, k] * s[m, k / 128].
void oracle_dequant_grad_y(const int8_t* q, const float* s, int64_t M, int64_t K, double* dy) {
  const int64_t Kg = (K + 127) / 128;
  for (int64_t m = 0; m < M; ++m)
    for (int64_t k = 0; k < K; ++k)
      dy[m * K + k] = static_cast<double>(q[m * K + k]) * static_cast<double>(s[m * Kg + k / 128]);
}

// The whole op with a quantized grad_y, outputs as in
// oracle_silu_dot_fwd_bwd_quant_fuse_fmt.
int oracle_silu_dot_fwd_bwd_quant_fuse_qgrad(const uint16_t* x, const int8_t* grad_y_q,
                                             const float* grad_y_s, uint8_t* grad_input_q,
                                             void* grad_input_s, uint8_t* y_q_t, void* y_s_t,
                                             int64_t M, int64_t K, int64_t group_size, int codes,
                                             int scales, int ys_layout) {
  const int64_t G = group_size;
  if (G < 1 || M < 0 || K < 0) return -1;
  if (codes < 0 || codes > 1 || scales < 0 || scales > 1 || ys_layout < 0 || ys_layout > 1) return -1;
  if (M == 0 || K == 0) return 0;
  std::vector<double> dy(M * K);
  oracle_dequant_grad_y(grad_y_q, grad_y_s, M, K, dy.data());
  std::vector<uint16_t> y(M * K), dg(M * K), du(M * K);
  oracle_swiglu_bwd_bf16_dy(x, dy.data(), M, K, y.data(), dg.data(), du.data());
  quantize_outputs_fmt(y.data(), dg.data(), du.data(), grad_input_q, grad_input_s, y_q_t, y_s_t,
                       M, K, G, codes, scales, ys_layout);
  return 0;
}

// The two quantizations of the first stage's bf16 y, d_gate, d_up.  Row
// groups are taken within each half of [d_gate | d_up]: ceil(K/G) groups of
// G channels per half, the last one holding the K - (ceil(K/G) - 1) * G
// channels left when G does not divide K; grad_input_s is [M, 2 ceil(K/G)],
// d_gate's groups first.
static void quantize_outputs_fmt(const uint16_t* y, const uint16_t* dg, const uint16_t* du,
                                 uint8_t* grad_input_q, void* grad_input_s, uint8_t* y_q_t,
                                 void* y_s_t, int64_t M, int64_t K, int64_t G, int codes,
                                 int scales, int ys_layout) {
  const int64_t Kg = (K + G - 1) / G;
  const int64_t Mg = (M + G - 1) / G;
  const int64_t sb = scales ? 1 : 4;   // bytes per scale
  uint8_t* gis = static_cast<uint8_t*>(grad_input_s);
  uint8_t* yst = static_cast<uint8_t*>(y_s_t);
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t j = 0; j < 2 * Kg; ++j) {
      const uint16_t* src = (j < Kg) ? &dg[m * K + j * G] : &du[m * K + (j - Kg) * G];
      const int64_t c0 = (j < Kg) ? j * G : (j - Kg) * G;   // first channel within its half
      const int64_t n = (K - c0 < G) ? K - c0 : G;
      oracle_quant_group_fmt(src, n, 1, &grad_input_q[m * 2 * K + (j < Kg ? 0 : K) + c0], 1,
                             gis + (m * 2 * Kg + j) * sb, codes, scales);
    }
  }
  for (int64_t k = 0; k < K; ++k) {
    for (int64_t i = 0; i < Mg; ++i) {
      const int64_t t0 = i * G;
      const int64_t n = (M - t0 < G) ? (M - t0) : G;
      const int64_t si = ys_layout ? (i * K + k) : (k * Mg + i);
      oracle_quant_group_fmt(&y[t0 * K + k], n, K, &y_q_t[k * M + t0], 1, yst + si * sb, codes,
                             scales);
    }
  }
}

// ---- forward-side neighbour: SwiGLU forward + q8_1 rows -----------------------

// Nearest IEEE binary16 of a double, ties to even, subnormals kept, overflow
// to infinity; returns the bit pattern.
uint16_t oracle_fp16_rne(double v) {
  if (std::isnan(v)) return 0x7E00;
  const uint16_t sign = std::signbit(v) ? 0x8000 : 0x0000;
  const double a = std::fabs(v);
  if (a == 0.0) return sign;
  int e = std::ilogb(a);
  if (e < -14) e = -14;                      // below the normal range the spacing stays 2^-24
  const double ulp = std::ldexp(1.0, e - 10);
  const double r = std::nearbyint(a / ulp) * ulp;
  if (r >= 65520.0) return sign | 0x7C00;   // 65504 + half its spacing rounds up to infinity
  if (r < std::ldexp(1.0, -14)) return sign | static_cast<uint16_t>(r / std::ldexp(1.0, -24));
  const int re = std::ilogb(r);
  const int mant = static_cast<int>(r / std::ldexp(1.0, re - 10)) - 1024;
  return sign | static_cast<uint16_t>(((re + 15) << 10) | mant);
}

// One row's h values (bf16 bits) for gate/up rows g, u of length n and row
// weight w (already 1 when there is none).
void oracle_swiglu_row(const uint16_t* g, const uint16_t* u, double w, int64_t n, double limit,
                       uint16_t* h) {
  for (int64_t k = 0; k < n; ++k) {
    double gv = bf16_to_float(g[k]);
    double uv = bf16_to_float(u[k]);
    if (limit > 0.0) {   // false for NaN: no clamp
      gv = gv < limit ? gv : limit;
      uv = uv < -limit ? -limit : (uv > limit ? limit : uv);
    }
    h[k] = oracle_bf16_rne(oracle_silu(gv) * uv * w);
  }
}

// One q8_1 block (36 bytes: fp16 d, fp16 sum, 32 int8) from 32 bf16 values.
void oracle_q8_1_block(const uint16_t* h, uint8_t* out) {
  float amax = 0.0f;
  for (int i = 0; i < 32; ++i) {
    const float a = std::fabs(bf16_to_float(h[i]));
    if (a > amax) amax = a;
  }
  int8_t q[32] = {0};
  uint16_t d16 = 0, s16 = 0;
  if (amax != 0.0f) {
    const float d = amax / 127.0f;
    long qsum = 0;
    for (int i = 0; i < 32; ++i) {
      float r = std::nearbyint(bf16_to_float(h[i]) / d);
      if (r > 127.0f) r = 127.0f;
      if (r < -127.0f) r = -127.0f;
      q[i] = static_cast<int8_t>(r);
      qsum += q[i];
    }
    d16 = oracle_fp16_rne(d);
    s16 = oracle_fp16_rne(static_cast<double>(d) * static_cast<double>(qsum));  // exact product
  }
  std::memcpy(out, &d16, 2);
  std::memcpy(out + 2, &s16, 2);
  std::memcpy(out + 4, q, 32);
}

// The forward op: gate, up [rows, inter] bf16; w [rows] fp32 or NULL;
// h [rows, inter] bf16; q8 [rows, inter/32] blocks of 36 bytes.  Returns 0,
// or -1 when inter is not a positive multiple of 32 or rows < 0.
int oracle_swiglu_q8_1_rows(const uint16_t* gate, const uint16_t* up, const float* w,
                            uint16_t* h, uint8_t* q8, int64_t rows, int64_t inter, float limit) {
  if (rows < 0 || inter < 32 || inter % 32 != 0) return -1;
  for (int64_t m = 0; m < rows; ++m) {
    const double wm = w ? static_cast<double>(w[m]) : 1.0;
    oracle_swiglu_row(&gate[m * inter], &up[m * inter], wm, inter, limit, &h[m * inter]);
    for (int64_t b = 0; b < inter / 32; ++b)
      oracle_q8_1_block(&h[m * inter + b * 32], &q8[(m * (inter / 32) + b) * 36]);
  }
  return 0;
}

}  // extern "C"

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
// tokens it holds; grad_input_s is [M, 2K/G] (d_gate groups first) and
// y_s_t is [K, ceil(M/G)].
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
//   oracle_quant_group     exact-rational check that scale is amax/127
//                          rounded once, nearest-integer brute force, exact
//                          ties to even, symmetry and monotonicity.
//   whole op               closed-form hand-derived cases (gate = 0, gate
//                          large), layout/transposition patterns, tail and
//                          zero groups, and a hand-derived golden fixture.

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

// Quantize one group of n bf16 values (element i at v[i*stride]) to int8:
// amax = max |v|; all-zero -> scale 1, q 0; else scale = amax/127 (fp32
// division) and q = clamp(round-half-even(v/scale), -127, 127) with the
// quotient taken in fp32.  Writes q[i*qstride] and *scale.
void oracle_quant_group(const uint16_t* v, int64_t n, int64_t stride,
                        int8_t* q, int64_t qstride, float* scale) {
  float amax = 0.0f;
  for (int64_t i = 0; i < n; ++i) {
    const float a = std::fabs(bf16_to_float(v[i * stride]));
    if (a > amax) amax = a;
  }
  if (amax == 0.0f) {
    *scale = 1.0f;
    for (int64_t i = 0; i < n; ++i) q[i * qstride] = 0;
    return;
  }
  const float s = amax / 127.0f;
  for (int64_t i = 0; i < n; ++i) {
    const float t = bf16_to_float(v[i * stride]) / s;
    float r = std::nearbyint(t);
    if (r > 127.0f) r = 127.0f;
    if (r < -127.0f) r = -127.0f;
    q[i * qstride] = static_cast<int8_t>(r);
  }
  *scale = s;
}

// First stage: the bf16 values y, d_gate, d_up ([M, K] each, bf16 bits) from
// x = [gate | up] ([M, 2K]) and grad_y ([M, K]).
void oracle_swiglu_bwd_bf16(const uint16_t* x, const uint16_t* grad_y,
                            int64_t M, int64_t K, uint16_t* y,
                            uint16_t* d_gate, uint16_t* d_up) {
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t k = 0; k < K; ++k) {
      const double g = bf16_to_float(x[m * 2 * K + k]);
      const double u = bf16_to_float(x[m * 2 * K + K + k]);
      const double dy = bf16_to_float(grad_y[m * K + k]);
      double yv, dg, du;
      oracle_swiglu_bwd_fp64(g, u, dy, &yv, &dg, &du);
      y[m * K + k] = oracle_bf16_rne(yv);
      d_gate[m * K + k] = oracle_bf16_rne(dg);
      d_up[m * K + k] = oracle_bf16_rne(du);
    }
  }
}

// The whole op.  Returns 0, or -1 for arguments the definition does not cover
// (group_size < 1, K not a multiple of group_size, negative sizes).
//   grad_input_q [M, 2K] int8     grad_input_s [M, 2K/G] fp32
//   y_q_t        [K, M]  int8     y_s_t        [K, ceil(M/G)] fp32
int oracle_silu_dot_fwd_bwd_quant_fuse(const uint16_t* x, const uint16_t* grad_y,
                                       int8_t* grad_input_q, float* grad_input_s,
                                       int8_t* y_q_t, float* y_s_t, int64_t M,
                                       int64_t K, int64_t group_size) {
  const int64_t G = group_size;
  if (G < 1 || M < 0 || K < 0 || K % G != 0) return -1;
  if (M == 0 || K == 0) return 0;
  const int64_t Kg = K / G;
  const int64_t Mg = (M + G - 1) / G;
  std::vector<uint16_t> y(M * K), dg(M * K), du(M * K);
  oracle_swiglu_bwd_bf16(x, grad_y, M, K, y.data(), dg.data(), du.data());

  // Row-wise: token m, group j of the 2K channels of [d_gate | d_up].
  for (int64_t m = 0; m < M; ++m) {
    for (int64_t j = 0; j < 2 * Kg; ++j) {
      const uint16_t* src = (j < Kg) ? &dg[m * K + j * G] : &du[m * K + (j - Kg) * G];
      oracle_quant_group(src, G, 1, &grad_input_q[m * 2 * K + j * G], 1,
                         &grad_input_s[m * 2 * Kg + j]);
    }
  }
  // Column-wise on y: channel k, token group i (the tail group holds M - i*G tokens);
  // stored transposed, y_q_t[k, t] for token t.
  for (int64_t k = 0; k < K; ++k) {
    for (int64_t i = 0; i < Mg; ++i) {
      const int64_t t0 = i * G;
      const int64_t n = (M - t0 < G) ? (M - t0) : G;
      oracle_quant_group(&y[t0 * K + k], n, K, &y_q_t[k * M + t0], 1,
                         &y_s_t[k * Mg + i]);
    }
  }
  return 0;
}

}  // extern "C"

// The fused kernel of silu_dot_fwd_bwd_quant_fuse for sm_100a.
//
// Operation ("kernelgen-challenge-9-task3-silu-quant", outputs section and
// constraints list): from x = [gate | up] (bf16 [M, 2K]) and grad_y (bf16
// [M, K]) recompute y = silu(gate) * up, form d_gate = grad_y * up * silu'(gate)
// and d_up = grad_y * silu(gate), round each to bf16, then write
//   grad_input_q/_s: [d_gate | d_up] quantized per token in 128-channel groups,
//   y_q_t/_s_t:      y transposed, quantized per channel in 128-token groups.
//
// Template variants (each its own instantiation, so a variant's work never
// reaches the others): group size 128, 64 or 32 (a tile holds whole groups
// of each); code format INT8 or FP8 E4M3, scale format fp32 or E8M0, y_s_t
// [K, Mg] or [Mg, K]; kY, the recomputed bf16 y also stored (read back from
// the shared y tile after the code stores);
// kQdy, grad_y read as INT8 codes (an 8-bit box in the stage's third slot)
// times one fp32 scale per token and 128 channels.
//
// Work decomposition.  A 128-token x 128-channel tile (i, j) holds exactly one
// quantization group on both axes, so tiles are independent.  The grid is
// persistent (at most one CTA per SM); CTA b walks tiles b, b + grid, ... in a
// banded order (8 tile rows per band, tile row fastest) so that the scale
// sectors of neighbouring tiles are written close together in time.
//
// Inside a CTA (16 warps, all of them compute):
//   * each tile arrives as two 64-row stages; a stage is three TMA boxes
//     (gate, up, grad_y; 64 x 128 bf16 each, 48 KB) in a STAGES-deep
//     shared-memory ring.  Load n of a CTA is tile n/2, half n%2, so any thread
//     can issue any load.  A load completes on an mbarrier (TMA byte count); the
//     warps release a slot through a shared counter and the warp that releases
//     it last issues the load that goes next into it -- there is no producer
//     warp, so every warp computes and may use 128 registers.
//     Rows past M are zero-filled by the TMA unit, and zeros never change an
//     amax, so a tail token group is quantized over exactly the tokens it holds.
//     Each slot has two mbarriers that take its loads in turn, so that with
//     an odd STAGES (consecutive loads of a slot going to different warp
//     halves, below) every barrier's uses still belong to one half.
//   * row pass: warps 0-7 take the first stage of every tile and warps 8-15
//     the second, so the two halves of the CTA work on different slots and a
//     slot waits for 8 warps, not 16.  A lane owns 32 channels of one token
//     row (4 lanes per row, 8 rows per warp): fp32 math in packed f32x2
//     instructions, bf16 rounding, the row amax of d_gate and d_up over its
//     chunks and then over the row's 4 lanes (2 shuffle steps on packed bf16
//     pairs), each lane computing its row's scales itself, quantization by
//     multiplication with the inverse scale, 8-byte stores per 8 channels; the
//     bf16 y values go to a shared [token][channel] tile (double-buffered
//     across tiles).  Per-row work (reductions, scales, the stage's wait and
//     release) is spread over 32 elements a lane, half the cost per element
//     of 16-channel lanes.
//   * column pass, one tile late (after the row pass of the next tile, so no
//     warp waits for the others at a tile boundary; two mbarriers per y buffer
//     say "all rows written" and "all columns read"): a thread owns 2 channels
//     x 16 tokens of the tile, reduces the column amax over the 8 threads that
//     share its channels, computes the two column scales, quantizes its 32 y
//     values and stores two 16-byte pieces of y_q_t rows; each group of 8
//     threads writes one 128-byte line.
//   * launch: the kernel is launched with programmatic stream serialization
//     and allows the next grid to launch at once, so a CTA starts as soon as
//     the previous grid's CTA on its SM exits, and waits (griddepcontrol) for
//     the whole previous grid before it loads.  Meanwhile it prefetches the
//     boxes of its first STAGES loads into L2, so they land from L2 after the
//     wait instead of taking a DRAM round trip.
//   * shared-memory layouts are chosen for conflict-free access: a lane of an
//     odd row takes its chunks in the order (4k + q) ^ 4, so each 8-lane
//     quarter of a warp reads 8 distinct bank groups, and the y tile's chunks
//     are XOR-swizzled by token.
//
// Every wait on an mbarrier is bounded (Params::wait_limit_ns).  A wait that
// runs out sets the device status word and a shared abort flag that every
// other wait polls, so all warps stop within one wait; after a final
// __syncthreads one thread waits (bounded) for the copies still in flight.
#pragma once

#include <cstdint>

#include "sdq_ptx.cuh"

namespace sdq {

constexpr int kG = 128;                             // group size = tile edge
constexpr int kStageRows = 64;                      // token rows per pipeline stage
constexpr int kStagesPerTile = kG / kStageRows;     // 2
constexpr int kBoxBytes = kStageRows * kG * 2;      // one bf16 box: 16 KB
constexpr int kStageBytes = 3 * kBoxBytes;          // gate + up + grad_y
constexpr int kQBoxBytes = kStageRows * kG;         // one INT8 grad_y box: 8 KB
constexpr int kYBytes = kG * kG * 2;                // bf16 y tile: 32 KB
constexpr int kWarps = 16;
constexpr int kThreads = kWarps * 32;
#ifndef SDQ_YBUF
#define SDQ_YBUF 2
#endif
constexpr int kYBuf = SDQ_YBUF;                     // y tiles in flight between row and column passes

constexpr int kDevTimeout = 1;  // bit in the device status word

// Device status word: OR of kDev* bits; read and cleared by sdq_device_status().
__device__ int g_sdq_dev_status;

// Output formats, template parameters of the kernel (so the page's format
// runs the same instructions as a kernel built for it alone): codes INT8
// (the page's) or OCP FP8 E4M3; scales fp32 (the page's) or E8M0 bytes (the
// smallest power of two not below amax/Qmax); y_s_t [K, Mg] (the page's) or
// [Mg, K].
struct Params {
  int8_t* giq;   // [M, 2K] code bytes
  void* gis;     // [M, 2K/128] fp32 or E8M0 bytes
  int8_t* yqt;   // [K, M] code bytes
  void* yst;     // [K, Mg] or [Mg, K], fp32 or E8M0 bytes
  int64_t M;
  int32_t K;
  int32_t Kg;        // 128-channel tiles per row (the last one may be partial: K % 128 != 0)
  int32_t gis_cols;  // 2 ceil(K / group size): columns of grad_input_s (d_up groups from gis_cols/2)
  uint8_t* y;        // optional bf16 y [M, K] (kernels built with kY)
  int64_t ld_y;
  const float* gys;  // INT8 grad_y's scales [M, K/128] (kernels built with kQdy)
  int64_t ld_gys;
  int64_t ld_yqt;    // elements from one row of each output to the next
  int64_t ld_yst;
  int32_t ld_giq;    // (at most 2^24: a tile's row offsets stay 32-bit products)
  int32_t ld_gis;
  int32_t Mg;
  int32_t num_tiles;
  int32_t yqt_vec16;  // ld_yqt % 16 == 0: y_q_t rows take 16-byte stores
  int32_t withhold_first_load;  // test hook: leave load 0 unissued so its wait runs out
  uint64_t wait_limit_ns;
};

template <int STAGES>
struct Smem {
  alignas(128) uint8_t ring[STAGES][kStageBytes];  // [gate | up | grad_y], each [64][128] bf16
  alignas(16) uint8_t ytile[kYBuf][kYBytes];       // bf16 y [token][channel], chunks swizzled
  alignas(16) float2 scale_tab[128];               // per bf16 mantissa m: scale and inverse for 2^0 (see group_scale)
  alignas(8) uint64_t full[STAGES][2];             // per slot, alternate loads (ring_bar_index)
  alignas(8) uint64_t y_ready[kYBuf];              // all threads wrote their rows of the y tile
  alignas(8) uint64_t y_free[kYBuf];               // all threads finished reading the y tile
  int released[STAGES];                            // warps done with the slot's current load
  int issued;                                      // loads issued so far (for the drain on abort)
  int abort;                                       // set by the first wait that runs out
};

template <int STAGES>
constexpr size_t smem_bytes() {
  return sizeof(Smem<STAGES>) + 128;  // + room to align the base to 128 B
}

// The ring barrier of load n and the parity a consumer waits on.  Each slot
// has two barriers that take its loads in turn, so consecutive uses of one
// barrier are loads n and n + 2 STAGES.  The two warp halves take alternate
// loads, so those are always the same half's, consumed in order: when a half
// waits on load n's barrier, the barrier is in load n's phase or just past it,
// never a phase behind (with one barrier per slot and an odd STAGES, a half
// that ran a tile ahead could find the slot a phase behind, with the same
// parity as the one it waits for, and read the slot before its copy landed).
__device__ __forceinline__ uint32_t ring_bar_index(uint32_t n, uint32_t stages) {
  return 2 * (n % stages) + ((n / stages) & 1u);
}
__device__ __forceinline__ uint32_t ring_parity(uint32_t n, uint32_t stages) {
  return (n / (2 * stages)) & 1u;
}

// Tile t -> (token-group i, channel-group j), banded: kTileBand tile rows per
// band, tile row fastest inside a band (a band of 1 is channel-group fastest).
#ifndef SDQ_TILE_BAND
#define SDQ_TILE_BAND 8
#endif
__device__ __forceinline__ void tile_ij(int t, int Mg, int Kg, int& i, int& j) {
  constexpr int kBand = SDQ_TILE_BAND;
  static_assert(kBand > 0 && (kBand & (kBand - 1)) == 0, "band height must be a power of two");
  const int band = t / (kBand * Kg);
  const int r = t - band * (kBand * Kg);
  const int rows = min(kBand, Mg - band * kBand);
  if (rows == kBand) {   // every band but the last: power-of-two height
    i = band * kBand + (r & (kBand - 1));
    j = r / kBand;
  } else {
    i = band * kBand + r % rows;
    j = r / rows;
  }
}

// Tensor coordinates (channel x, token y) of the boxes of load n of this CTA.
__device__ __forceinline__ void load_coords(const Params& p, uint32_t n, int& x, int& y) {
  const int t = blockIdx.x + static_cast<int>(n / kStagesPerTile) * gridDim.x;
  int i, j;
  tile_ij(t, p.Mg, p.Kg, i, j);
  x = j * kG;
  y = i * kG + static_cast<int>(n % kStagesPerTile) * kStageRows;
}

// Load n of this CTA: stage n % 2 of its (n / 2)-th tile, into slot n % STAGES.
// The three input tensor maps (gate, up, grad_y: [M, K] bf16 each, with their
// own row strides; gate and up may be the two halves of one x = [gate | up]).
template <int STAGES, bool kQdy>
__device__ __forceinline__ void issue_load(Smem<STAGES>& s, const CUtensorMap* mgate,
                                           const CUtensorMap* mup, const CUtensorMap* mdy,
                                           const Params& p, uint32_t n, uint64_t pol) {
  int x, r;
  load_coords(p, n, x, r);
  const uint32_t slot = n % STAGES;
  const uint32_t fb = smem_u32(&s.full[0][0] + ring_bar_index(n, STAGES));
  mbar_arrive_expect_tx(fb, kQdy ? 2 * kBoxBytes + kQBoxBytes : kStageBytes);
  const uint32_t dst = smem_u32(s.ring[slot]);
  tma_load_2d(dst, mgate, fb, x, r, pol);
  tma_load_2d(dst + kBoxBytes, mup, fb, x, r, pol);
  tma_load_2d(dst + 2 * kBoxBytes, mdy, fb, x, r, pol);
}

// bf16 pair -> two floats (exact).
__device__ __forceinline__ float2 unpack2(uint32_t v) { return make_float2(bf16_lo(v), bf16_hi(v)); }

// Two elements: y = silu(g)*u, d_gate = dy*u*silu'(g), d_up = dy*silu(g) in
// fp32 (packed pairs), with silu'(g) = sigma(g)*(1 + g*(1 - sigma(g)))
// = silu*(1 - sigma) + sigma.  Results as bf16 pairs.
__device__ __forceinline__ void swiglu_bwd2f(uint32_t gw, uint32_t uw, float2 dy, uint32_t& y,
                                             uint32_t& dg, uint32_t& du) {
  constexpr float kNegLog2e = -1.4426950408889634f;  // e^-g = 2^(-g log2 e)
  const float2 g = unpack2(gw), u = unpack2(uw);
  const float2 one = make_float2(1.0f, 1.0f);
  const float2 xl = __fmul2_rn(g, make_float2(kNegLog2e, kNegLog2e));
  const float2 d = __fadd2_rn(make_float2(ex2_approx(xl.x), ex2_approx(xl.y)), one);
  const float2 sg = make_float2(rcp_approx(d.x), rcp_approx(d.y));  // 0 or 1 when saturated
  const float2 silu = __fmul2_rn(g, sg);
  const float2 oms = __ffma2_rn(sg, make_float2(-1.0f, -1.0f), one);
  const float2 dsilu = __ffma2_rn(silu, oms, sg);
  const float2 yy = __fmul2_rn(silu, u);
  const float2 gg = __fmul2_rn(__fmul2_rn(dy, u), dsilu);
  const float2 uu = __fmul2_rn(dy, silu);
  y = pack_bf16x2(yy.x, yy.y);
  dg = pack_bf16x2(gg.x, gg.y);
  du = pack_bf16x2(uu.x, uu.y);
}

__device__ __forceinline__ void swiglu_bwd2(uint32_t gw, uint32_t uw, uint32_t dw, uint32_t& y,
                                            uint32_t& dg, uint32_t& du) {
  swiglu_bwd2f(gw, uw, unpack2(dw), y, dg, du);
}

// Eight INT8 codes (channel order) times their group's scale: four fp32
// pairs, each product rounded once.  A code c becomes a float without the
// quarter-rate integer conversion: c + 128 (the byte XOR 0x80) placed in the
// low mantissa byte of 2^23 is the float 2^23 + 128 + c, and subtracting
// 2^23 + 128 leaves c exactly.
__device__ __forceinline__ void dequant8(uint2 q, float sc, float2* out) {
  constexpr float kBias = 8388736.0f;   // 2^23 + 128
  const float2 s2 = make_float2(sc, sc);
  const float2 nb = make_float2(-kBias, -kBias);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t w = (h ? q.y : q.x) ^ 0x80808080u;
#pragma unroll
    for (int p = 0; p < 2; ++p) {   // bytes 2p, 2p+1 into the low byte of 0x4B000000 (2^23)
      const float lo = __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7540u | (2 * p)));
      const float hi = __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7540u | (2 * p + 1)));
      out[2 * h + p] = __fmul2_rn(__fadd2_rn(make_float2(lo, hi), nb), s2);
    }
  }
}

// Scale and inverse scale of a group from its amax, given as non-negative
// bf16 bits, for codes up to Qmax (127 for INT8, 448 for E4M3):
//   fp32 scales: scale = fl(amax / Qmax), inv = fl(1 / scale);
//   E8M0 scales: scale = the smallest power of two >= fl(amax / Qmax),
//                clamped to [2^-127, 2^127], inv = 1 / scale (exact);
// an all-zero group gets scale 1.  A bf16 amax is (1 + m/128) * 2^e, and
// fl(amax / Qmax) = fl((1 + m/128) / Qmax) * 2^e exactly whenever both are
// normal floats; so a 128-entry table holds, per mantissa m, the scale and
// inverse for e = 0 (fl((1 + m/128)/Qmax) and its reciprocal, or the power of
// two above it and its reciprocal), and 2^e goes into the exponent fields.
// That holds for every bf16 exponent field >= kTableEx; smaller amaxes (below
// 2^-117) take the out-of-line IEEE path.  There, with fp32 scales, 1/scale can
// exceed the float range, so the returned inverse is meant for values
// pre-multiplied by kTinyPre (= 2^64) and comes back negated as a marker:
// (v * 2^64) * fl(1/(scale * 2^64)) is the same real number as v * fl(1/scale).
// E8M0 inverses are at most 2^127 and need no marker.
constexpr float kTinyPre = 18446744073709551616.0f;  // 2^64
constexpr uint32_t kTableEx = 10;

template <bool kE4M3>
__host__ __device__ constexpr float qmax() { return kE4M3 ? 448.0f : 127.0f; }

// Exponent k of the smallest power of two >= s (s > 0, finite, subnormals included).
__device__ __forceinline__ int ceil_log2(float s) {
  const uint32_t b = __float_as_uint(s);
  if (b >= 0x00800000u) return static_cast<int>(b >> 23) - 127 + ((b & 0x007FFFFFu) != 0u ? 1 : 0);
  return (31 - __clz(static_cast<int>(b))) - 149 + ((b & (b - 1u)) != 0u ? 1 : 0);
}

// 2^k as a float for -127 <= k <= 127 (2^-127 is subnormal).
__device__ __forceinline__ float pow2f(int k) {
  return k >= -126 ? __uint_as_float(static_cast<uint32_t>(k + 127) << 23) : __uint_as_float(0x00400000u);
}

// Table entry for mantissa m (scale and inverse for a bf16 exponent field of 127).
template <bool kE4M3, bool kE8M0>
__device__ __forceinline__ float2 scale_table_entry(int m) {
  const float t = __fdiv_rn(1.0f + static_cast<float>(m) * (1.0f / 128.0f), qmax<kE4M3>());
  if (!kE8M0) return make_float2(t, __frcp_rn(t));
  const int k = ceil_log2(t);
  return make_float2(pow2f(k), pow2f(-k));
}

// The rare branch, kept out of line so the common path stays short.
template <bool kE4M3, bool kE8M0>
__device__ __noinline__ float2 tiny_group_scale(uint32_t abits) {
  if (abits == 0u) return make_float2(1.0f, 1.0f);
  const float s = __fdiv_rn(__uint_as_float(abits << 16), qmax<kE4M3>());
  if (!kE8M0) return make_float2(s, -__frcp_rn(s * kTinyPre));
  const int k = max(ceil_log2(s), -127);   // a bf16 amax never needs more than 2^122
  return make_float2(pow2f(k), pow2f(-k));
}

template <bool kE4M3, bool kE8M0>
__device__ __forceinline__ void group_scale(uint32_t abits, const float2* tab, float& scale,
                                            float& inv_marked) {
  const uint32_t ex = abits >> 7;
  if (ex >= kTableEx) {
    const float2 t = tab[abits & 127u];
    const int sh = (static_cast<int>(ex) - 127) << 23;
    scale = __int_as_float(__float_as_int(t.x) + sh);
    inv_marked = __int_as_float(__float_as_int(t.y) - sh);
  } else {
    const float2 r = tiny_group_scale<kE4M3, kE8M0>(abits);
    scale = r.x;
    inv_marked = r.y;
  }
}

// A scale into an fp32 array, or as its E8M0 byte (a power of two in
// [2^-127, 2^127] carries its byte in the float's exponent field; 2^-127,
// subnormal, gives 0).
template <bool kE8M0>
__device__ __forceinline__ void store_scale(void* base, int64_t idx, float scale) {
  if (kE8M0) static_cast<uint8_t*>(base)[idx] = static_cast<uint8_t>(__float_as_uint(scale) >> 23);
  else static_cast<float*>(base)[idx] = scale;
}

// A bf16 pair times `inv` (each half pre-multiplied by `pre` first).  INT8:
// round-half-even codes, each the low byte of its float's bits (the constant
// 1.5 * 2^23 inside the fused multiply-add rounds to an integer).  E4M3: the
// two fp32 products.
template <bool kE4M3, bool kTiny>
__device__ __forceinline__ float2 quant2(uint32_t v, float2 inv, float2 pre, float2 scl) {
  float2 x = unpack2(v);
  if (kTiny) x = __fmul2_rn(x, pre);
  if (kE4M3) {
    // The quotient x / scale correctly rounded to fp32, from the reciprocal
    // and one correction (Markstein): r = x * inv, then the exact remainder
    // x - r * scale, then r + remainder * inv.  E4M3 keeps three mantissa
    // bits, so x / scale often sits exactly on a rounding tie of the code,
    // where the plain product could fall on either side.
    const float2 r = __fmul2_rn(x, inv);
    const float2 e = __ffma2_rn(make_float2(-r.x, -r.y), scl, x);
    return __ffma2_rn(e, inv, r);
  }
  return __ffma2_rn(x, inv, make_float2(12582912.0f, 12582912.0f));
}

// Four codes (in byte order a.x, a.y, b.x, b.y) from two quant2 results.
template <bool kE4M3>
__device__ __forceinline__ uint32_t pack_codes(float2 a, float2 b) {
  if (kE4M3) return e4m3x4(a.x, a.y, b.x, b.y);
  return pack_low_bytes(__float_as_uint(a.x), __float_as_uint(a.y), __float_as_uint(b.x),
                        __float_as_uint(b.y));
}

// Sixteen codes of one row piece (8 bf16 pairs) with one inverse scale.
// `scale`: the group's scale (times kTinyPre for the tiny path), used by the
// E4M3 quotient correction only.
template <bool kE4M3, bool kTiny>
__device__ __forceinline__ uint4 quant16(const uint32_t (&v)[8], float inv, float scale) {
  const float2 iv = make_float2(inv, inv);
  const float2 pre = make_float2(kTinyPre, kTinyPre);
  const float2 sc = make_float2(scale, scale);
  uint32_t w[4];
#pragma unroll
  for (int k = 0; k < 4; ++k)
    w[k] = pack_codes<kE4M3>(quant2<kE4M3, kTiny>(v[2 * k], iv, pre, sc),
                             quant2<kE4M3, kTiny>(v[2 * k + 1], iv, pre, sc));
  return make_uint4(w[0], w[1], w[2], w[3]);
}

// Column pass: 16 tokens x 2 channels (one bf16 pair per token) -> two
// 16-byte code rows (low channel, high channel).
template <bool kE4M3, bool kTiny>
__device__ __forceinline__ void quant_cols(const uint32_t (&v)[16], float2 inv, float2 pre,
                                           float2 scl, uint4& lo, uint4& hi) {
  float2 q[16];
#pragma unroll
  for (int t = 0; t < 16; ++t) q[t] = quant2<kE4M3, kTiny>(v[t], inv, pre, scl);
  uint32_t wl[4], wh[4];
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    // low channel: the .x of tokens 4w..4w+3; high channel: the .y
    wl[w] = pack_codes<kE4M3>(make_float2(q[4 * w].x, q[4 * w + 1].x), make_float2(q[4 * w + 2].x, q[4 * w + 3].x));
    wh[w] = pack_codes<kE4M3>(make_float2(q[4 * w].y, q[4 * w + 1].y), make_float2(q[4 * w + 2].y, q[4 * w + 3].y));
  }
  lo = make_uint4(wl[0], wl[1], wl[2], wl[3]);
  hi = make_uint4(wh[0], wh[1], wh[2], wh[3]);
}

// 16 code bytes to a y_q_t row piece that may be cut short by the token count
// or unaligned (M % 16 != 0).
__device__ __forceinline__ void store_codes(int8_t* dst, uint4 o, int nb, bool vec16) {
  if (vec16 && nb >= 16) {
    st_cs_v4(dst, o);
    return;
  }
#pragma unroll
  for (int b = 0; b < 16; ++b) {
    const uint32_t w = b < 4 ? o.x : b < 8 ? o.y : b < 12 ? o.z : o.w;
    if (b < nb) dst[b] = static_cast<int8_t>(w >> ((b & 3) * 8));
  }
}

// Bounded wait that also gives up as soon as another warp of the CTA has set
// the abort flag; the first wait to run out sets the flag and the status word.
__device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t parity, uint64_t limit_ns,
                                              volatile int* abort_flag) {
  if (mbar_test_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > limit_ns) {
      *abort_flag = 1;
      atomicOr(&g_sdq_dev_status, kDevTimeout);
      return false;
    }
  }
  return true;
}

// Quantization groups of kGS = 32, 64 or 128 elements: a 128 x 128 tile holds
// 128/kGS groups along each axis, and since a row-pass lane holds 16
// consecutive channels of a row and a column-pass thread 16 consecutive
// tokens of a channel pair, a group is kGS/16 neighbouring lanes (threads):
// its amax takes log2(kGS/16) shuffle steps.
template <int kGS>
__device__ __forceinline__ uint32_t group_amax(uint32_t m) {
  static_assert(kGS == 32 || kGS == 64 || kGS == 128, "group size 32, 64 or 128");
#pragma unroll
  for (int o = 1; o < kGS / 16; o <<= 1) m = absmax_bf16x2(m, __shfl_xor_sync(0xffffffffu, m, o));
  return m;
}

// Column pass of one tile: this thread's channels 2cp, 2cp+1 and tokens
// 16kc .. 16kc+15 of the bf16 y tile -> column amax over the kGS/16 threads
// that share the channels and the token group, the two column scales, codes,
// two 16-byte pieces of y_q_t rows.
template <int kGS, bool kE4M3, bool kE8M0, bool kYsMgK>
__device__ __forceinline__ void column_pass(const uint8_t* yt, const float2* tab, const Params& p,
                                            int i, int j, int64_t row0, int valid, int cp, int kc) {
  constexpr unsigned kFull = 0xffffffffu;
  uint32_t v[16];
  const uint8_t* col = yt + (16 * kc) * (kG * 2) + ((cp ^ (4 * kc)) << 2);
#pragma unroll
  for (int tt = 0; tt < 16; ++tt) v[tt] = *reinterpret_cast<const uint32_t*>(col + tt * (kG * 2));
  uint32_t m = absmax_bf16x2(v[0], v[1]);
#pragma unroll
  for (int tt = 2; tt < 16; ++tt) m = absmax_bf16x2(m, v[tt]);
  m = group_amax<kGS>(m) & 0x7FFF7FFFu;
  float s_lo, i_lo, s_hi, i_hi;
  group_scale<kE4M3, kE8M0>(m & 0xFFFFu, tab, s_lo, i_lo);
  group_scale<kE4M3, kE8M0>(m >> 16, tab, s_hi, i_hi);
  const int ch = j * kG + 2 * cp;
  const bool ch_ok = ch < p.K;     // a partial channel tile's missing channels are zeros, not stored
  // the first two threads of each token group store its low / high channel
  // scale, for the groups that hold a token (a tail tile's later groups don't)
  constexpr int kTpg = kGS / 16;   // threads per token group
  const int gk = kc & (kTpg - 1);
  const int tg = kc / kTpg;        // token group within the tile
  if (gk < 2 && tg * kGS < valid && ch_ok) {
    const int64_t grp = int64_t(i) * (kG / kGS) + tg;
    store_scale<kE8M0>(p.yst, kYsMgK ? grp * p.ld_yst + ch + gk : int64_t(ch + gk) * p.ld_yst + grp,
                       gk ? s_hi : s_lo);
  }
  uint4 lo, hi;
  if (__any_sync(kFull, i_lo < 0.0f || i_hi < 0.0f)) {   // a tiny group in this warp (rare)
    // pre-multiply only the tiny channels; the others use factor 1
    const float2 pre = make_float2(i_lo < 0.0f ? kTinyPre : 1.0f, i_hi < 0.0f ? kTinyPre : 1.0f);
    quant_cols<kE4M3, true>(v, make_float2(fabsf(i_lo), fabsf(i_hi)), pre,
                            make_float2(s_lo * pre.x, s_hi * pre.y), lo, hi);
  } else {
    quant_cols<kE4M3, false>(v, make_float2(i_lo, i_hi), make_float2(1.0f, 1.0f), make_float2(s_lo, s_hi),
                             lo, hi);
  }
  const int tok = 16 * kc;
  if (tok < valid && ch_ok) {
    const int nb = min(16, valid - tok);
    int8_t* dst = p.yqt + int64_t(ch) * p.ld_yqt + row0 + tok;
    store_codes(dst, lo, nb, p.yqt_vec16 != 0);
    store_codes(dst + p.ld_yqt, hi, nb, p.yqt_vec16 != 0);
  }
}

// Eight codes of one 16-byte chunk (4 bf16 pairs) with one inverse scale;
// `scale` as in quant16.
template <bool kE4M3, bool kTiny>
__device__ __forceinline__ uint2 quant8(const uint32_t* v, float inv, float scale) {
  const float2 iv = make_float2(inv, inv);
  const float2 pre = make_float2(kTinyPre, kTinyPre);
  const float2 sc = make_float2(scale, scale);
  return make_uint2(pack_codes<kE4M3>(quant2<kE4M3, kTiny>(v[0], iv, pre, sc), quant2<kE4M3, kTiny>(v[1], iv, pre, sc)),
                    pack_codes<kE4M3>(quant2<kE4M3, kTiny>(v[2], iv, pre, sc), quant2<kE4M3, kTiny>(v[3], iv, pre, sc)));
}

// Tile sequence of this CTA (tiles blockIdx.x, blockIdx.x + gridDim.x, ...)
// in the banded order of tile_ij, stepped without a division per tile: the
// position within the current band advances by gridDim.x and wraps into
// the next band.
struct TileWalk {
  int bsz;    // tiles per band: kBand * Kg
  int band;
  int r;      // position inside the band
  __device__ __forceinline__ void start(int t, int Kg) {
    bsz = SDQ_TILE_BAND * Kg;
    band = t / bsz;
    r = t - band * bsz;
  }
  __device__ __forceinline__ void next() {
    r += gridDim.x;
    while (r >= bsz) {
      r -= bsz;
      ++band;
    }
  }
  __device__ __forceinline__ void ij(int Mg, int& i, int& j) const {
    constexpr int kBand = SDQ_TILE_BAND;
    const int rows = min(kBand, Mg - band * kBand);
    if (rows == kBand) {
      i = band * kBand + (r & (kBand - 1));
      j = r / kBand;
    } else {
      i = band * kBand + r % rows;
      j = r / rows;
    }
  }
};

template <int STAGES, int kGS, bool kE4M3, bool kE8M0, bool kYsMgK, bool kY, bool kQdy>
__global__ void __launch_bounds__(kThreads, 1)
    fuse_kernel(const __grid_constant__ CUtensorMap map_gate, const __grid_constant__ CUtensorMap map_up,
                const __grid_constant__ CUtensorMap map_gy,
                const Params p) {
  constexpr unsigned kFull = 0xffffffffu;
  constexpr int kNG = kG / kGS;     // row groups per tensor in a tile row: 1, 2, 4
  constexpr int kSPG = 4 / kNG;     // a lane's chunks per group: 4, 2, 1
  extern __shared__ uint8_t smem_raw[];
  auto& s = *reinterpret_cast<Smem<STAGES>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~static_cast<uintptr_t>(127));
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  // row pass: warps 0-7 take stage 0 of every tile, warps 8-15 stage 1; lane
  // (rr, q) of warp wi owns row 8 wi + rr of the stage and its 16-byte chunks
  // ch[k] = (4k + q) ^ 4 (rr & 1), k = 0..3 (8 channels each): an 8-lane
  // quarter of the warp then reads 8 distinct bank groups
  const int grp = warp >> 3;
  const int rr = lane >> 2;
  const int q = lane & 3;
  const int par = rr & 1;
  const int srow = (warp & 7) * 8 + rr;
  const int r = grp * kStageRows + srow;   // this lane's row within the tile
  int ch[4];
#pragma unroll
  for (int k = 0; k < 4; ++k) ch[k] = (4 * k + q) ^ (4 * par);
  // column pass: thread = 8 * cp + kc owns channels 2cp, 2cp+1 and tokens 16kc..16kc+15
  const int cp = tid >> 3;
  const int kc = tid & 7;
  const int my_tiles = (p.num_tiles - static_cast<int>(blockIdx.x) + gridDim.x - 1) / gridDim.x;
  const uint32_t total = static_cast<uint32_t>(my_tiles) * kStagesPerTile;
  const uint64_t pol = l2_policy_evict_first();  // inputs are read exactly once

  if (tid < 128) s.scale_tab[tid] = scale_table_entry<kE4M3, kE8M0>(tid);
  if (tid == 0) {
    prefetch_tensormap(&map_gate);
    prefetch_tensormap(&map_up);
    prefetch_tensormap(&map_gy);
    for (int st = 0; st < STAGES; ++st) {
      mbar_init(smem_u32(&s.full[st][0]), 1);
      mbar_init(smem_u32(&s.full[st][1]), 1);
      s.released[st] = 0;
    }
    for (int b = 0; b < kYBuf; ++b) {
      mbar_init(smem_u32(&s.y_ready[b]), kThreads);
      mbar_init(smem_u32(&s.y_free[b]), kThreads);
    }
    s.abort = 0;
    fence_mbar_init();
    // While the previous grid of the stream finishes (this CTA can start as
    // soon as its SM is free), warm L2 with the boxes of the first loads:
    // they then land from L2 right after the wait instead of from DRAM.
    const uint32_t first = total < STAGES ? total : STAGES;
    for (uint32_t n = 0; n < first; ++n) {
      int x, y;
      load_coords(p, n, x, y);
      tma_prefetch_l2_2d(&map_gate, x, y);
      tma_prefetch_l2_2d(&map_up, x, y);
      tma_prefetch_l2_2d(&map_gy, x, y);
    }
    grid_dependency_wait();   // inputs may come from the previous kernel in the stream
    s.issued = static_cast<int>(first);
    for (uint32_t n = 0; n < first; ++n)
      if (n != 0 || !p.withhold_first_load)
        issue_load<STAGES, kQdy>(s, &map_gate, &map_up, &map_gy, p, n, pol);
  }
  grid_dependency_wait();   // every thread: global memory only after the previous grid is done
  grid_launch_dependents();
  __syncthreads();

  const int K = p.K;
  const int64_t M = p.M;
  const float2* tab = s.scale_tab;
  volatile int* abort_flag = &s.abort;
  const uint64_t lim = p.wait_limit_ns;
  bool ok = true;
  // The column pass of tile k runs after the row pass of tile k+1, so warps
  // never wait for each other at a tile boundary: y_ready[b] says every
  // thread has written its rows of the tile in y buffer b, y_free[b] that
  // every thread has read it; with kYBuf buffers a buffer is rewritten
  // kYBuf tiles later, which leaves a warp slack.  Waits depend only on
  // earlier points of the same per-warp sequence, so they cannot wait on
  // each other in a cycle.
  int pi = 0, pj = 0, pvalid = 0;   // the tile whose column pass is pending
  int64_t prow0 = 0;
  TileWalk walk;
  walk.start(blockIdx.x, p.Kg);

  for (int k = 0; k < my_tiles && ok; ++k) {
    if (k > 0) walk.next();
    int i, j;
    walk.ij(p.Mg, i, j);
    const int64_t row0 = int64_t(i) * kG;
    const int valid = static_cast<int>(M - row0 < kG ? M - row0 : int64_t(kG));
    const int cvalid = min(kG, K - j * kG);   // channels of this tile (fewer in a partial last one)
    const int yb = k % kYBuf;   // y buffer of this tile; tile t completes phase t / kYBuf of its barriers
    const uint32_t n = static_cast<uint32_t>(k) * kStagesPerTile + grp;   // this warp's load
    const uint32_t slot = n % STAGES;
    float dsc = 0.0f;   // INT8 grad_y: the scale of this lane's row in tile column j
    if constexpr (kQdy) {
      if (r < valid) dsc = __ldg(p.gys + (row0 + r) * p.ld_gys + j);
    }
    ok = __all_sync(kFull, wait_or_abort(smem_u32(&s.full[0][0] + ring_bar_index(n, STAGES)),
                                         ring_parity(n, STAGES), lim, abort_flag));
    if (!ok) break;

    // ---- stage -> registers, then release the slot (the last of the 8 warps refills it)
    uint4 gv[4], uv[4], dv[4];
    float2 dq[16];   // INT8 grad_y, dequantized
    {
      const uint8_t* src = s.ring[slot] + srow * (kG * 2);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        gv[c] = *reinterpret_cast<const uint4*>(src + ch[c] * 16);
        uv[c] = *reinterpret_cast<const uint4*>(src + kBoxBytes + ch[c] * 16);
        if constexpr (kQdy) {
          const uint8_t* qsrc = s.ring[slot] + 2 * kBoxBytes + srow * kG;
          dequant8(*reinterpret_cast<const uint2*>(qsrc + ch[c] * 8), dsc, dq + 4 * c);
        } else {
          dv[c] = *reinterpret_cast<const uint4*>(src + 2 * kBoxBytes + ch[c] * 16);
        }
      }
    }
    __syncwarp();
    if (lane == 0) {
      __threadfence_block();
      if (atomicAdd(&s.released[slot], 1) == kWarps / 2 - 1) {
        __threadfence_block();
        s.released[slot] = 0;
        const uint32_t nn = n + STAGES;
        if (nn < total) {
          atomicMax(&s.issued, static_cast<int>(nn + 1));
          issue_load<STAGES, kQdy>(s, &map_gate, &map_up, &map_gy, p, nn, pol);
        }
      }
    }

    // ---- the y buffer was last read by the column pass of tile k - kYBuf
    if (k >= kYBuf) {
      ok = __all_sync(kFull, wait_or_abort(smem_u32(&s.y_free[yb]), (k / kYBuf - 1) & 1, lim, abort_flag));
      if (!ok) break;
    }

    // ---- math, bf16 rounding; y to the shared tile (chunks swizzled by
    // token)
    uint32_t dgp[16], dup[16];   // chunk c: words 4c .. 4c+3
    const int key = (r >> 4) & 7;
    uint8_t* yrow = s.ytile[yb] + r * (kG * 2);
    {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t yv[4];
        const uint32_t g4[4] = {gv[c].x, gv[c].y, gv[c].z, gv[c].w};
        const uint32_t u4[4] = {uv[c].x, uv[c].y, uv[c].z, uv[c].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if constexpr (kQdy) {
            swiglu_bwd2f(g4[e], u4[e], dq[4 * c + e], yv[e], dgp[4 * c + e], dup[4 * c + e]);
          } else {
            const uint32_t d4[4] = {dv[c].x, dv[c].y, dv[c].z, dv[c].w};
            swiglu_bwd2(g4[e], u4[e], d4[e], yv[e], dgp[4 * c + e], dup[4 * c + e]);
          }
        }
        *reinterpret_cast<uint4*>(yrow + (ch[c] ^ key) * 16) = make_uint4(yv[0], yv[1], yv[2], yv[3]);
      }
    }

    // ---- row amax of d_gate (hi half) and d_up (lo half) per group: over the
    // lane's chunks of the group, then over the 4 lanes of the row
    uint32_t pr[kNG];
#pragma unroll
    for (int g = 0; g < kNG; ++g) {
      const int w0 = 4 * kSPG * g;
      uint32_t a = absmax_bf16x2(dgp[w0], dgp[w0 + 1]), b = absmax_bf16x2(dup[w0], dup[w0 + 1]);
#pragma unroll
      for (int w = w0 + 2; w < w0 + 4 * kSPG; ++w) {
        a = absmax_bf16x2(a, dgp[w]);
        b = absmax_bf16x2(b, dup[w]);
      }
      uint32_t m = absmax_bf16x2(__byte_perm(a, b, 0x1054), __byte_perm(a, b, 0x3276));
      m = absmax_bf16x2(m, __shfl_xor_sync(kFull, m, 1));
      pr[g] = absmax_bf16x2(m, __shfl_xor_sync(kFull, m, 2)) & 0x7FFF7FFFu;
    }

    // ---- scales of the row's groups (each of its 4 lanes computes them all)
    float sg[kNG], ig[kNG], su[kNG], iu[kNG];
    bool tiny = false;
#pragma unroll
    for (int g = 0; g < kNG; ++g) {
      group_scale<kE4M3, kE8M0>(pr[g] >> 16, tab, sg[g], ig[g]);
      group_scale<kE4M3, kE8M0>(pr[g] & 0xFFFFu, tab, su[g], iu[g]);
      tiny |= ig[g] < 0.0f || iu[g] < 0.0f;
    }
    // local group g is group gg of the tile row (the chunk order swaps the
    // 32-channel groups of odd rows); lane 2g + t stores tensor t's scale of
    // group g (both tensors from lane g when there are 4 groups)
    if (r < valid) {
      const int64_t sb = (row0 + r) * p.ld_gis + int64_t(j) * kNG;
#pragma unroll
      for (int g = 0; g < kNG; ++g) {
        const int gg = kNG == 4 ? (g ^ par) : g;
        if (gg * kGS < cvalid) {
#pragma unroll
          for (int t = 0; t < 2; ++t)
            if ((kNG == 4 ? g : 2 * g + t) == q)
              store_scale<kE8M0>(p.gis, sb + gg + t * (p.gis_cols >> 1), t ? su[g] : sg[g]);
        }
      }
    }

    // ---- quantize the row's d_gate / d_up: chunk c with its group's scale
    if (r < valid) {
      int8_t* dst = p.giq + (row0 + r) * p.ld_giq + int64_t(j) * kG;
      if (__any_sync(__activemask(), tiny)) {   // a tiny group in this warp (rare)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int g = c / kSPG;
          const uint2 og = ig[g] < 0.0f ? quant8<kE4M3, true>(dgp + 4 * c, -ig[g], sg[g] * kTinyPre)
                                        : quant8<kE4M3, false>(dgp + 4 * c, ig[g], sg[g]);
          const uint2 ou = iu[g] < 0.0f ? quant8<kE4M3, true>(dup + 4 * c, -iu[g], su[g] * kTinyPre)
                                        : quant8<kE4M3, false>(dup + 4 * c, iu[g], su[g]);
          if (ch[c] * 8 < cvalid) {
            st_cs_v2(dst + ch[c] * 8, og);
            st_cs_v2(dst + K + ch[c] * 8, ou);
          }
        }
      } else {
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int g = c / kSPG;
          const uint2 og = quant8<kE4M3, false>(dgp + 4 * c, ig[g], sg[g]);
          const uint2 ou = quant8<kE4M3, false>(dup + 4 * c, iu[g], su[g]);
          if (ch[c] * 8 < cvalid) {
            st_cs_v2(dst + ch[c] * 8, og);
            st_cs_v2(dst + K + ch[c] * 8, ou);
          }
        }
      }
    }
    // ---- y itself, bf16 (optional output), read back from the lane's own
    // chunks of the shared tile: issued after the code stores, so the math
    // above does not wait behind them
    if constexpr (kY) {
      if (r < valid) {
        int8_t* yg = reinterpret_cast<int8_t*>(p.y) + 2 * ((row0 + r) * p.ld_y + int64_t(j) * kG);
#pragma unroll
        for (int c = 0; c < 4; ++c)
          if (ch[c] * 8 < cvalid)
            st_cs_v4(yg + ch[c] * 16, *reinterpret_cast<const uint4*>(yrow + (ch[c] ^ key) * 16));
      }
    }
    mbar_arrive(smem_u32(&s.y_ready[yb]));   // every thread: its y rows of tile k are written

    // ================= column pass of the previous tile
    if (k >= 1) {
      const int pb = (k - 1) % kYBuf;
      ok = __all_sync(kFull, wait_or_abort(smem_u32(&s.y_ready[pb]), ((k - 1) / kYBuf) & 1, lim,
                                           abort_flag));
      if (!ok) break;
      column_pass<kGS, kE4M3, kE8M0, kYsMgK>(s.ytile[pb], tab, p, pi, pj, prow0, pvalid, cp, kc);
      mbar_arrive(smem_u32(&s.y_free[pb]));
    }
    pi = i;
    pj = j;
    prow0 = row0;
    pvalid = valid;
  }

  // column pass of the last tile
  if (ok && my_tiles > 0) {
    const int k = my_tiles - 1;
    ok = __all_sync(kFull, wait_or_abort(smem_u32(&s.y_ready[k % kYBuf]), (k / kYBuf) & 1, lim,
                                         abort_flag));
    if (ok) column_pass<kGS, kE4M3, kE8M0, kYsMgK>(s.ytile[k % kYBuf], tab, p, pi, pj, prow0, pvalid, cp, kc);
  }

  __syncthreads();   // every thread arrives here, whether it stopped early or not
  if (tid == 0 && *abort_flag) {
    // Leave no copy in flight into this CTA's shared memory: the last load
    // issued into each slot is the only one whose completion can be pending.
    const uint32_t issued = static_cast<uint32_t>(s.issued);
    const uint32_t first = issued > STAGES ? issued - STAGES : 0;
    for (uint32_t n = first; n < issued; ++n)
      mbar_wait(smem_u32(&s.full[0][0] + ring_bar_index(n, STAGES)), ring_parity(n, STAGES), lim);
  }
}

}  // namespace sdq

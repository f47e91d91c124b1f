// The fused kernel of silu_dot_fwd_bwd_quant_fuse for sm_100a.
//
// Operation ("kernelgen-challenge-9-task3-silu-quant", outputs section and
// constraints list): from x = [gate | up] (bf16 [M, 2K]) and grad_y (bf16
// [M, K]) recompute y = silu(gate) * up, form d_gate = grad_y * up * silu'(gate)
// and d_up = grad_y * silu(gate), round each to bf16, then write
//   grad_input_q/_s: [d_gate | d_up] quantized per token in 128-channel groups,
//   y_q_t/_s_t:      y transposed, quantized per channel in 128-token groups.
//
// Work decomposition.  A 128-token x 128-channel tile (i, j) holds exactly one
// quantization group on both axes, so tiles are independent.  The grid is
// persistent (at most one CTA per SM); CTA b walks tiles b, b + grid, ...
// in a banded order (8 tile rows per band, tile row fastest) so that the
// scale sectors of neighbouring tiles are written close together in time.
//
// Inside a CTA:
//   * one producer thread streams each tile as four 32-row sub-tiles; a
//     sub-tile is three TMA boxes (gate, up, grad_y; 32 x 128 bf16 each,
//     24 KB) into a STAGES-deep shared-memory ring guarded by full/empty
//     mbarriers.  Rows past M are zero-filled by the TMA unit, and zeros never
//     change an amax, so the tail token group is quantized over exactly the
//     tokens it holds.
//   * NW consumer warps read a stage into registers and release it at once.
//     A half-warp owns one token row of the stage, 8 channels per lane:
//     fp32 math, bf16 rounding, the row amax of d_gate and d_up by a 4-step
//     shuffle reduction on packed bf16 pairs, scales (amax/127, correctly
//     rounded) computed once per (row, half) by one lane each, quantization
//     by multiplication with the inverse scale, 8-byte coalesced stores.
//   * the bf16 y values stay in registers for the whole tile; the column amax
//     is reduced in registers, across the two half-warps by one shuffle and
//     across warps through shared memory.  After the 128 column scales, each
//     lane quantizes its y values and writes them transposed into an int8
//     staging tile (row = channel) whose 4-byte words are XOR-swizzled by
//     channel so the byte-column writes are bank-conflict free; the tile then
//     leaves as 16-byte stores, each 8-lane group writing one 128-byte line
//     of y_q_t.
//
// Every wait on an mbarrier is bounded (Params::wait_limit_ns).  A wait that
// runs out sets the device status word; the consumers agree on stopping at the
// next tile boundary through a barrier-reduction, and the producer waits
// (bounded) for its own in-flight copies before it returns.
#pragma once

#include <cstdint>

#include "sdq_ptx.cuh"

namespace sdq {

constexpr int kG = 128;                               // group size = tile edge
constexpr int kSubRows = 32;                          // token rows per pipeline stage
constexpr int kNumSub = kG / kSubRows;                // stages per tile
constexpr int kTensorStageBytes = kSubRows * kG * 2;  // one bf16 box: 8 KB
constexpr int kStageBytes = 3 * kTensorStageBytes;    // gate + up + grad_y

constexpr int kDevTimeout = 1;  // bit in the device status word

// Device status word: OR of kDev* bits; read and cleared by sdq_device_status().
__device__ int g_sdq_dev_status;

struct Params {
  int8_t* giq;   // [M, 2K]
  float* gis;    // [M, 2K/128]
  int8_t* yqt;   // [K, M]
  float* yst;    // [K, Mg]
  int64_t M;
  int32_t K;
  int32_t Kg;
  int32_t Mg;
  int32_t num_tiles;
  int32_t yqt_vec16;  // M % 16 == 0: y_q_t rows take 16-byte stores
  uint64_t wait_limit_ns;
};

template <int NW, int STAGES>
struct Config {
  static constexpr int kConsumerWarps = NW;
  static constexpr int kConsumers = NW * 32;
  static constexpr int kThreads = kConsumers + 32;       // + one producer warp
  static constexpr int kRowsPerLane = kSubRows / (2 * NW);
  static_assert(kRowsPerLane >= 1 && kRowsPerLane * 2 * NW == kSubRows, "NW must divide 16");
};

template <int NW, int STAGES>
struct Smem {
  alignas(128) uint8_t ring[STAGES][kStageBytes];  // [gate | up | grad_y], each [32][128] bf16
  alignas(16) uint8_t yt[kG * kG];                 // int8 y^T: row = channel, 4-byte words swizzled
  alignas(16) uint16_t colmax[NW][kG];             // per-warp column amax (bf16 bits)
  alignas(16) float inv_y[kG];                     // 1 / column scale
  alignas(8) uint64_t full[STAGES];
  alignas(8) uint64_t empty[STAGES];
};

template <int NW, int STAGES>
constexpr size_t smem_bytes() {
  return sizeof(Smem<NW, STAGES>) + 128;  // + room to align the base to 128 B
}

// Tile t -> (token-group i, channel-group j), banded: 8 tile rows per band,
// tile row fastest inside a band.
__device__ __forceinline__ void tile_ij(int t, int Mg, int Kg, int& i, int& j) {
  constexpr int kBand = 8;
  const int band = t / (kBand * Kg);
  const int r = t - band * (kBand * Kg);
  const int rows = min(kBand, Mg - band * kBand);
  i = band * kBand + r % rows;
  j = r / rows;
}

// One element: y = silu(g)*u, d_gate = dy*u*silu'(g), d_up = dy*silu(g), fp32.
__device__ __forceinline__ void swiglu_bwd(float g, float u, float dy, float& y, float& dg,
                                           float& du) {
  const float sg = __fdividef(1.0f, 1.0f + __expf(-g));  // sigma(g); 0 or 1 when saturated
  const float silu = g * sg;
  y = silu * u;
  dg = (dy * u) * (sg * fmaf(g, 1.0f - sg, 1.0f));
  du = dy * silu;
}

// Scale and inverse scale of a group from its amax: amax/127 correctly
// rounded; an all-zero group gets scale 1.
__device__ __forceinline__ void group_scale(float amax, float& scale, float& inv) {
  scale = 1.0f;
  inv = 1.0f;
  if (amax != 0.0f) {
    scale = __fdiv_rn(amax, 127.0f);
    inv = __frcp_rn(scale);
  }
}

template <int NW, int STAGES>
__device__ __forceinline__ void producer(Smem<NW, STAGES>& s, const CUtensorMap* mx,
                                         const CUtensorMap* mg, const Params& p) {
  prefetch_tensormap(mx);
  prefetch_tensormap(mg);
  const uint64_t pol = l2_policy_evict_first();  // inputs are read exactly once
  uint32_t n = 0;                                // stages issued
  bool ok = true;
  for (int t = blockIdx.x; ok && t < p.num_tiles; t += gridDim.x) {
    int i, j;
    tile_ij(t, p.Mg, p.Kg, i, j);
    const int64_t row0 = int64_t(i) * kG;
    const int valid = static_cast<int>((p.M - row0 < kG ? p.M - row0 : int64_t(kG)));
    const int nsub = (valid + kSubRows - 1) / kSubRows;
    for (int sub = 0; sub < nsub; ++sub) {
      const uint32_t slot = n % STAGES;
      const uint32_t ph = (n / STAGES) & 1u;
      if (!mbar_wait(smem_u32(&s.empty[slot]), ph ^ 1u, p.wait_limit_ns)) {
        atomicOr(&g_sdq_dev_status, kDevTimeout);
        ok = false;
        break;
      }
      const uint32_t fb = smem_u32(&s.full[slot]);
      mbar_arrive_expect_tx(fb, kStageBytes);
      const uint32_t dst = smem_u32(s.ring[slot]);
      const int r = static_cast<int>(row0) + sub * kSubRows;
      tma_load_2d(dst, mx, fb, j * kG, r, pol);                               // gate
      tma_load_2d(dst + kTensorStageBytes, mx, fb, p.K + j * kG, r, pol);     // up
      tma_load_2d(dst + 2 * kTensorStageBytes, mg, fb, j * kG, r, pol);       // grad_y
      ++n;
    }
  }
  if (!ok) {
    // Leave no copy in flight into this CTA's shared memory: the last load
    // into each slot is the only one whose completion can still be pending.
    const uint32_t first = n > STAGES ? n - STAGES : 0;
    for (uint32_t k = first; k < n; ++k)
      mbar_wait(smem_u32(&s.full[k % STAGES]), (k / STAGES) & 1u, p.wait_limit_ns);
  }
}

template <int NW, int STAGES>
__device__ __forceinline__ void consumer(Smem<NW, STAGES>& s, const Params& p, int warp,
                                         int lane) {
  using C = Config<NW, STAGES>;
  constexpr int RPL = C::kRowsPerLane;          // token rows per lane per stage
  constexpr int kRowsPerWarp = 2 * RPL;
  constexpr unsigned kFull = 0xffffffffu;
  const int h = lane >> 4;                      // half-warp
  const int q = lane & 15;                      // channels 8q .. 8q+7 of the tile
  const int rho = (2 * warp + h) * RPL;         // first of this lane's rows in a stage
  const int tid = threadIdx.x;                  // 0 .. kConsumers-1
  const int K = p.K;
  const int Kg = p.Kg;
  const int64_t M = p.M;
  uint32_t n = 0;                               // stages consumed
  bool abort = false;

  for (int t = blockIdx.x; t < p.num_tiles; t += gridDim.x) {
    int i, j;
    tile_ij(t, p.Mg, Kg, i, j);
    const int64_t row0 = int64_t(i) * kG;
    const int valid = static_cast<int>((M - row0 < kG ? M - row0 : int64_t(kG)));
    const int nsub = (valid + kSubRows - 1) / kSubRows;

    uint32_t yv[kNumSub][RPL][4];   // bf16 pairs of y, channels (8q+2k, 8q+2k+1)
    uint32_t cmax[4] = {0u, 0u, 0u, 0u};

#pragma unroll
    for (int sub = 0; sub < kNumSub; ++sub) {
#pragma unroll
      for (int e = 0; e < RPL; ++e)
#pragma unroll
        for (int k = 0; k < 4; ++k) yv[sub][e][k] = 0u;
      if (sub >= nsub || abort) continue;

      const uint32_t slot = n % STAGES;
      const uint32_t ph = (n / STAGES) & 1u;
      ++n;
      const bool got = mbar_wait(smem_u32(&s.full[slot]), ph, p.wait_limit_ns);
      if (__any_sync(kFull, !got)) {
        abort = true;
        if (lane == 0) atomicOr(&g_sdq_dev_status, kDevTimeout);
        continue;
      }

      // ---- stage -> registers, then hand the slot back to the producer
      const uint8_t* st = s.ring[slot];
      uint4 gv[RPL], uv[RPL], dv[RPL];
#pragma unroll
      for (int e = 0; e < RPL; ++e) {
        const int off = (rho + e) * (kG * 2) + q * 16;
        gv[e] = *reinterpret_cast<const uint4*>(st + off);
        uv[e] = *reinterpret_cast<const uint4*>(st + kTensorStageBytes + off);
        dv[e] = *reinterpret_cast<const uint4*>(st + 2 * kTensorStageBytes + off);
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(smem_u32(&s.empty[slot]));

      // ---- math, bf16 rounding, row amax of d_gate / d_up
      uint32_t dgp[RPL][4], dup[RPL][4], P[RPL];
#pragma unroll
      for (int e = 0; e < RPL; ++e) {
        const uint32_t* ga = reinterpret_cast<const uint32_t*>(&gv[e]);
        const uint32_t* ua = reinterpret_cast<const uint32_t*>(&uv[e]);
        const uint32_t* da = reinterpret_cast<const uint32_t*>(&dv[e]);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          float y0, y1, g0, g1, u0, u1;
          swiglu_bwd(bf16_lo(ga[k]), bf16_lo(ua[k]), bf16_lo(da[k]), y0, g0, u0);
          swiglu_bwd(bf16_hi(ga[k]), bf16_hi(ua[k]), bf16_hi(da[k]), y1, g1, u1);
          yv[sub][e][k] = pack_bf16x2(y0, y1);
          dgp[e][k] = pack_bf16x2(g0, g1);
          dup[e][k] = pack_bf16x2(u0, u1);
          cmax[k] = absmax_bf16x2(cmax[k], yv[sub][e][k]);
        }
        const uint32_t a = absmax_bf16x2(absmax_bf16x2(dgp[e][0], dgp[e][1]),
                                         absmax_bf16x2(dgp[e][2], dgp[e][3]));
        const uint32_t b = absmax_bf16x2(absmax_bf16x2(dup[e][0], dup[e][1]),
                                         absmax_bf16x2(dup[e][2], dup[e][3]));
        // (hi half: d_gate, lo half: d_up)
        uint32_t pr = absmax_bf16x2(__byte_perm(a, b, 0x1054), __byte_perm(a, b, 0x3276));
#pragma unroll
        for (int off = 1; off < 16; off <<= 1)
          pr = absmax_bf16x2(pr, __shfl_xor_sync(kFull, pr, off));
        P[e] = pr & 0x7FFF7FFFu;
      }

      // ---- row scales: lane 2*rw + w computes (row rw of this warp, w = 0 d_gate / 1 d_up)
      const int rw = (lane >> 1) & (kRowsPerWarp - 1);
      const int src = (rw / RPL) << 4;
      uint32_t psel = __shfl_sync(kFull, P[0], src);
      if constexpr (RPL == 2) {
        const uint32_t p1 = __shfl_sync(kFull, P[1], src);
        psel = (rw & 1) ? p1 : psel;
      }
      const uint32_t abits = (lane & 1) ? (psel & 0xFFFFu) : (psel >> 16);
      float scale, inv;
      group_scale(__uint_as_float(abits << 16), scale, inv);
      const int64_t srow0 = row0 + sub * kSubRows;
      if (lane < 2 * kRowsPerWarp) {
        const int64_t row = srow0 + 2 * warp * RPL + rw;
        if (row < M) p.gis[row * (2 * Kg) + (lane & 1) * Kg + j] = scale;
      }

      // ---- quantize d_gate / d_up rows and store 8 bytes each
#pragma unroll
      for (int e = 0; e < RPL; ++e) {
        const int sl = 2 * (h * RPL + e);
        const float ig = __shfl_sync(kFull, inv, sl);
        const float iu = __shfl_sync(kFull, inv, sl + 1);
        const int64_t row = srow0 + rho + e;
        if (row < M) {
          uint2 og, ou;
          og.x = pack_low_bytes(quant_bits(bf16_lo(dgp[e][0]), ig), quant_bits(bf16_hi(dgp[e][0]), ig),
                                quant_bits(bf16_lo(dgp[e][1]), ig), quant_bits(bf16_hi(dgp[e][1]), ig));
          og.y = pack_low_bytes(quant_bits(bf16_lo(dgp[e][2]), ig), quant_bits(bf16_hi(dgp[e][2]), ig),
                                quant_bits(bf16_lo(dgp[e][3]), ig), quant_bits(bf16_hi(dgp[e][3]), ig));
          ou.x = pack_low_bytes(quant_bits(bf16_lo(dup[e][0]), iu), quant_bits(bf16_hi(dup[e][0]), iu),
                                quant_bits(bf16_lo(dup[e][1]), iu), quant_bits(bf16_hi(dup[e][1]), iu));
          ou.y = pack_low_bytes(quant_bits(bf16_lo(dup[e][2]), iu), quant_bits(bf16_hi(dup[e][2]), iu),
                                quant_bits(bf16_lo(dup[e][3]), iu), quant_bits(bf16_hi(dup[e][3]), iu));
          int8_t* dst = p.giq + row * (2 * int64_t(K)) + j * kG + q * 8;
          *reinterpret_cast<uint2*>(dst) = og;
          *reinterpret_cast<uint2*>(dst + K) = ou;
        }
      }
    }

    // ---- tile end: column amax over the tile's tokens
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t c = cmax[k] & 0x7FFF7FFFu;
      cmax[k] = absmax_bf16x2(c, __shfl_xor_sync(kFull, c, 16)) & 0x7FFF7FFFu;
    }
    if (h == 0)
      *reinterpret_cast<uint4*>(&s.colmax[warp][q * 8]) = make_uint4(cmax[0], cmax[1], cmax[2], cmax[3]);
    if (bar_red_or(1, C::kConsumers, abort)) break;  // every consumer stops together

    if (tid < kG) {
      uint32_t m = 0;
#pragma unroll
      for (int w = 0; w < NW; ++w) m = max(m, static_cast<uint32_t>(s.colmax[w][tid]));
      float scale, inv;
      group_scale(__uint_as_float(m << 16), scale, inv);
      p.yst[int64_t(j * kG + tid) * p.Mg + i] = scale;
      s.inv_y[tid] = inv;
    }
    bar_sync(1, C::kConsumers);

    // ---- quantize y and write it transposed into the staging tile
    float iv[8];
    *reinterpret_cast<float4*>(&iv[0]) = *reinterpret_cast<const float4*>(&s.inv_y[q * 8]);
    *reinterpret_cast<float4*>(&iv[4]) = *reinterpret_cast<const float4*>(&s.inv_y[q * 8 + 4]);
#pragma unroll
    for (int sub = 0; sub < kNumSub; ++sub) {
      const int tok = sub * kSubRows + rho;         // first token (within the tile) of this lane
      const uint32_t word = static_cast<uint32_t>(tok >> 2) ^ static_cast<uint32_t>(q);
      const uint32_t boff = (word << 2) + (tok & 3);
#pragma unroll
      for (int k = 0; k < 4; ++k) {
#pragma unroll
        for (int hi = 0; hi < 2; ++hi) {
          const int ch = q * 8 + 2 * k + hi;
          const float inv = iv[2 * k + hi];
          uint8_t* row = s.yt + ch * kG;
          if constexpr (RPL == 2) {
            const float v0 = hi ? bf16_hi(yv[sub][0][k]) : bf16_lo(yv[sub][0][k]);
            const float v1 = hi ? bf16_hi(yv[sub][1][k]) : bf16_lo(yv[sub][1][k]);
            const uint32_t b2 = __byte_perm(quant_bits(v0, inv), quant_bits(v1, inv), 0x0040);
            *reinterpret_cast<uint16_t*>(row + boff) = static_cast<uint16_t>(b2);
          } else {
            const float v0 = hi ? bf16_hi(yv[sub][0][k]) : bf16_lo(yv[sub][0][k]);
            row[boff] = static_cast<uint8_t>(quant_bits(v0, inv));
          }
        }
      }
    }
    bar_sync(1, C::kConsumers);

    // ---- staging tile -> y_q_t: 16-token chunks, 8 lanes per 128-byte channel row
#pragma unroll
    for (int it = 0; it < (kG * kG / 16) / C::kConsumers; ++it) {
      const int idx = it * C::kConsumers + tid;
      const int c = idx >> 3;
      const int kc = idx & 7;
      const uint32_t x = static_cast<uint32_t>(c >> 3);   // the row's swizzle key
      const uint4 v = *reinterpret_cast<const uint4*>(s.yt + c * kG + ((kc ^ (x >> 2)) << 4));
      // logical word m sits at word m ^ (x & 3) of the physical chunk
      const bool s1 = x & 1u, s2 = x & 2u;
      const uint32_t a0 = s1 ? v.y : v.x, a1 = s1 ? v.x : v.y;
      const uint32_t a2 = s1 ? v.w : v.z, a3 = s1 ? v.z : v.w;
      const uint4 o = make_uint4(s2 ? a2 : a0, s2 ? a3 : a1, s2 ? a0 : a2, s2 ? a1 : a3);
      const int64_t tok = row0 + kc * 16;
      if (tok < M) {
        int8_t* dst = p.yqt + int64_t(j * kG + c) * M + tok;
        if (p.yqt_vec16) {
          *reinterpret_cast<uint4*>(dst) = o;
        } else {
          const uint32_t w4[4] = {o.x, o.y, o.z, o.w};
          const int nb = static_cast<int>((M - tok < 16 ? M - tok : int64_t(16)));
          for (int b = 0; b < nb; ++b) dst[b] = static_cast<int8_t>(w4[b >> 2] >> ((b & 3) * 8));
        }
      }
    }
  }
}

template <int NW, int STAGES>
__global__ void __launch_bounds__(Config<NW, STAGES>::kThreads, 1)
    fuse_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_gy,
                const Params p) {
  extern __shared__ uint8_t smem_raw[];
  auto& s = *reinterpret_cast<Smem<NW, STAGES>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~static_cast<uintptr_t>(127));
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int st = 0; st < STAGES; ++st) {
      mbar_init(smem_u32(&s.full[st]), 1);
      mbar_init(smem_u32(&s.empty[st]), NW);
    }
    fence_mbar_init();
  }
  __syncthreads();
  if (warp == NW) {
    if (lane == 0) producer<NW, STAGES>(s, &map_x, &map_gy, p);
    return;
  }
  consumer<NW, STAGES>(s, p, warp, lane);
}

}  // namespace sdq

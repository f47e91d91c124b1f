// The fused kernel of silu_dot_fwd_bwd_quant_fuse at group size 256.
//
// Same operation as sdq_kernel.cuh ("kernelgen-challenge-9-task3-silu-quant",
// outputs section and constraints list), with the page's group_size argument
// at 256: row groups of 256 channels of [d_gate | d_up] (each within its
// half), column groups of 256 tokens of y.  A 128 x 128 tile no longer holds
// whole groups, so the work unit is a 256-token x 256-channel block, which
// holds exactly one group on each axis:
//
//   * the unit arrives as sixteen 16-row stages of 16 x 256 elements per
//     input (gate, up, grad_y: 24 KB a stage) in a 4-slot ring, with the
//     128-group kernel's protocol (mbarrier per slot, the last warp to
//     release a slot issues its next load); warps 0-7 take the even stages
//     and warps 8-15 the odd ones, so each half has two slots of its own and
//     a slot waits for 8 warps;
//   * row pass: a lane owns 16 channels of one row (16 lanes a row, 2 rows a
//     warp), so a whole 256-channel row group is one half-warp: its amax
//     takes four shuffle steps and the row is quantized and stored at once;
//   * the bf16 y values of the whole unit (256 x 256, 128 KB) go to shared
//     memory; once every row is in, the column pass quantizes each channel's
//     256 tokens (a thread takes 2 channels x 32 tokens, twice; 8 threads
//     share a column group);
//   * there is one y buffer (two would not fit next to the ring), so a
//     unit's row pass waits until every thread has read its column words of
//     the unit before (each thread holds its 64 words in registers and hands
//     the tile back before its column arithmetic); the ring keeps loading
//     meanwhile.
//
// Rows past M and channels past K are zero-filled by the TMA unit; zeros
// never change an amax, and their outputs are not stored, so a tail token
// group and a shorter last channel group are quantized over what they hold.
// Every wait is bounded like the 128-group kernel's.
#pragma once

#include "sdq_kernel.cuh"

namespace sdq {

constexpr int kG2 = 256;                             // group size = unit edge
constexpr int kStageRows2 = 16;                      // token rows per stage
constexpr int kStagesPerUnit = kG2 / kStageRows2;    // 16
constexpr int kBoxBytes2 = kStageRows2 * kG2 * 2;    // one bf16 box: 8 KB
constexpr int kStageBytes2 = 3 * kBoxBytes2;         // 24 KB
constexpr int kQBoxBytes2 = kStageRows2 * kG2;       // one INT8 grad_y box: 4 KB
constexpr int kYBytes2 = kG2 * kG2 * 2;              // bf16 y of a unit: 128 KB

template <int STAGES>
struct Smem256 {
  alignas(128) uint8_t ring[STAGES][kStageBytes2];
  alignas(16) uint8_t ytile[kYBytes2];               // [token][channel], 16-byte chunks swizzled
  alignas(16) float2 scale_tab[128];
  alignas(8) uint64_t full[STAGES][2];               // per slot, alternate loads (ring_bar_index)
  alignas(8) uint64_t y_ready;                       // every thread wrote its y rows of the unit
  alignas(8) uint64_t y_free;                        // every thread finished the unit's column pass
  int released[STAGES];
  int issued;
  int abort;
};

template <int STAGES>
constexpr size_t smem_bytes256() {
  return sizeof(Smem256<STAGES>) + 128;
}

// Tensor coordinates (channel x, token y) of the boxes of load n of this CTA.
__device__ __forceinline__ void load_coords256(const Params& p, uint32_t n, int& x, int& y) {
  const int t = blockIdx.x + static_cast<int>(n / kStagesPerUnit) * gridDim.x;
  int i, j;
  tile_ij(t, p.Mg, p.Kg, i, j);
  x = j * kG2;
  y = i * kG2 + static_cast<int>(n % kStagesPerUnit) * kStageRows2;
}

// Load n of this CTA: stage n % 16 of its (n / 16)-th unit into slot n % STAGES.
template <int STAGES, bool kQdy>
__device__ __forceinline__ void issue_load256(Smem256<STAGES>& s, const CUtensorMap* mgate,
                                              const CUtensorMap* mup, const CUtensorMap* mdy,
                                              const Params& p, uint32_t n, uint64_t pol) {
  int x, r;
  load_coords256(p, n, x, r);
  const uint32_t slot = n % STAGES;
  const uint32_t fb = smem_u32(&s.full[0][0] + ring_bar_index(n, STAGES));
  mbar_arrive_expect_tx(fb, kQdy ? 2 * kBoxBytes2 + kQBoxBytes2 : kStageBytes2);
  const uint32_t dst = smem_u32(s.ring[slot]);
  tma_load_2d(dst, mgate, fb, x, r, pol);
  tma_load_2d(dst + kBoxBytes2, mup, fb, x, r, pol);
  tma_load_2d(dst + 2 * kBoxBytes2, mdy, fb, x, r, pol);
}

// Byte offset of 16-byte chunk c (0..31) of token row `tok` in the y tile:
// chunks XOR-swizzled by bits 5..7 of the token, so the column pass (8
// threads of a warp on tokens 32 apart, 4 on neighbouring channel pairs)
// reads 32 distinct banks.
__device__ __forceinline__ int y256_off(int tok, int c) {
  return tok * (kG2 * 2) + ((c ^ ((tok >> 5) & 7)) << 4);
}

// Column pass of one task: channels 2cp, 2cp+1 and tokens 32kc .. 32kc+31 of
// the unit, in two parts: the words are read from the y tile first (so the
// tile can be handed back before the arithmetic), then the column amax over
// the 8 threads (kc = 0..7) that share the channels, the two scales, codes,
// four 16-byte pieces of y_q_t rows.
__device__ __forceinline__ void column_load256(const uint8_t* yt, int cp, int kc, uint32_t (&v)[32]) {
#pragma unroll
  for (int tt = 0; tt < 32; ++tt)
    v[tt] = *reinterpret_cast<const uint32_t*>(yt + y256_off(32 * kc + tt, cp >> 2) + ((cp & 3) << 2));
}

template <bool kE4M3, bool kE8M0, bool kYsMgK>
__device__ __forceinline__ void column_quant256(const uint32_t (&v)[32], const float2* tab, const Params& p,
                                                int i, int j, int64_t row0, int valid, int cp, int kc) {
  constexpr unsigned kFull = 0xffffffffu;
  uint32_t m = absmax_bf16x2(v[0], v[1]);
#pragma unroll
  for (int tt = 2; tt < 32; ++tt) m = absmax_bf16x2(m, v[tt]);
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) m = absmax_bf16x2(m, __shfl_xor_sync(kFull, m, o));
  m &= 0x7FFF7FFFu;
  float s_lo, i_lo, s_hi, i_hi;
  group_scale<kE4M3, kE8M0>(m & 0xFFFFu, tab, s_lo, i_lo);
  group_scale<kE4M3, kE8M0>(m >> 16, tab, s_hi, i_hi);
  const int ch = j * kG2 + 2 * cp;
  const bool ch_ok = ch < p.K;
  if (kc < 2 && ch_ok)
    store_scale<kE8M0>(p.yst, kYsMgK ? int64_t(i) * p.ld_yst + ch + kc : int64_t(ch + kc) * p.ld_yst + i,
                       kc ? s_hi : s_lo);
  const bool tiny = __any_sync(kFull, i_lo < 0.0f || i_hi < 0.0f);
  const float2 pre = make_float2(i_lo < 0.0f ? kTinyPre : 1.0f, i_hi < 0.0f ? kTinyPre : 1.0f);
  const float2 inv = make_float2(fabsf(i_lo), fabsf(i_hi));
  const float2 scl = make_float2(s_lo * pre.x, s_hi * pre.y);
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t w[16];
#pragma unroll
    for (int tt = 0; tt < 16; ++tt) w[tt] = v[16 * h + tt];
    uint4 lo, hi;
    if (tiny) quant_cols<kE4M3, true>(w, inv, pre, scl, lo, hi);
    else quant_cols<kE4M3, false>(w, inv, make_float2(1.0f, 1.0f), scl, lo, hi);
    const int tok = 32 * kc + 16 * h;
    if (tok < valid && ch_ok) {
      const int nb = min(16, valid - tok);
      int8_t* dst = p.yqt + int64_t(ch) * p.ld_yqt + row0 + tok;
      store_codes(dst, lo, nb, p.yqt_vec16 != 0);
      store_codes(dst + p.ld_yqt, hi, nb, p.yqt_vec16 != 0);
    }
  }
}

template <int STAGES, bool kE4M3, bool kE8M0, bool kYsMgK, bool kY, bool kQdy>
__global__ void __launch_bounds__(kThreads, 1)
    fuse256_kernel(const __grid_constant__ CUtensorMap map_gate, const __grid_constant__ CUtensorMap map_up,
                   const __grid_constant__ CUtensorMap map_gy, const Params p) {
  constexpr unsigned kFull = 0xffffffffu;
  extern __shared__ uint8_t smem_raw[];
  auto& s = *reinterpret_cast<Smem256<STAGES>*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~static_cast<uintptr_t>(127));
  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  // row pass: lane = 16 * rr + cq owns 16-byte chunks ca, cb (8 channels
  // each) of row srow of the stage; chunks ordered so that each 8-lane
  // quarter of the warp reads 8 distinct bank groups
  const int grp = warp >> 3;   // even (0) or odd (1) stages of every unit
  const int rr = lane >> 4;
  const int cq = lane & 15;
  const int ca = 2 * cq + ((cq >> 2) & 1);
  const int cb = 2 * cq + 1 - ((cq >> 2) & 1);
  const int srow = (warp & 7) * 2 + rr;
  // column pass: thread = 8 * cp + kc, channel pairs cp and cp + 64
  const int cp0 = tid >> 3;
  const int kc = tid & 7;
  const int my_units = (p.num_tiles - static_cast<int>(blockIdx.x) + gridDim.x - 1) / gridDim.x;
  const uint32_t total = static_cast<uint32_t>(my_units) * kStagesPerUnit;
  const uint64_t pol = l2_policy_evict_first();

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
    mbar_init(smem_u32(&s.y_ready), kThreads);
    mbar_init(smem_u32(&s.y_free), kThreads);
    s.abort = 0;
    fence_mbar_init();
    // L2 prefetch of the first loads' boxes while the previous grid finishes
    // (as in the 128-group kernel)
    const uint32_t first = total < STAGES ? total : STAGES;
    for (uint32_t n = 0; n < first; ++n) {
      int x, y;
      load_coords256(p, n, x, y);
      tma_prefetch_l2_2d(&map_gate, x, y);
      tma_prefetch_l2_2d(&map_up, x, y);
      tma_prefetch_l2_2d(&map_gy, x, y);
    }
    grid_dependency_wait();
    s.issued = static_cast<int>(first);
    for (uint32_t n = 0; n < first; ++n)
      if (n != 0 || !p.withhold_first_load) issue_load256<STAGES, kQdy>(s, &map_gate, &map_up, &map_gy, p, n, pol);
  }
  grid_dependency_wait();
  grid_launch_dependents();
  __syncthreads();

  const int K = p.K;
  const int64_t M = p.M;
  const float2* tab = s.scale_tab;
  volatile int* abort_flag = &s.abort;
  const uint64_t lim = p.wait_limit_ns;
  bool ok = true;

  for (int k = 0; k < my_units && ok; ++k) {
    const int t = blockIdx.x + k * gridDim.x;
    int i, j;
    tile_ij(t, p.Mg, p.Kg, i, j);
    const int64_t row0 = int64_t(i) * kG2;
    const int valid = static_cast<int>(M - row0 < kG2 ? M - row0 : int64_t(kG2));
    const int cvalid = min(kG2, K - j * kG2);
    int8_t* giq_u = p.giq + row0 * p.ld_giq + j * kG2;
    const int64_t gis_u = row0 * p.ld_gis + j;

    // ================= row pass over this half's eight stages of the unit
    for (int sub2 = 0; sub2 < kStagesPerUnit / 2; ++sub2) {
      const int sub = 2 * sub2 + grp;
      const uint32_t n = static_cast<uint32_t>(k) * kStagesPerUnit + sub;
      const uint32_t slot = n % STAGES;
      const int r = sub * kStageRows2 + srow;   // this lane's row within the unit
      float dsc = 0.0f;
      if constexpr (kQdy) {   // INT8 grad_y: its scale per token and 128 channels
        if (r < valid && j * kG2 + 16 * cq < K) dsc = __ldg(p.gys + (row0 + r) * p.ld_gys + 2 * j + (cq >> 3));
      }
      ok = __all_sync(kFull, wait_or_abort(smem_u32(&s.full[0][0] + ring_bar_index(n, STAGES)),
                                           ring_parity(n, STAGES), lim, abort_flag));
      if (!ok) break;

      uint32_t gw[8], uw[8], dw[8];
      float2 dq[8];
      {
        const uint8_t* src = s.ring[slot] + srow * (kG2 * 2);
        const uint4 g0 = *reinterpret_cast<const uint4*>(src + ca * 16);
        const uint4 g1 = *reinterpret_cast<const uint4*>(src + cb * 16);
        const uint4 u0 = *reinterpret_cast<const uint4*>(src + kBoxBytes2 + ca * 16);
        const uint4 u1 = *reinterpret_cast<const uint4*>(src + kBoxBytes2 + cb * 16);
        gw[0] = g0.x; gw[1] = g0.y; gw[2] = g0.z; gw[3] = g0.w;
        gw[4] = g1.x; gw[5] = g1.y; gw[6] = g1.z; gw[7] = g1.w;
        uw[0] = u0.x; uw[1] = u0.y; uw[2] = u0.z; uw[3] = u0.w;
        uw[4] = u1.x; uw[5] = u1.y; uw[6] = u1.z; uw[7] = u1.w;
        if constexpr (kQdy) {
          const uint8_t* qsrc = s.ring[slot] + 2 * kBoxBytes2 + srow * kG2;
          dequant8(*reinterpret_cast<const uint2*>(qsrc + ca * 8), dsc, dq);
          dequant8(*reinterpret_cast<const uint2*>(qsrc + cb * 8), dsc, dq + 4);
        } else {
          const uint4 d0 = *reinterpret_cast<const uint4*>(src + 2 * kBoxBytes2 + ca * 16);
          const uint4 d1 = *reinterpret_cast<const uint4*>(src + 2 * kBoxBytes2 + cb * 16);
          dw[0] = d0.x; dw[1] = d0.y; dw[2] = d0.z; dw[3] = d0.w;
          dw[4] = d1.x; dw[5] = d1.y; dw[6] = d1.z; dw[7] = d1.w;
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
            issue_load256<STAGES, kQdy>(s, &map_gate, &map_up, &map_gy, p, nn, pol);
          }
        }
      }

      uint32_t yv[8], dgp[8], dup[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        if constexpr (kQdy) swiglu_bwd2f(gw[c], uw[c], dq[c], yv[c], dgp[c], dup[c]);
        else swiglu_bwd2(gw[c], uw[c], dw[c], yv[c], dgp[c], dup[c]);
      }

      // ---- y to the unit's shared tile; it was last read by the column
      // pass of the previous unit
      if (sub2 == 0 && k >= 1) {
        ok = __all_sync(kFull, wait_or_abort(smem_u32(&s.y_free), (k - 1) & 1, lim, abort_flag));
        if (!ok) break;
      }
      *reinterpret_cast<uint4*>(s.ytile + y256_off(r, ca)) = make_uint4(yv[0], yv[1], yv[2], yv[3]);
      *reinterpret_cast<uint4*>(s.ytile + y256_off(r, cb)) = make_uint4(yv[4], yv[5], yv[6], yv[7]);
      if constexpr (kY) {
        if (r < valid) {
          int8_t* yg = reinterpret_cast<int8_t*>(p.y) + 2 * ((row0 + r) * p.ld_y + int64_t(j) * kG2);
          if (ca * 8 < cvalid) st_cs_v4(yg + ca * 16, make_uint4(yv[0], yv[1], yv[2], yv[3]));
          if (cb * 8 < cvalid) st_cs_v4(yg + cb * 16, make_uint4(yv[4], yv[5], yv[6], yv[7]));
        }
      }

      // ---- row amax of d_gate (hi half) and d_up (lo half) over the 16 lanes of the row
      uint32_t a = absmax_bf16x2(dgp[0], dgp[1]), b = absmax_bf16x2(dup[0], dup[1]);
#pragma unroll
      for (int c = 2; c < 8; ++c) {
        a = absmax_bf16x2(a, dgp[c]);
        b = absmax_bf16x2(b, dup[c]);
      }
      uint32_t pr = absmax_bf16x2(__byte_perm(a, b, 0x1054), __byte_perm(a, b, 0x3276));
#pragma unroll
      for (int o = 1; o < 16; o <<= 1) pr = absmax_bf16x2(pr, __shfl_xor_sync(kFull, pr, o));
      pr &= 0x7FFF7FFFu;
      float sg, ig, su, iu;
      group_scale<kE4M3, kE8M0>(pr >> 16, tab, sg, ig);
      group_scale<kE4M3, kE8M0>(pr & 0xFFFFu, tab, su, iu);
      if (cq < 2 && r < valid)
        store_scale<kE8M0>(p.gis, gis_u + int64_t(r) * p.ld_gis + cq * (p.gis_cols >> 1), cq ? su : sg);

      if (r < valid) {
        uint4 og, ou;
        if (__any_sync(__activemask(), ig < 0.0f || iu < 0.0f)) {
          og = (ig < 0.0f) ? quant16<kE4M3, true>(dgp, -ig, sg * kTinyPre) : quant16<kE4M3, false>(dgp, ig, sg);
          ou = (iu < 0.0f) ? quant16<kE4M3, true>(dup, -iu, su * kTinyPre) : quant16<kE4M3, false>(dup, iu, su);
        } else {
          og = quant16<kE4M3, false>(dgp, ig, sg);
          ou = quant16<kE4M3, false>(dup, iu, su);
        }
        int8_t* dst = giq_u + int64_t(r) * p.ld_giq;   // (255 x 2^24 leaves int range)
        if (ca * 8 < cvalid) {
          st_cs_v2(dst + ca * 8, make_uint2(og.x, og.y));
          st_cs_v2(dst + K + ca * 8, make_uint2(ou.x, ou.y));
        }
        if (cb * 8 < cvalid) {
          st_cs_v2(dst + cb * 8, make_uint2(og.z, og.w));
          st_cs_v2(dst + K + cb * 8, make_uint2(ou.z, ou.w));
        }
      }
    }
    if (!ok) break;
    mbar_arrive(smem_u32(&s.y_ready));

    // ================= column pass of this unit: channel pairs cp0 and cp0 + 64
    ok = __all_sync(kFull, wait_or_abort(smem_u32(&s.y_ready), k & 1, lim, abort_flag));
    if (!ok) break;
    {
      uint32_t va[32], vb[32];
      column_load256(s.ytile, cp0, kc, va);
      column_load256(s.ytile, cp0 + 64, kc, vb);
      mbar_arrive(smem_u32(&s.y_free));   // the tile's words are in registers: it may be rewritten
      column_quant256<kE4M3, kE8M0, kYsMgK>(va, tab, p, i, j, row0, valid, cp0, kc);
      column_quant256<kE4M3, kE8M0, kYsMgK>(vb, tab, p, i, j, row0, valid, cp0 + 64, kc);
    }
  }

  __syncthreads();
  if (tid == 0 && *abort_flag) {
    const uint32_t issued = static_cast<uint32_t>(s.issued);
    const uint32_t first = issued > STAGES ? issued - STAGES : 0;
    for (uint32_t n = first; n < issued; ++n)
      mbar_wait(smem_u32(&s.full[0][0] + ring_bar_index(n, STAGES)), ring_parity(n, STAGES), lim);
  }
}

}  // namespace sdq

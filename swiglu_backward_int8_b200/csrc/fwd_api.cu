// C ABI of the forward-side neighbour, sdq_swiglu_q8_1 (declared in
// include/sdq.h): argument validation and the launch of the streaming kernel.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "fwd_kernel.cuh"
#include "sdq.h"

namespace sdq_internal {
int cuda_fail(cudaError_t e);   // records e for sdq_last_cuda_error (sdq_api.cu)
}

namespace {

constexpr int kMaxDevices = 64;

int fwd_cuda_fail(cudaError_t e) { return sdq_internal::cuda_fail(e); }

struct FwdDevice {
  std::once_flag once;
  cudaError_t err = cudaSuccess;
  int ctas = 0;   // resident CTAs of the kernel on the whole device
};
FwdDevice g_fwd[kMaxDevices];

}  // namespace

extern "C" {

int sdq_validate_swiglu_q8_1(const void* gate, int64_t ld_gate, const void* up, int64_t ld_up,
                             const float* w, const void* h, int64_t ld_h, const void* q8,
                             int64_t rows, int64_t inter) {
  if (rows < 0 || rows > SDQ_MAX_M || inter < 32 || inter % 32 != 0 || inter > SDQ_MAX_K)
    return SDQ_ERR_SHAPE;
  if (rows == 0) return SDQ_OK;
  if (!gate || !up || !h || !q8) return SDQ_ERR_NULL;
  if (ld_gate < inter || ld_up < inter || ld_h < inter || ld_gate > SDQ_MAX_LD ||
      ld_up > SDQ_MAX_LD || ld_h > SDQ_MAX_LD)
    return SDQ_ERR_STRIDE;
  const uintptr_t a16 = reinterpret_cast<uintptr_t>(gate) | reinterpret_cast<uintptr_t>(up) |
                        reinterpret_cast<uintptr_t>(h);
  const uintptr_t a4 = reinterpret_cast<uintptr_t>(q8) | reinterpret_cast<uintptr_t>(w);
  if ((a16 & 15u) || (a4 & 3u) || ((ld_gate | ld_up | ld_h) & 7)) return SDQ_ERR_ALIGN;
  return SDQ_OK;
}

int sdq_swiglu_q8_1(const void* gate, int64_t ld_gate, const void* up, int64_t ld_up,
                    const float* w, void* h, int64_t ld_h, void* q8, int64_t rows, int64_t inter,
                    float limit, void* stream) {
  const int st = sdq_validate_swiglu_q8_1(gate, ld_gate, up, ld_up, w, h, ld_h, q8, rows, inter);
  if (st != SDQ_OK || rows == 0) return st;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fwd_cuda_fail(e);
  if (dev < 0 || dev >= kMaxDevices) return fwd_cuda_fail(cudaErrorInvalidDevice);
  FwdDevice& fd = g_fwd[dev];
  std::call_once(fd.once, [&fd, dev] {
    int sms = 0, per_sm = 0;
    fd.err = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    if (fd.err == cudaSuccess)
      fd.err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, sdq::fwd::swiglu_q8_1_kernel,
                                                             sdq::fwd::kThreads, 0);
    fd.ctas = sms * std::max(per_sm, 1);
  });
  if (fd.err != cudaSuccess) return fwd_cuda_fail(fd.err);
  sdq::fwd::Params p;
  p.gate = static_cast<const uint8_t*>(gate);
  p.up = static_cast<const uint8_t*>(up);
  p.w = w;
  p.h = static_cast<uint8_t*>(h);
  p.q8 = static_cast<uint8_t*>(q8);
  p.rows = rows;
  p.ld_gate = ld_gate;
  p.ld_up = ld_up;
  p.ld_h = ld_h;
  p.inter = static_cast<int32_t>(inter);
  p.units_per_row = static_cast<int32_t>((inter + sdq::fwd::kUnit - 1) / sdq::fwd::kUnit);
  p.clamp = limit > 0.0f ? 1 : 0;   // false for NaN
  p.limit = p.clamp ? limit : 0.0f;
  const int64_t warps = rows * p.units_per_row;
  const int64_t need = (warps * 32 + sdq::fwd::kThreads - 1) / sdq::fwd::kThreads;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(std::min<int64_t>(need, fd.ctas)));
  cfg.blockDim = dim3(sdq::fwd::kThreads);
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, sdq::fwd::swiglu_q8_1_kernel, p);
  if (e != cudaSuccess) return fwd_cuda_fail(e);
  return SDQ_OK;
}

}  // extern "C"

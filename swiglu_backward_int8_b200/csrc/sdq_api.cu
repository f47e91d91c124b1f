// C ABI of silu_dot_fwd_bwd_quant_fuse (declared in include/sdq.h): argument
// validation, TMA descriptors, the launch of the fused sm_100a kernel, and the
// chunked host-buffer path.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstdlib>
#include <mutex>

#include "sdq.h"
#include "sdq_kernel.cuh"
#include "sdq_kernel256.cuh"

namespace {

// Pipeline depth of the kernels' shared-memory rings (compile-time
// overridable for tuning sweeps): three 48 KB stages for the 128 x 128-tile
// kernel (its two warp halves work on different slots, and a third slot
// keeps a load in flight for each), four 24 KB stages for the 256-group
// kernel (two per warp half, next to its 128 KB y buffer).
#ifndef SDQ_STAGES
#define SDQ_STAGES 3
#endif
constexpr int kStages = SDQ_STAGES;
#ifndef SDQ_STAGES256
#define SDQ_STAGES256 4
#endif
constexpr int kStages256 = SDQ_STAGES256;

constexpr int kMaxDevices = 64;

// One kernel per group size (32, 64, 128 in the 128 x 128-tile kernel; 256
// in the 256 x 256-unit kernel), output format (SDQ_FMT_* bits 0..2),
// whether bf16 y is written too, and whether grad_y comes as INT8 codes with
// scales.
using KernelFn = void (*)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const sdq::Params);
constexpr int kFormats = 8;
constexpr int kGroupSizes = 4;
constexpr int kKernels = 2 * 2 * kGroupSizes * kFormats;

template <int G, bool kY, bool kQ>
constexpr KernelFn kernel_of(int f) {
  switch (f) {
    case 0: return sdq::fuse_kernel<kStages, G, false, false, false, kY, kQ>;
    case 1: return sdq::fuse_kernel<kStages, G, true, false, false, kY, kQ>;
    case 2: return sdq::fuse_kernel<kStages, G, false, true, false, kY, kQ>;
    case 3: return sdq::fuse_kernel<kStages, G, true, true, false, kY, kQ>;
    case 4: return sdq::fuse_kernel<kStages, G, false, false, true, kY, kQ>;
    case 5: return sdq::fuse_kernel<kStages, G, true, false, true, kY, kQ>;
    case 6: return sdq::fuse_kernel<kStages, G, false, true, true, kY, kQ>;
    default: return sdq::fuse_kernel<kStages, G, true, true, true, kY, kQ>;
  }
}

template <bool kY, bool kQ>
constexpr KernelFn kernel256_of(int f) {
  switch (f) {
    case 0: return sdq::fuse256_kernel<kStages256, false, false, false, kY, kQ>;
    case 1: return sdq::fuse256_kernel<kStages256, true, false, false, kY, kQ>;
    case 2: return sdq::fuse256_kernel<kStages256, false, true, false, kY, kQ>;
    case 3: return sdq::fuse256_kernel<kStages256, true, true, false, kY, kQ>;
    case 4: return sdq::fuse256_kernel<kStages256, false, false, true, kY, kQ>;
    case 5: return sdq::fuse256_kernel<kStages256, true, false, true, kY, kQ>;
    case 6: return sdq::fuse256_kernel<kStages256, false, true, true, kY, kQ>;
    default: return sdq::fuse256_kernel<kStages256, true, true, true, kY, kQ>;
  }
}

template <bool kY, bool kQ>
KernelFn kernel_of_group(int g, int f) {
  return g == 0 ? kernel_of<32, kY, kQ>(f) : g == 1 ? kernel_of<64, kY, kQ>(f)
       : g == 2 ? kernel_of<128, kY, kQ>(f) : kernel256_of<kY, kQ>(f);
}

// Kernel number n = 32 * (2 * INT8 grad_y + y written) + 8 * (0, 1, 2, 3 for
// group size 32, 64, 128, 256) + format bits.
KernelFn kernel_at(int n) {
  const int v = n / (kGroupSizes * kFormats);   // 0..3: (y, INT8 grad_y) bits
  const int g = (n % (kGroupSizes * kFormats)) / kFormats, f = n % kFormats;
  switch (v) {
    case 0: return kernel_of_group<false, false>(g, f);
    case 1: return kernel_of_group<true, false>(g, f);
    case 2: return kernel_of_group<false, true>(g, f);
    default: return kernel_of_group<true, true>(g, f);
  }
}

bool is_group256(int n) { return (n % (kGroupSizes * kFormats)) / kFormats == 3; }

int group_index(int32_t group_size) {
  return group_size == 32 ? 0 : group_size == 64 ? 1 : group_size == 128 ? 2 : 3;
}

KernelFn kernel_for(int32_t group_size, uint32_t format, bool y, bool qdy) {
  return kernel_at(((qdy ? 2 : 0) + (y ? 1 : 0)) * kGroupSizes * kFormats + group_index(group_size) * kFormats +
                   static_cast<int>(format & (kFormats - 1)));
}

// Dynamic shared memory of the kernel for a group size.
size_t smem_for(int32_t group_size) {
  return group_size == 256 ? sdq::smem_bytes256<kStages256>() : sdq::smem_bytes<kStages>();
}

bool group_size_supported(int32_t g) { return g == 32 || g == 64 || g == SDQ_GROUP_SIZE || g == 256; }
thread_local int t_last_cuda_error = 0;

int cuda_fail(cudaError_t e) {
  t_last_cuda_error = static_cast<int>(e);
  cudaGetLastError();  // clear the sticky-free error so the next call starts clean
  return SDQ_ERR_CUDA;
}

}  // namespace

// Shared with the library's other translation units (fwd_api.cu).
namespace sdq_internal {
int cuda_fail(cudaError_t e) { return ::cuda_fail(e); }
}  // namespace sdq_internal

namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

uint64_t wait_limit_ns() {
  static uint64_t v = [] {
    const char* e = std::getenv("SDQ_WAIT_LIMIT_MS");
    const long long ms = e ? std::atoll(e) : 0;
    return static_cast<uint64_t>(ms > 0 ? ms : 4000) * 1000000ull;
  }();
  return v;
}

struct DeviceState {
  std::once_flag init;
  cudaError_t init_err = cudaSuccess;
  int sms = 0;
  // host-buffer pipeline: copy streams and events, guarded by `mu`
  std::mutex mu;
  bool pipe_ready = false;
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t start = nullptr, in_ready[2] = {}, out_ready[2] = {}, buf_free[2] = {};
};
DeviceState g_dev[kMaxDevices];

int current_device(DeviceState** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= kMaxDevices) return cuda_fail(cudaErrorInvalidDevice);
  DeviceState& d = g_dev[dev];
  std::call_once(d.init, [&d, dev] {
    d.init_err = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
    for (int n = 0; n < kKernels; ++n) {
      const auto kernel = kernel_at(n);
      const size_t smem = is_group256(n) ? sdq::smem_bytes256<kStages256>() : sdq::smem_bytes<kStages>();
      if (d.init_err == cudaSuccess)
        d.init_err = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          static_cast<int>(smem));
      int blocks = 0;
      if (d.init_err == cudaSuccess)
        d.init_err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&blocks, kernel, sdq::kThreads, smem);
      if (d.init_err == cudaSuccess && blocks < 1) d.init_err = cudaErrorLaunchOutOfResources;
    }
  });
  if (d.init_err != cudaSuccess) return cuda_fail(d.init_err);
  *out = &d;
  return SDQ_OK;
}

// A [rows, inner] row-major array of bf16 (or, with `bytes`, 8-bit codes)
// read in boxes of 64 rows x 128 elements.
int make_map(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows,
             uint64_t row_bytes, bool bytes = false, bool group256 = false) {
  auto fn = encode_fn();
  if (!fn) return cuda_fail(cudaErrorNotSupported);
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {row_bytes};
  // boxes of 64 rows x 128 elements, or 32 rows x 256 for the 256-group kernel
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(group256 ? sdq::kG2 : sdq::kG),
                             static_cast<cuuint32_t>(group256 ? sdq::kStageRows2 : sdq::kStageRows)};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, bytes ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                  const_cast<void*>(base), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
  return SDQ_OK;
}

// One call's arrays and leading dimensions (elements from one row to the
// next), as sdq_fuse_strided takes them.
struct Arrays {
  const void* gate; int64_t ld_gate;
  const void* up;   int64_t ld_up;
  const void* gy;   int64_t ld_gy;
  void* giq; int64_t ld_giq;
  void* gis; int64_t ld_gis;
  void* yqt; int64_t ld_yqt;
  void* yst; int64_t ld_yst;
  void* y = nullptr; int64_t ld_y = 0;   // optional bf16 y
  const void* gys = nullptr; int64_t ld_gys = 0;   // set: gy holds INT8 codes, these their scales
};

// Contiguous arrays of the page's layout: x = [gate | up] [M, 2K], grad_y
// [M, K], the outputs packed.
Arrays packed(const void* x, const void* gy, void* giq, void* gis, void* yqt, void* yst, int64_t M,
              int64_t K, int32_t group_size, uint32_t format) {
  const int64_t gsz = group_size > 0 ? group_size : 1;
  Arrays a;
  a.gate = x;
  a.ld_gate = 2 * K;
  a.up = x ? static_cast<const uint8_t*>(x) + 2 * K : nullptr;   // bf16: K elements on
  a.ld_up = 2 * K;
  a.gy = gy;
  a.ld_gy = K;
  a.giq = giq;
  a.ld_giq = 2 * K;
  a.gis = gis;
  a.ld_gis = 2 * ((K + gsz - 1) / gsz);
  a.yqt = yqt;
  a.ld_yqt = M;
  a.yst = yst;
  a.ld_yst = (format & SDQ_FMT_YS_MG_K) ? K : (M + gsz - 1) / gsz;
  return a;
}

// Launch on validated arguments (M > 0).  `format`: SDQ_FMT_* bits;
// `limit_ns` = 0: the default wait limit; `withhold` = 1 only for the
// failure-path test hook.
int launch(const Arrays& a, int64_t M, int64_t K, int32_t group_size, uint32_t format,
           cudaStream_t stream, uint64_t limit_ns = 0, int withhold = 0) {
  DeviceState* d = nullptr;
  int st = current_device(&d);
  if (st != SDQ_OK) return st;
  const bool g256 = group_size == 256;
  const int64_t unit = g256 ? sdq::kG2 : sdq::kG;   // tile / unit edge
  CUtensorMap mgate, mup, mdy;
  if ((st = make_map(&mgate, a.gate, K, M, 2 * a.ld_gate, false, g256)) != SDQ_OK) return st;
  if ((st = make_map(&mup, a.up, K, M, 2 * a.ld_up, false, g256)) != SDQ_OK) return st;
  const bool qdy = a.gys != nullptr;
  if ((st = make_map(&mdy, a.gy, K, M, (qdy ? 1 : 2) * a.ld_gy, qdy, g256)) != SDQ_OK) return st;
  sdq::Params p;
  p.giq = static_cast<int8_t*>(a.giq);
  p.gis = a.gis;
  p.yqt = static_cast<int8_t*>(a.yqt);
  p.yst = a.yst;
  p.M = M;
  p.K = static_cast<int32_t>(K);
  p.Kg = static_cast<int32_t>((K + unit - 1) / unit);
  p.Mg = static_cast<int32_t>((M + unit - 1) / unit);
  p.gis_cols = static_cast<int32_t>(2 * ((K + group_size - 1) / group_size));
  p.ld_giq = static_cast<int32_t>(a.ld_giq);
  p.ld_gis = static_cast<int32_t>(a.ld_gis);
  p.ld_yqt = a.ld_yqt;
  p.y = static_cast<uint8_t*>(a.y);
  p.ld_y = a.ld_y;
  p.gys = static_cast<const float*>(a.gys);
  p.ld_gys = a.ld_gys;
  p.ld_yst = a.ld_yst;
  p.num_tiles = p.Mg * p.Kg;
  p.yqt_vec16 = (a.ld_yqt % 16 == 0) ? 1 : 0;
  p.wait_limit_ns = limit_ns ? limit_ns : wait_limit_ns();
  p.withhold_first_load = withhold;
  const int grid = std::min(p.num_tiles, d->sms);
  // Programmatic stream serialization: this launch may begin while the
  // previous kernel of the stream drains; the kernel's griddepcontrol.wait
  // keeps every global access behind that kernel's completion.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(sdq::kThreads);
  cfg.dynamicSmemBytes = smem_for(group_size);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kernel_for(group_size, format, a.y != nullptr, qdy), mgate, mup, mdy, p);
  if (e != cudaSuccess) return cuda_fail(e);
  e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  return SDQ_OK;
}

size_t align256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

struct ChunkLayout {
  size_t x, gy, giq, gis, yqt, yst, total;  // byte offsets inside one buffer set
};

ChunkLayout chunk_layout(int64_t CR, int64_t K) {
  const int64_t Kg = (K + sdq::kG - 1) / sdq::kG;
  ChunkLayout L;
  size_t off = 0;
  L.x = off;   off += align256(size_t(CR) * 2 * K * 2);
  L.gy = off;  off += align256(size_t(CR) * K * 2);
  L.giq = off; off += align256(size_t(CR) * 2 * K);
  L.gis = off; off += align256(size_t(CR) * 2 * Kg * 4);
  L.yqt = off; off += align256(size_t(K) * CR);
  L.yst = off; off += align256(size_t(K) * (CR / sdq::kG) * 4);
  L.total = off;
  return L;
}

int64_t choose_chunk_rows(int64_t M, int64_t K) {
  // Aim for at least four chunks so copies and kernels overlap, with each
  // chunk's inputs at most ~64 MB.
  const int64_t by_count = ((M + 3) / 4 + sdq::kG - 1) / sdq::kG * sdq::kG;
  int64_t by_bytes = (int64_t(64) << 20) / (6 * K) / sdq::kG * sdq::kG;
  by_bytes = std::max<int64_t>(by_bytes, sdq::kG);
  return std::max<int64_t>(sdq::kG, std::min(by_count, by_bytes));
}

}  // namespace

extern "C" {

const char* sdq_version(void) { return "0.1.0"; }

int sdq_last_cuda_error(void) { return t_last_cuda_error; }

const char* sdq_status_string(int status) {
  switch (status) {
    case SDQ_OK: return "SDQ_OK";
    case SDQ_ERR_NULL: return "SDQ_ERR_NULL: a required pointer is NULL";
    case SDQ_ERR_GROUP: return "SDQ_ERR_GROUP: group_size must be 32, 64, 128 or 256 (128 for the host-buffer entry points)";
    case SDQ_ERR_SHAPE: return "SDQ_ERR_SHAPE: need M >= 0 and K a positive multiple of 16 within the size limits";
    case SDQ_ERR_ALIGN: return "SDQ_ERR_ALIGN: x, grad_y, grad_input_q, y_q_t need 16-byte and scales 4-byte alignment";
    case SDQ_ERR_CUDA: return "SDQ_ERR_CUDA: a CUDA call failed (see sdq_last_cuda_error)";
    case SDQ_ERR_TIMEOUT: return "SDQ_ERR_TIMEOUT: a device-side wait ran past its limit";
    case SDQ_ERR_WORKSPACE: return "SDQ_ERR_WORKSPACE: workspace too small or misaligned";
    case SDQ_ERR_TOO_LARGE: return "SDQ_ERR_TOO_LARGE: K exceeds what fits in the fixed scratch of sdq_fuse_host_noalloc (SDQ_NOALLOC_MAX_K)";
    case SDQ_ERR_FORMAT: return "SDQ_ERR_FORMAT: unknown bits in the output format";
    case SDQ_ERR_STRIDE: return "SDQ_ERR_STRIDE: a leading dimension is smaller than its row or above SDQ_MAX_LD";
    default: return "SDQ_ERR_UNKNOWN";
  }
}

int sdq_validate_strided(const void* gate, int64_t ld_gate, const void* up, int64_t ld_up,
                         const void* grad_y, int64_t ld_grad_y, const void* grad_input_q,
                         int64_t ld_grad_input_q, const void* grad_input_s, int64_t ld_grad_input_s,
                         const void* y_q_t, int64_t ld_y_q_t, const void* y_s_t, int64_t ld_y_s_t,
                         const void* y, int64_t ld_y, int64_t M, int64_t K, int32_t group_size,
                         uint32_t format) {
  if (format & ~static_cast<uint32_t>(SDQ_FMT_E4M3 | SDQ_FMT_E8M0 | SDQ_FMT_YS_MG_K))
    return SDQ_ERR_FORMAT;
  if (!group_size_supported(group_size)) return SDQ_ERR_GROUP;
  if (M < 0 || K < 1 || K % SDQ_K_MULTIPLE != 0 || M > SDQ_MAX_M || K > SDQ_MAX_K)
    return SDQ_ERR_SHAPE;
  const int64_t tiles = ((M + SDQ_GROUP_SIZE - 1) / SDQ_GROUP_SIZE) *
                        ((K + SDQ_GROUP_SIZE - 1) / SDQ_GROUP_SIZE);
  if (tiles > INT32_MAX) return SDQ_ERR_SHAPE;
  if (M == 0) return SDQ_OK;
  if (!gate || !up || !grad_y || !grad_input_q || !grad_input_s || !y_q_t || !y_s_t)
    return SDQ_ERR_NULL;
  const int64_t groups_m = (M + group_size - 1) / group_size;
  const int64_t need_yst = (format & SDQ_FMT_YS_MG_K) ? K : groups_m;
  const int64_t lds[7] = {ld_gate, ld_up, ld_grad_y, ld_grad_input_q, ld_grad_input_s, ld_y_q_t, ld_y_s_t};
  const int64_t need[7] = {K, K, K, 2 * K, 2 * ((K + group_size - 1) / group_size), M, need_yst};
  for (int k = 0; k < 7; ++k)
    if (lds[k] < need[k] || lds[k] > SDQ_MAX_LD) return SDQ_ERR_STRIDE;
  if (ld_grad_input_q > SDQ_MAX_LD_ROWS || ld_grad_input_s > SDQ_MAX_LD_ROWS) return SDQ_ERR_STRIDE;
  const uintptr_t a16 = reinterpret_cast<uintptr_t>(gate) | reinterpret_cast<uintptr_t>(up) |
                        reinterpret_cast<uintptr_t>(grad_y) | reinterpret_cast<uintptr_t>(grad_input_q) |
                        reinterpret_cast<uintptr_t>(y_q_t);
  const uintptr_t a4 = reinterpret_cast<uintptr_t>(grad_input_s) | reinterpret_cast<uintptr_t>(y_s_t);
  if ((a16 & 15u) || (!(format & SDQ_FMT_E8M0) && (a4 & 3u))) return SDQ_ERR_ALIGN;
  // rows of the bf16 inputs start on 16 bytes (tensor-map strides), rows of
  // grad_input_q on 16 bytes (vector stores)
  if ((ld_gate | ld_up | ld_grad_y) & 7 || ld_grad_input_q & 15) return SDQ_ERR_ALIGN;
  if (y) {   // optional bf16 y: rows on 16 bytes
    if (ld_y < K || ld_y > SDQ_MAX_LD) return SDQ_ERR_STRIDE;
    if ((reinterpret_cast<uintptr_t>(y) & 15u) || (ld_y & 7)) return SDQ_ERR_ALIGN;
  }
  return SDQ_OK;
}

int sdq_validate_format(const void* x, const void* grad_y, const void* grad_input_q,
                        const void* grad_input_s, const void* y_q_t, const void* y_s_t, int64_t M,
                        int64_t K, int32_t group_size, uint32_t format) {
  const Arrays a = packed(x, grad_y, const_cast<void*>(grad_input_q), const_cast<void*>(grad_input_s),
                          const_cast<void*>(y_q_t), const_cast<void*>(y_s_t), M, K, group_size, format);
  return sdq_validate_strided(a.gate, a.ld_gate, a.up, a.ld_up, a.gy, a.ld_gy, a.giq, a.ld_giq, a.gis,
                              a.ld_gis, a.yqt, a.ld_yqt, a.yst, a.ld_yst, nullptr, 0, M, K, group_size,
                              format);
}

int sdq_validate(const void* x, const void* grad_y, const int8_t* grad_input_q,
                 const float* grad_input_s, const int8_t* y_q_t, const float* y_s_t, int64_t M,
                 int64_t K, int32_t group_size) {
  return sdq_validate_format(x, grad_y, grad_input_q, grad_input_s, y_q_t, y_s_t, M, K, group_size, 0);
}

int sdq_fuse_format(const void* x, const void* grad_y, void* grad_input_q, void* grad_input_s,
                    void* y_q_t, void* y_s_t, int64_t M, int64_t K, int32_t group_size,
                    uint32_t format, void* stream) {
  const int st = sdq_validate_format(x, grad_y, grad_input_q, grad_input_s, y_q_t, y_s_t, M, K,
                                     group_size, format);
  if (st != SDQ_OK || M == 0) return st;
  return launch(packed(x, grad_y, grad_input_q, grad_input_s, y_q_t, y_s_t, M, K, group_size, format),
                M, K, group_size, format, static_cast<cudaStream_t>(stream));
}

int sdq_fuse_strided(const void* gate, int64_t ld_gate, const void* up, int64_t ld_up,
                     const void* grad_y, int64_t ld_grad_y, void* grad_input_q,
                     int64_t ld_grad_input_q, void* grad_input_s, int64_t ld_grad_input_s,
                     void* y_q_t, int64_t ld_y_q_t, void* y_s_t, int64_t ld_y_s_t, void* y,
                     int64_t ld_y, int64_t M, int64_t K, int32_t group_size, uint32_t format,
                     void* stream) {
  const int st = sdq_validate_strided(gate, ld_gate, up, ld_up, grad_y, ld_grad_y, grad_input_q,
                                      ld_grad_input_q, grad_input_s, ld_grad_input_s, y_q_t, ld_y_q_t,
                                      y_s_t, ld_y_s_t, y, ld_y, M, K, group_size, format);
  if (st != SDQ_OK || M == 0) return st;
  const Arrays a = {gate, ld_gate, up, ld_up, grad_y, ld_grad_y, grad_input_q, ld_grad_input_q,
                    grad_input_s, ld_grad_input_s, y_q_t, ld_y_q_t, y_s_t, ld_y_s_t, y, ld_y};
  return launch(a, M, K, group_size, format, static_cast<cudaStream_t>(stream));
}

int sdq_validate_int8_grad_y(const void* gate, int64_t ld_gate, const void* up, int64_t ld_up,
                             const void* grad_y_q, int64_t ld_grad_y_q, const float* grad_y_s,
                             int64_t ld_grad_y_s, const void* grad_input_q, int64_t ld_grad_input_q,
                             const void* grad_input_s, int64_t ld_grad_input_s, const void* y_q_t,
                             int64_t ld_y_q_t, const void* y_s_t, int64_t ld_y_s_t, const void* y,
                             int64_t ld_y, int64_t M, int64_t K, int32_t group_size,
                             uint32_t format) {
  const int st = sdq_validate_strided(gate, ld_gate, up, ld_up, grad_y_q, ld_grad_y_q, grad_input_q,
                                      ld_grad_input_q, grad_input_s, ld_grad_input_s, y_q_t,
                                      ld_y_q_t, y_s_t, ld_y_s_t, y, ld_y, M, K, group_size, format);
  if (st != SDQ_OK || M == 0) return st;
  if (!grad_y_s) return SDQ_ERR_NULL;
  if (ld_grad_y_s < (K + SDQ_GROUP_SIZE - 1) / SDQ_GROUP_SIZE || ld_grad_y_s > SDQ_MAX_LD)
    return SDQ_ERR_STRIDE;
  // code rows start on 16 bytes (tensor-map stride); scales are fp32
  if ((ld_grad_y_q & 15) || (reinterpret_cast<uintptr_t>(grad_y_s) & 3u)) return SDQ_ERR_ALIGN;
  return SDQ_OK;
}

int sdq_fuse_int8_grad_y(const void* gate, int64_t ld_gate, const void* up, int64_t ld_up,
                         const void* grad_y_q, int64_t ld_grad_y_q, const float* grad_y_s,
                         int64_t ld_grad_y_s, void* grad_input_q, int64_t ld_grad_input_q,
                         void* grad_input_s, int64_t ld_grad_input_s, void* y_q_t, int64_t ld_y_q_t,
                         void* y_s_t, int64_t ld_y_s_t, void* y, int64_t ld_y, int64_t M, int64_t K,
                         int32_t group_size, uint32_t format, void* stream) {
  const int st = sdq_validate_int8_grad_y(gate, ld_gate, up, ld_up, grad_y_q, ld_grad_y_q, grad_y_s,
                                          ld_grad_y_s, grad_input_q, ld_grad_input_q, grad_input_s,
                                          ld_grad_input_s, y_q_t, ld_y_q_t, y_s_t, ld_y_s_t, y, ld_y,
                                          M, K, group_size, format);
  if (st != SDQ_OK || M == 0) return st;
  const Arrays a = {gate, ld_gate, up, ld_up, grad_y_q, ld_grad_y_q, grad_input_q, ld_grad_input_q,
                    grad_input_s, ld_grad_input_s, y_q_t, ld_y_q_t, y_s_t, ld_y_s_t, y, ld_y,
                    grad_y_s, ld_grad_y_s};
  return launch(a, M, K, group_size, format, static_cast<cudaStream_t>(stream));
}

int sdq_fuse(const void* x, const void* grad_y, int8_t* grad_input_q, float* grad_input_s,
             int8_t* y_q_t, float* y_s_t, int64_t M, int64_t K, int32_t group_size, void* stream) {
  return sdq_fuse_format(x, grad_y, grad_input_q, grad_input_s, y_q_t, y_s_t, M, K, group_size, 0,
                         stream);
}

size_t sdq_fuse_host_workspace_bytes(int64_t M, int64_t K, int64_t chunk_rows) {
  if (M < 1 || K < 1 || K % SDQ_K_MULTIPLE != 0 || K > SDQ_MAX_K || M > SDQ_MAX_M) return 0;
  if (chunk_rows < 0 || chunk_rows % SDQ_GROUP_SIZE != 0) return 0;
  const int64_t CR = chunk_rows ? chunk_rows : choose_chunk_rows(M, K);
  return 2 * chunk_layout(CR, K).total;
}

int sdq_fuse_host(const void* x, const void* grad_y, int8_t* grad_input_q, float* grad_input_s,
                  int8_t* y_q_t, float* y_s_t, int64_t M, int64_t K, int32_t group_size,
                  void* workspace, size_t workspace_bytes, int64_t chunk_rows, void* stream) {
  if (group_size != SDQ_GROUP_SIZE) return SDQ_ERR_GROUP;
  if (M < 0 || K < 1 || K % SDQ_K_MULTIPLE != 0 || M > SDQ_MAX_M || K > SDQ_MAX_K ||
      chunk_rows < 0 || chunk_rows % SDQ_GROUP_SIZE != 0)
    return SDQ_ERR_SHAPE;
  if (M == 0) return SDQ_OK;
  if (!x || !grad_y || !grad_input_q || !grad_input_s || !y_q_t || !y_s_t) return SDQ_ERR_NULL;
  if (!workspace) return SDQ_ERR_NULL;
  const int64_t CR = chunk_rows ? chunk_rows : choose_chunk_rows(M, K);
  const ChunkLayout L = chunk_layout(CR, K);
  if (workspace_bytes < 2 * L.total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return SDQ_ERR_WORKSPACE;

  DeviceState* d = nullptr;
  int st = current_device(&d);
  if (st != SDQ_OK) return st;
  std::lock_guard<std::mutex> lock(d->mu);
  cudaError_t e = cudaSuccess;
  if (!d->pipe_ready) {
    if ((e = cudaStreamCreateWithFlags(&d->h2d, cudaStreamNonBlocking)) != cudaSuccess) return cuda_fail(e);
    if ((e = cudaStreamCreateWithFlags(&d->d2h, cudaStreamNonBlocking)) != cudaSuccess) return cuda_fail(e);
    cudaEvent_t* evs[] = {&d->start, &d->in_ready[0], &d->in_ready[1], &d->out_ready[0],
                          &d->out_ready[1], &d->buf_free[0], &d->buf_free[1]};
    for (cudaEvent_t* ev : evs)
      if ((e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming)) != cudaSuccess) return cuda_fail(e);
    d->pipe_ready = true;
  }
  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const int64_t Kg = (K + SDQ_GROUP_SIZE - 1) / SDQ_GROUP_SIZE;
  const int64_t Mg = (M + SDQ_GROUP_SIZE - 1) / SDQ_GROUP_SIZE;
  const auto* xh = static_cast<const uint8_t*>(x);
  const auto* gh = static_cast<const uint8_t*>(grad_y);
  auto* ws = static_cast<uint8_t*>(workspace);

#define SDQ_CHECK(call)                         \
  do {                                          \
    if ((e = (call)) != cudaSuccess) return cuda_fail(e); \
  } while (0)

  // Order everything after the work already queued on the caller's stream.
  SDQ_CHECK(cudaEventRecord(d->start, cs));
  SDQ_CHECK(cudaStreamWaitEvent(d->h2d, d->start, 0));
  SDQ_CHECK(cudaStreamWaitEvent(d->d2h, d->start, 0));
  const int64_t nchunks = (M + CR - 1) / CR;
  for (int64_t c = 0; c < nchunks; ++c) {
    const int b = static_cast<int>(c & 1);
    uint8_t* base = ws + b * L.total;
    const int64_t m0 = c * CR;
    const int64_t mc = std::min(CR, M - m0);
    const int64_t mcg = (mc + SDQ_GROUP_SIZE - 1) / SDQ_GROUP_SIZE;
    // host -> device (after the chunk that last used this buffer set has left)
    if (c >= 2) SDQ_CHECK(cudaStreamWaitEvent(d->h2d, d->buf_free[b], 0));
    SDQ_CHECK(cudaMemcpyAsync(base + L.x, xh + m0 * 4 * K, size_t(mc) * 4 * K,
                              cudaMemcpyHostToDevice, d->h2d));
    SDQ_CHECK(cudaMemcpyAsync(base + L.gy, gh + m0 * 2 * K, size_t(mc) * 2 * K,
                              cudaMemcpyHostToDevice, d->h2d));
    SDQ_CHECK(cudaEventRecord(d->in_ready[b], d->h2d));
    // kernel on the caller's stream
    SDQ_CHECK(cudaStreamWaitEvent(cs, d->in_ready[b], 0));
    st = launch(packed(base + L.x, base + L.gy, base + L.giq, base + L.gis, base + L.yqt, base + L.yst,
                       mc, K, SDQ_GROUP_SIZE, 0),
                mc, K, SDQ_GROUP_SIZE, 0, cs);
    if (st != SDQ_OK) return st;
    SDQ_CHECK(cudaEventRecord(d->out_ready[b], cs));
    // device -> host
    SDQ_CHECK(cudaStreamWaitEvent(d->d2h, d->out_ready[b], 0));
    SDQ_CHECK(cudaMemcpyAsync(grad_input_q + m0 * 2 * K, base + L.giq, size_t(mc) * 2 * K,
                              cudaMemcpyDeviceToHost, d->d2h));
    SDQ_CHECK(cudaMemcpyAsync(grad_input_s + m0 * 2 * Kg, base + L.gis, size_t(mc) * 2 * Kg * 4,
                              cudaMemcpyDeviceToHost, d->d2h));
    SDQ_CHECK(cudaMemcpy2DAsync(y_q_t + m0, size_t(M), base + L.yqt, size_t(mc), size_t(mc),
                                size_t(K), cudaMemcpyDeviceToHost, d->d2h));
    SDQ_CHECK(cudaMemcpy2DAsync(y_s_t + m0 / SDQ_GROUP_SIZE, size_t(Mg) * 4, base + L.yst,
                                size_t(mcg) * 4, size_t(mcg) * 4, size_t(K),
                                cudaMemcpyDeviceToHost, d->d2h));
    SDQ_CHECK(cudaEventRecord(d->buf_free[b], d->d2h));
  }
  // The caller's stream completes only after the last copies have landed.
  SDQ_CHECK(cudaStreamWaitEvent(cs, d->buf_free[(nchunks - 1) & 1], 0));
  if (nchunks > 1) SDQ_CHECK(cudaStreamWaitEvent(cs, d->buf_free[nchunks & 1], 0));
#undef SDQ_CHECK
  return SDQ_OK;
}

}  // extern "C"

namespace {

// Staging area of sdq_fuse_host_noalloc: one chunk of x and grad_y and of the
// four outputs.  In host code this name is only a stand-in; the kernel gets
// the device address looked up per device below.
static __device__ __align__(256) uint8_t g_noalloc_scratch[SDQ_NOALLOC_SCRATCH_BYTES];

// The array's device address per device, looked up by the first call that
// succeeds in doing so (a failed lookup is not remembered: the next call
// tries again).
struct NoallocDevice {
  std::mutex mu;
  uint8_t* ptr = nullptr;
};
NoallocDevice g_noalloc[kMaxDevices];

// Largest multiple of 128 rows whose single buffer set fits in the array.
int64_t noalloc_chunk_rows(int64_t K) {
  int64_t rows = 0;
  for (int64_t cr = SDQ_GROUP_SIZE; chunk_layout(cr, K).total <= SDQ_NOALLOC_SCRATCH_BYTES;
       cr += SDQ_GROUP_SIZE)
    rows = cr;
  return rows;
}

}  // namespace

extern "C" {

int sdq_fuse_host_noalloc(const void* x, const void* grad_y, int8_t* grad_input_q,
                          float* grad_input_s, int8_t* y_q_t, float* y_s_t, int64_t M, int64_t K,
                          int32_t group_size, void* stream) {
  if (group_size != SDQ_GROUP_SIZE) return SDQ_ERR_GROUP;
  if (M < 0 || K < 1 || K % SDQ_K_MULTIPLE != 0 || M > SDQ_MAX_M || K > SDQ_MAX_K)
    return SDQ_ERR_SHAPE;
  if (K > SDQ_NOALLOC_MAX_K) return SDQ_ERR_TOO_LARGE;
  if (M == 0) return SDQ_OK;
  if (!x || !grad_y || !grad_input_q || !grad_input_s || !y_q_t || !y_s_t) return SDQ_ERR_NULL;
  const int64_t max_rows = noalloc_chunk_rows(K);
  if (max_rows < SDQ_GROUP_SIZE) return SDQ_ERR_TOO_LARGE;
  const int64_t CR = std::min(max_rows, (M + SDQ_GROUP_SIZE - 1) / SDQ_GROUP_SIZE * SDQ_GROUP_SIZE);
  const ChunkLayout L = chunk_layout(CR, K);

  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (dev < 0 || dev >= kMaxDevices) return cuda_fail(cudaErrorInvalidDevice);
  NoallocDevice& nd = g_noalloc[dev];
  uint8_t* base = nullptr;
  {
    std::lock_guard<std::mutex> lock(nd.mu);
    if (!nd.ptr) {
      void* p = nullptr;
      if ((e = cudaGetSymbolAddress(&p, g_noalloc_scratch)) != cudaSuccess) return cuda_fail(e);
      nd.ptr = static_cast<uint8_t*>(p);
    }
    base = nd.ptr;
  }

  cudaStream_t cs = static_cast<cudaStream_t>(stream);
  const int64_t Kg = (K + SDQ_GROUP_SIZE - 1) / SDQ_GROUP_SIZE;
  const int64_t Mg = (M + SDQ_GROUP_SIZE - 1) / SDQ_GROUP_SIZE;
  const auto* xh = static_cast<const uint8_t*>(x);
  const auto* gh = static_cast<const uint8_t*>(grad_y);
  for (int64_t m0 = 0; m0 < M; m0 += CR) {
    const int64_t mc = std::min(CR, M - m0);
    const int64_t mcg = (mc + SDQ_GROUP_SIZE - 1) / SDQ_GROUP_SIZE;
    if ((e = cudaMemcpyAsync(base + L.x, xh + m0 * 4 * K, size_t(mc) * 4 * K,
                             cudaMemcpyHostToDevice, cs)) != cudaSuccess)
      return cuda_fail(e);
    if ((e = cudaMemcpyAsync(base + L.gy, gh + m0 * 2 * K, size_t(mc) * 2 * K,
                             cudaMemcpyHostToDevice, cs)) != cudaSuccess)
      return cuda_fail(e);
    const int st = launch(packed(base + L.x, base + L.gy, base + L.giq, base + L.gis, base + L.yqt,
                                 base + L.yst, mc, K, SDQ_GROUP_SIZE, 0),
                          mc, K, SDQ_GROUP_SIZE, 0, cs);
    if (st != SDQ_OK) return st;
    if ((e = cudaMemcpyAsync(grad_input_q + m0 * 2 * K, base + L.giq, size_t(mc) * 2 * K,
                             cudaMemcpyDeviceToHost, cs)) != cudaSuccess)
      return cuda_fail(e);
    if ((e = cudaMemcpyAsync(grad_input_s + m0 * 2 * Kg, base + L.gis, size_t(mc) * 2 * Kg * 4,
                             cudaMemcpyDeviceToHost, cs)) != cudaSuccess)
      return cuda_fail(e);
    if ((e = cudaMemcpy2DAsync(y_q_t + m0, size_t(M), base + L.yqt, size_t(mc), size_t(mc),
                               size_t(K), cudaMemcpyDeviceToHost, cs)) != cudaSuccess)
      return cuda_fail(e);
    if ((e = cudaMemcpy2DAsync(y_s_t + m0 / SDQ_GROUP_SIZE, size_t(Mg) * 4, base + L.yst,
                               size_t(mcg) * 4, size_t(mcg) * 4, size_t(K),
                               cudaMemcpyDeviceToHost, cs)) != cudaSuccess)
      return cuda_fail(e);
  }
  return SDQ_OK;
}

int sdq_fuse_test_stall(const void* x, const void* grad_y, int8_t* grad_input_q,
                        float* grad_input_s, int8_t* y_q_t, float* y_s_t, int64_t M, int64_t K,
                        int32_t group_size, int64_t wait_limit_ns, void* stream) {
  const int st = sdq_validate(x, grad_y, grad_input_q, grad_input_s, y_q_t, y_s_t, M, K, group_size);
  if (st != SDQ_OK || M == 0) return st;
  if (wait_limit_ns < 1000 || wait_limit_ns > 1000000000) return SDQ_ERR_SHAPE;
  return launch(packed(x, grad_y, grad_input_q, grad_input_s, y_q_t, y_s_t, M, K, group_size, 0), M,
                K, group_size, 0, static_cast<cudaStream_t>(stream), static_cast<uint64_t>(wait_limit_ns),
                1);
}

int sdq_device_status(void* stream) {
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  int v = 0;
  if ((e = cudaMemcpyFromSymbol(&v, sdq::g_sdq_dev_status, sizeof v)) != cudaSuccess) return cuda_fail(e);
  if (v) {
    const int zero = 0;
    if ((e = cudaMemcpyToSymbol(sdq::g_sdq_dev_status, &zero, sizeof zero)) != cudaSuccess)
      return cuda_fail(e);
    return SDQ_ERR_TIMEOUT;
  }
  return SDQ_OK;
}

}  // extern "C"

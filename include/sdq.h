/*
 * sdq.h -- C ABI of the B200 (sm_100a) implementation of
 * silu_dot_fwd_bwd_quant_fuse: fused SwiGLU forward recompute, backward, and
 * dual-axis INT8 quantization.
 *
 * Source of the operation: "kernelgen-challenge-9-task3-silu-quant"
 *   - entry point section: silu_dot_fwd_bwd_quant_fuse(x, grad_y,
 *     grad_input_q, grad_input_s, y_q_t, y_s_t, group_size=128), outputs
 *     preallocated by the caller and written in place;
 *   - outputs section: recompute y = silu(gate) * up, compute the backward
 *     gradients, write [d_gate, d_up] quantized row-wise in 128-channel groups
 *     (grad_input_q / grad_input_s) and y transposed and quantized in
 *     128-token groups (y_q_t / y_s_t);
 *   - constraints list: 128x128 tiles (both quantization axes use groups of
 *     128); forward, backward and both quantizations fused; the bf16
 *     round-trip kept before quantization; quantization by multiplication
 *     with a precomputed inverse scale.
 *
 * Definitions used (where the page is silent):
 *   x = [gate | up] along channels, bf16 [M, 2K] row-major;
 *   grad_y bf16 [M, K] row-major;
 *   y = silu(g) * u, d_gate = grad_y * u * silu'(g), d_up = grad_y * silu(g),
 *   each computed in fp32 and rounded once to bf16 (nearest even);
 *   per group: amax = max |v|; all-zero group -> scale 1, q 0; otherwise
 *   scale = amax / 127 (fp32, correctly rounded) and
 *   q = round-half-even(v * (1/scale)) in [-127, 127];
 *   a tail token group (M % 128 != 0) is quantized over the tokens it holds,
 *   and likewise, when 128 does not divide K, the last channel group of each
 *   half of [d_gate | d_up] over the K - 128 (Kg - 1) channels it holds
 *   (Kg = ceil(K/128); groups never cross from d_gate into d_up).
 *
 * Output layouts (all row-major, contiguous):
 *   grad_input_q int8 [M, 2K]             columns 0..K-1 = d_gate, K..2K-1 = d_up
 *   grad_input_s fp32 [M, 2 Kg]           column j < Kg: d_gate group j;
 *                                         column Kg + j: d_up group j
 *   y_q_t        int8 [K, M]              y transposed: y_q_t[k, m] quantizes y[m, k]
 *   y_s_t        fp32 [K, ceil(M/128)]    y_s_t[k, i]: scale of tokens 128i..128i+127
 * (for group_size 32, 64 or 256 read that size for 128 in the scale shapes;
 * the group_size argument is the page's: 32 and 64 are groups a 128 x 128
 * tile holds whole, 256 runs a kernel with 256 x 256 units.)
 *
 * Threading and ownership: the caller owns every buffer.  The device entry
 * point allocates nothing, keeps no pointer after it returns, and is
 * asynchronous on the given stream (no implicit synchronization).  Calls on
 * different streams may run concurrently; concurrent calls must not share
 * output buffers.  Inputs and outputs must not overlap.
 *
 * Stream order: the op's kernel is launched with programmatic stream
 * serialization, so its blocks may start while the kernel before it on the
 * stream is finishing; they read and write the arrays only after that
 * kernel has completed.  Before that point a block only prefetches the first
 * input tiles it will read into L2, which changes no value it reads.
 *
 * Per-device state: the library sets up, once per device and process, the
 * kernels' attributes, the copy streams and events of sdq_fuse_host, and
 * the device address of sdq_fuse_host_noalloc's array.  All of it belongs
 * to the device's primary context: after cudaDeviceReset (or anything else
 * that destroys that context) the library must not be called again on that
 * device in the same process.
 *
 * Errors: every entry point returns an sdq_status.  On a validation error
 * nothing is launched and nothing is written.  SDQ_ERR_CUDA means a CUDA
 * call failed; sdq_last_cuda_error() returns its cudaError_t code.
 */
#ifndef SDQ_H_
#define SDQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum sdq_status {
  SDQ_OK = 0,
  SDQ_ERR_NULL = 1,      /* a required pointer is NULL (with M > 0)                  */
  SDQ_ERR_GROUP = 2,     /* group_size not 32, 64, 128 or 256 (host-buffer entries: 128) */
  SDQ_ERR_SHAPE = 3,     /* M < 0, K < 1, K % 16 != 0, or a size above the limits    */
  SDQ_ERR_ALIGN = 4,     /* x, grad_y, grad_input_q, y_q_t not 16-byte aligned, or a
                            scale pointer not 4-byte aligned                          */
  SDQ_ERR_CUDA = 5,      /* a CUDA runtime/driver call failed (see sdq_last_cuda_error) */
  SDQ_ERR_TIMEOUT = 6,   /* a device-side wait hit its time limit (sdq_device_status) */
  SDQ_ERR_WORKSPACE = 7, /* the workspace given to sdq_fuse_host is too small        */
  SDQ_ERR_TOO_LARGE = 8, /* sdq_fuse_host_noalloc: K too large for its fixed scratch  */
  SDQ_ERR_FORMAT = 9,    /* sdq_fuse_format: unknown bits in `format`                */
  SDQ_ERR_STRIDE = 10    /* sdq_fuse_strided: a leading dimension below its row length
                            or above SDQ_MAX_LD                                      */
} sdq_status;

/* Largest accepted sizes: M < 2^31 (tensor-map coordinates are 32-bit) and
 * K <= 2^20 channels. */
#define SDQ_GROUP_SIZE 128
#define SDQ_MAX_M 2147483647LL
#define SDQ_MAX_K 1048576LL
#define SDQ_K_MULTIPLE 16      /* K must be a multiple of this (16-byte code rows)   */
#define SDQ_MAX_LD (1LL << 36) /* largest leading dimension (tensor-map strides < 2^40 bytes) */
#define SDQ_MAX_LD_ROWS (1LL << 24) /* largest ld of grad_input_q and grad_input_s     */

/*
 * sdq_fuse -- the op on device buffers.
 *   x             device, bf16 [M, 2K], 16-byte aligned
 *   grad_y        device, bf16 [M, K], 16-byte aligned
 *   grad_input_q  device, int8 [M, 2K], 16-byte aligned      (written)
 *   grad_input_s  device, fp32 [M, 2 ceil(K/128)], 4-byte aligned (written)
 *   y_q_t         device, int8 [K, M], 16-byte aligned       (written)
 *   y_s_t         device, fp32 [K, ceil(M/128)], 4-byte aligned (written)
 *   M             tokens (rows of x), 0 <= M <= SDQ_MAX_M; M == 0 is a no-op
 *   K             channels of gate/up, a positive multiple of SDQ_K_MULTIPLE
 *                 (16), <= SDQ_MAX_K
 *   group_size    128 (the page's), or 32, 64 or 256: tokens per column group
 *                 and channels per row group; grad_input_s is then
 *                 [M, 2 ceil(K/group_size)] (d_up groups from column
 *                 ceil(K/group_size) on) and y_s_t [K, ceil(M/group_size)]
 *   stream        a cudaStream_t (NULL = the legacy default stream)
 * Launches one persistent kernel on the current device.  Returns SDQ_OK once
 * the launch is enqueued.
 */
int sdq_fuse(const void* x, const void* grad_y, int8_t* grad_input_q,
             float* grad_input_s, int8_t* y_q_t, float* y_s_t, int64_t M,
             int64_t K, int32_t group_size, void* stream);

/*
 * sdq_validate -- the argument checks of sdq_fuse alone: no CUDA call, no
 * launch.  Returns the status sdq_fuse would return before launching.
 */
int sdq_validate(const void* x, const void* grad_y, const int8_t* grad_input_q,
                 const float* grad_input_s, const int8_t* y_q_t,
                 const float* y_s_t, int64_t M, int64_t K, int32_t group_size);

/*
 * Output formats of sdq_fuse_format, OR-ed together (0 = the page's: INT8
 * codes, fp32 scales, y_s_t [K, ceil(M/128)]).  The page says only that the
 * outputs feed quantized GEMMs; these variants give the layouts such GEMMs
 * take, each following a public definition:
 *   SDQ_FMT_E4M3     codes are OCP FP8 E4M3 bytes (sign, 4 exponent bits with
 *                    bias 7, 3 mantissa bits, no infinities, largest finite
 *                    448) in place of INT8: scale = fl32(amax / 448), code =
 *                    E4M3 round-to-nearest-even of v * (1/scale), saturated
 *                    to +-448.  Same shapes; one byte per code.
 *   SDQ_FMT_E8M0     scales are OCP Microscaling E8M0 bytes (value 2^(e-127))
 *                    in place of fp32: the smallest power of two not below
 *                    fl32(amax / Qmax) (Qmax = 127 for INT8, 448 for E4M3),
 *                    clamped to [2^-127, 2^127]; an all-zero group gets 2^0
 *                    (byte 127).  The scale arrays hold one byte per scale
 *                    (any alignment); every element stays inside the code
 *                    range, and the codes are v * 2^-e exactly rounded.
 *   SDQ_FMT_YS_MG_K  y_s_t is [ceil(M/128), K] (y_s_t[i, k] = scale of tokens
 *                    128i.. of channel k) instead of [K, ceil(M/128)].
 * In every format an all-zero group has scale 1 and the code of v / 1 (an
 * E4M3 -0.0 element keeps its sign: 0x80).
 */
#define SDQ_FMT_E4M3 1u
#define SDQ_FMT_E8M0 2u
#define SDQ_FMT_YS_MG_K 4u

/*
 * sdq_fuse_format -- sdq_fuse with a chosen output format.  The code arrays
 * are bytes (int8 or E4M3 bits); the scale arrays are fp32 (4-byte aligned)
 * or E8M0 bytes; all other arguments, the alignment of x, grad_y and the
 * code arrays, and the errors are those of sdq_fuse.  SDQ_ERR_FORMAT for
 * unknown bits.  format = 0 is exactly sdq_fuse.
 */
int sdq_fuse_format(const void* x, const void* grad_y, void* grad_input_q,
                    void* grad_input_s, void* y_q_t, void* y_s_t, int64_t M,
                    int64_t K, int32_t group_size, uint32_t format, void* stream);

/* The argument checks of sdq_fuse_format alone: no CUDA call, no launch. */
int sdq_validate_format(const void* x, const void* grad_y, const void* grad_input_q,
                        const void* grad_input_s, const void* y_q_t,
                        const void* y_s_t, int64_t M, int64_t K,
                        int32_t group_size, uint32_t format);

/*
 * sdq_fuse_strided -- sdq_fuse_format on arrays with their own row strides:
 * each array is row-major with `ld_*` ELEMENTS from the start of one row to
 * the next (at least the row length; up to SDQ_MAX_LD), and gate and up are
 * separate [M, K] arrays.  The page's x = [gate | up] is gate = x,
 * up = x + K (elements), ld_gate = ld_up = 2K; a slice of a wider buffer,
 * padded rows, or gate and up held apart are all the same call.
 *   gate, up, grad_y   device, bf16 [M, K] each; 16-byte aligned; ld a
 *                      multiple of 8 (rows start on 16 bytes)
 *   grad_input_q       [M, 2K] codes; 16-byte aligned; ld a multiple of 16,
 *                      at most SDQ_MAX_LD_ROWS
 *   grad_input_s       [M, 2 ceil(K/group_size)] scales; that many <= ld <=
 *                      SDQ_MAX_LD_ROWS
 *   y_q_t              [K, M] codes; 16-byte aligned; any ld >= M (a multiple
 *                      of 16 takes 16-byte stores, others byte stores)
 *   y_s_t              [K, ceil(M/group_size)] (or [ceil(M/group_size), K]
 *                      with SDQ_FMT_YS_MG_K) scales
 *   y                  optional (NULL: not written, ld_y ignored): the
 *                      recomputed y itself, bf16 [M, K], the very values
 *                      y_q_t quantizes (e.g. for an fp32-accumulated check of
 *                      the GEMM that consumes y_q_t); 16-byte aligned, ld a
 *                      multiple of 8, K <= ld <= SDQ_MAX_LD.  The page
 *                      ("outputs" section) lists no such output; it serves
 *                      the step after the op.
 *   M, K, group_size, format, stream: as sdq_fuse_format.
 * Inputs may overlap each other (gate and up often do: two halves of one
 * buffer); outputs must not overlap inputs or each other.  SDQ_ERR_STRIDE
 * for a leading dimension out of range, SDQ_ERR_ALIGN for a misaligned one.
 */
int sdq_fuse_strided(const void* gate, int64_t ld_gate, const void* up, int64_t ld_up,
                     const void* grad_y, int64_t ld_grad_y, void* grad_input_q,
                     int64_t ld_grad_input_q, void* grad_input_s, int64_t ld_grad_input_s,
                     void* y_q_t, int64_t ld_y_q_t, void* y_s_t, int64_t ld_y_s_t,
                     void* y, int64_t ld_y, int64_t M, int64_t K, int32_t group_size,
                     uint32_t format, void* stream);

/* The argument checks of sdq_fuse_strided alone: no CUDA call, no launch. */
int sdq_validate_strided(const void* gate, int64_t ld_gate, const void* up, int64_t ld_up,
                         const void* grad_y, int64_t ld_grad_y, const void* grad_input_q,
                         int64_t ld_grad_input_q, const void* grad_input_s,
                         int64_t ld_grad_input_s, const void* y_q_t, int64_t ld_y_q_t,
                         const void* y_s_t, int64_t ld_y_s_t, const void* y, int64_t ld_y,
                         int64_t M, int64_t K, int32_t group_size, uint32_t format);

/*
 * sdq_fuse_int8_grad_y -- sdq_fuse_strided with grad_y handed over already
 * quantized, as the step after the op in a chained INT8 backward would hand
 * it over: in the row-group format this op writes for grad_input.  The page
 * ("entry point" section) takes grad_y in bf16; this entry reads
 *   grad_y_q   device, INT8 codes [M, K]; 16-byte aligned; ld a multiple of
 *              16 (rows start on 16 bytes), K <= ld <= SDQ_MAX_LD
 *   grad_y_s   device, fp32 scales [M, ceil(K/128)], one per token and 128
 *              consecutive channels (the last one of a row over what is
 *              left); 4-byte aligned; ceil(K/128) <= ld <= SDQ_MAX_LD
 * and takes grad_y[m, k] = grad_y_q[m, k] * grad_y_s[m, k / 128], each
 * product rounded once to fp32; everything else (the optional y included)
 * as sdq_fuse_strided.  Statuses as sdq_fuse_strided, plus SDQ_ERR_NULL for a
 * NULL grad_y_s.
 */
int sdq_fuse_int8_grad_y(const void* gate, int64_t ld_gate, const void* up, int64_t ld_up,
                         const void* grad_y_q, int64_t ld_grad_y_q, const float* grad_y_s,
                         int64_t ld_grad_y_s, void* grad_input_q, int64_t ld_grad_input_q,
                         void* grad_input_s, int64_t ld_grad_input_s, void* y_q_t,
                         int64_t ld_y_q_t, void* y_s_t, int64_t ld_y_s_t, void* y, int64_t ld_y,
                         int64_t M, int64_t K, int32_t group_size, uint32_t format, void* stream);

/* The argument checks of sdq_fuse_int8_grad_y alone: no CUDA call, no launch. */
int sdq_validate_int8_grad_y(const void* gate, int64_t ld_gate, const void* up, int64_t ld_up,
                             const void* grad_y_q, int64_t ld_grad_y_q, const float* grad_y_s,
                             int64_t ld_grad_y_s, const void* grad_input_q,
                             int64_t ld_grad_input_q, const void* grad_input_s,
                             int64_t ld_grad_input_s, const void* y_q_t, int64_t ld_y_q_t,
                             const void* y_s_t, int64_t ld_y_s_t, const void* y, int64_t ld_y,
                             int64_t M, int64_t K, int32_t group_size, uint32_t format);

/*
 * sdq_swiglu_q8_1 -- the forward-side neighbour of the backward op: the
 * SwiGLU forward and the q8_1 row quantization of its output in one pass.
 * Source: the launcher kquant_swiglu_q8_1_rows on the page with the K-quant
 * kernels ("h[rows, inter] = bf16(swiglu(gate, up) * w[row]), then the q8_1
 * blocks of those bf16 rows"; "block_q8_1: 32 int8 + half2 (d, sum)", 36
 * bytes; inter a multiple of 32).  Definitions where that page is silent:
 *   h[m, k] = bf16(silu(g) * u * w[m]), computed in fp32, rounded once to
 *   bf16 (nearest even); with limit > 0, g = min(gate, limit) and
 *   u = clamp(up, -limit, limit) first (limit <= 0 or NaN: no clamp);
 *   per block of 32 consecutive h of a row: d32 = fl32(amax / 127),
 *   q = round-half-even(h * (1/d32)) in [-127, 127], d = fp16(d32),
 *   sum = fp16(d32 * sum(q)); an all-zero block is all zero; a block is
 *   half2 (d, sum) first (d in the low half), then the 32 codes.
 *   gate, up   device, bf16 [rows, inter], 16-byte aligned, ld a multiple of 8
 *   w          device, fp32 [rows] (a per-row weight, e.g. a router
 *              weight), 4-byte aligned; NULL = 1
 *   h          device, bf16 [rows, inter], 16-byte aligned, ld a multiple of 8
 *              (written)
 *   q8         device, [rows, inter/32] blocks of 36 bytes, contiguous,
 *              4-byte aligned (written)
 *   rows       0 <= rows <= SDQ_MAX_M (0: no-op); inter: a multiple of 32,
 *              32 <= inter <= SDQ_MAX_K; ld_* in elements, >= inter
 * One streaming kernel on `stream`; allocates nothing.  Errors as sdq_fuse
 * (SDQ_ERR_SHAPE, SDQ_ERR_NULL, SDQ_ERR_STRIDE, SDQ_ERR_ALIGN, SDQ_ERR_CUDA).
 */
int sdq_swiglu_q8_1(const void* gate, int64_t ld_gate, const void* up, int64_t ld_up,
                    const float* w, void* h, int64_t ld_h, void* q8, int64_t rows,
                    int64_t inter, float limit, void* stream);

/* The argument checks of sdq_swiglu_q8_1 alone: no CUDA call, no launch. */
int sdq_validate_swiglu_q8_1(const void* gate, int64_t ld_gate, const void* up, int64_t ld_up,
                             const float* w, const void* h, int64_t ld_h, const void* q8,
                             int64_t rows, int64_t inter);

/*
 * sdq_fuse_host -- the op on HOST buffers (same shapes and layouts as
 * sdq_fuse; page-locked host memory gives overlapped copies, pageable memory
 * works but copies synchronously).  The rows are processed in chunks through
 * a caller-provided device workspace: host->device copy of a chunk of x and
 * grad_y, the kernel, device->host copy of the chunk's four outputs, with the
 * copies of one chunk overlapping the kernel of another.  Enqueued on
 * `stream`; the host outputs are complete once `stream` has been
 * synchronized.
 *   workspace        device memory, 256-byte aligned, owned by the caller
 *   workspace_bytes  at least sdq_fuse_host_workspace_bytes(M, K, chunk_rows)
 *   chunk_rows       rows per chunk, a multiple of 128 (0 = choose)
 */
int sdq_fuse_host(const void* x, const void* grad_y, int8_t* grad_input_q,
                  float* grad_input_s, int8_t* y_q_t, float* y_s_t, int64_t M,
                  int64_t K, int32_t group_size, void* workspace,
                  size_t workspace_bytes, int64_t chunk_rows, void* stream);

/* Device workspace sdq_fuse_host needs for this shape and chunk size
 * (chunk_rows = 0: the size it would choose).  0 for invalid arguments. */
size_t sdq_fuse_host_workspace_bytes(int64_t M, int64_t K, int64_t chunk_rows);

/*
 * sdq_fuse_host_noalloc -- sdq_fuse_host for callers that cannot allocate
 * device memory.  (The page has no counterpart: this entry exists for
 * callers of this library, not for the method.)
 *
 * Who needs it: code that holds no device allocator of its own or must not
 * call one -- a plain C/C++ host program that only has host buffers, a
 * plugin inside a framework whose caching allocator owns all device memory
 * (a cudaMalloc behind its back can fail or fragment the pool), or a service
 * that forbids device allocation after start-up.  Such a caller cannot
 * provide the workspace that sdq_fuse_host asks for.
 *
 * Same arguments, shapes, layouts and results as sdq_fuse_host, minus the
 * workspace.  The staging buffers live in one fixed device array of
 * SDQ_NOALLOC_SCRATCH_BYTES inside this library (every GPU that loads the
 * library holds it until the process exits).  The rows go through it in
 * chunks of a multiple of 128 rows, as many as fit; host->device copy,
 * kernel and device->host copy of each chunk are queued on `stream` alone.
 * The call allocates nothing: no cudaMalloc/cudaFree, no stream or event
 * creation.
 *   - Limit: a 128-row chunk must fit, i.e. K <= SDQ_NOALLOC_MAX_K; larger K
 *     returns SDQ_ERR_TOO_LARGE before any CUDA call.  M is unlimited.
 *   - Set-up: the first call on each device looks up the array's device
 *     address (cudaGetSymbolAddress) with that device current; make that
 *     first call before any stream capture.  A failed lookup returns
 *     SDQ_ERR_CUDA and is tried again by the next call.
 *   - Host buffers: page-locked (cudaHostAlloc / cudaHostRegister) for the
 *     copies to run asynchronously.  Pageable buffers give the same results,
 *     but the CUDA runtime then copies through its own staging memory and
 *     the device->host copies return only once they are done, so the call
 *     blocks the host until the last chunk's kernel has run.
 *   - Sharing: all calls on a device share the one array, and it keeps the
 *     last call's contents (every byte a call reads is written by that same
 *     call first, so nothing needs clearing).  Calls that overlap on the GPU
 *     (on different streams, or from different threads) race on the array:
 *     serialize them.
 *   - Host outputs are complete once `stream` has been synchronized.
 */
#define SDQ_NOALLOC_SCRATCH_BYTES (32u << 20)
#define SDQ_NOALLOC_MAX_K 28800LL
int sdq_fuse_host_noalloc(const void* x, const void* grad_y, int8_t* grad_input_q,
                          float* grad_input_s, int8_t* y_q_t, float* y_s_t, int64_t M,
                          int64_t K, int32_t group_size, void* stream);

/*
 * sdq_fuse_test_stall -- test hook for the failure path, not for production
 * use: sdq_fuse with the kernel's first shared-memory load withheld, so every
 * CTA's first wait on its pipeline runs out after `wait_limit_ns`
 * (1 us .. 1 s; outside that, SDQ_ERR_SHAPE).  The kernel then stops early,
 * leaving its outputs incomplete, and the next sdq_device_status returns
 * SDQ_ERR_TIMEOUT.  Nothing faults or hangs: every wait in the kernel is
 * bounded, and the CUDA context stays usable for the next call.  (The page
 * has no counterpart: it exists to test this library's failure detection.)
 */
int sdq_fuse_test_stall(const void* x, const void* grad_y, int8_t* grad_input_q,
                        float* grad_input_s, int8_t* y_q_t, float* y_s_t, int64_t M,
                        int64_t K, int32_t group_size, int64_t wait_limit_ns, void* stream);

/*
 * sdq_device_status -- synchronizes `stream`, then reads and clears the
 * device-side status word of the current device: SDQ_OK, or
 * SDQ_ERR_TIMEOUT if a kernel's wait on its shared-memory pipeline ran past
 * its limit (the kernel then stops early and its outputs are incomplete).
 */
int sdq_device_status(void* stream);

/* Human-readable name of a status code (static storage). */
const char* sdq_status_string(int status);

/* cudaError_t of the last CUDA failure seen by this thread (0 if none). */
int sdq_last_cuda_error(void);

/* Library version, e.g. "0.1.0". */
const char* sdq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SDQ_H_ */

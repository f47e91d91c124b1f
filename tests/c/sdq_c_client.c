/*
 * A plain C99 client of the library's C ABI (include/sdq.h): it shows that
 * the header compiles as C and that the entry points link and run with no
 * C++ or Python in between.
 *
 *   sdq_c_client cpu
 *       version, status strings and argument checks only (no GPU needed);
 *   sdq_c_client gpu DIR M K
 *       reads DIR/x.bin (bf16 [M, 2K]) and DIR/grad_y.bin (bf16 [M, K]),
 *       runs sdq_fuse on device buffers it allocates itself with the CUDA
 *       runtime, and writes DIR/grad_input_q.bin, grad_input_s.bin,
 *       y_q_t.bin, y_s_t.bin; then runs sdq_fuse_host on the same host
 *       arrays and checks that it gives the same bytes.
 * Exit status 0 on success; a message on stderr otherwise.
 */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "sdq.h"

#ifdef SDQ_C_CLIENT_GPU
#include <cuda_runtime_api.h>
#endif

static int fail(const char* what) {
  fprintf(stderr, "sdq_c_client: %s\n", what);
  return 1;
}

static int cpu_checks(void) {
  const uintptr_t a = (uintptr_t)1 << 20; /* aligned fake addresses: only validated */
  const void* p = (const void*)a;
  int s;
  if (strcmp(sdq_version(), "0.1.0") != 0) return fail("version");
  for (s = 0; s <= 10; ++s)
    if (!sdq_status_string(s) || !*sdq_status_string(s)) return fail("status string");
  if (sdq_validate(p, p, (const int8_t*)p, (const float*)p, (const int8_t*)p, (const float*)p, 256,
                   256, 128) != SDQ_OK)
    return fail("validate: good arguments");
  if (sdq_validate(p, p, (const int8_t*)p, (const float*)p, (const int8_t*)p, (const float*)p, 256,
                   100, 128) != SDQ_ERR_SHAPE)
    return fail("validate: K % 128");
  if (sdq_validate(p, p, (const int8_t*)p, (const float*)p, (const int8_t*)p, (const float*)p, 256,
                   256, 96) != SDQ_ERR_GROUP)
    return fail("validate: group size");
  if (sdq_validate(NULL, p, (const int8_t*)p, (const float*)p, (const int8_t*)p, (const float*)p,
                   256, 256, 128) != SDQ_ERR_NULL)
    return fail("validate: NULL x");
  if (sdq_validate((const char*)p + 8, p, (const int8_t*)p, (const float*)p, (const int8_t*)p,
                   (const float*)p, 256, 256, 128) != SDQ_ERR_ALIGN)
    return fail("validate: misaligned x");
  if (sdq_fuse_host_workspace_bytes(4096, 1408, 0) == 0) return fail("workspace size");
  return 0;
}

#ifdef SDQ_C_CLIENT_GPU
static void* read_file(const char* dir, const char* name, size_t bytes) {
  char path[4096];
  FILE* f;
  void* buf = malloc(bytes ? bytes : 1);
  snprintf(path, sizeof path, "%s/%s", dir, name);
  f = fopen(path, "rb");
  if (!f || !buf || fread(buf, 1, bytes, f) != bytes) {
    if (f) fclose(f);
    free(buf);
    return NULL;
  }
  fclose(f);
  return buf;
}

static int write_file(const char* dir, const char* name, const void* buf, size_t bytes) {
  char path[4096];
  FILE* f;
  snprintf(path, sizeof path, "%s/%s", dir, name);
  f = fopen(path, "wb");
  if (!f) return 1;
  if (fwrite(buf, 1, bytes, f) != bytes) {
    fclose(f);
    return 1;
  }
  return fclose(f) != 0;
}

static int gpu_run(const char* dir, int64_t M, int64_t K) {
  const int64_t Kg = K / 128, Mg = (M + 127) / 128;
  const size_t bx = (size_t)M * 2 * K * 2, bgy = (size_t)M * K * 2;
  const size_t sizes[4] = {(size_t)M * 2 * K, (size_t)M * 2 * Kg * 4, (size_t)K * M, (size_t)K * Mg * 4};
  const char* names[4] = {"grad_input_q.bin", "grad_input_s.bin", "y_q_t.bin", "y_s_t.bin"};
  void *xh = read_file(dir, "x.bin", bx), *gh = read_file(dir, "grad_y.bin", bgy);
  void *xd = NULL, *gd = NULL, *od[4] = {NULL, NULL, NULL, NULL}, *oh[4], *oh2[4], *ws = NULL;
  size_t wsb;
  int i, st;
  if (!xh || !gh) return fail("reading the inputs");
  if (cudaMalloc(&xd, bx) != cudaSuccess || cudaMalloc(&gd, bgy) != cudaSuccess) return fail("cudaMalloc");
  for (i = 0; i < 4; ++i) {
    if (cudaMalloc(&od[i], sizes[i]) != cudaSuccess) return fail("cudaMalloc");
    oh[i] = malloc(sizes[i]);
    oh2[i] = malloc(sizes[i]);
    if (!oh[i] || !oh2[i]) return fail("malloc");
  }
  if (cudaMemcpy(xd, xh, bx, cudaMemcpyHostToDevice) != cudaSuccess ||
      cudaMemcpy(gd, gh, bgy, cudaMemcpyHostToDevice) != cudaSuccess)
    return fail("cudaMemcpy to the device");
  st = sdq_fuse(xd, gd, (int8_t*)od[0], (float*)od[1], (int8_t*)od[2], (float*)od[3], M, K, 128,
                NULL);
  if (st != SDQ_OK) return fail(sdq_status_string(st));
  if (cudaDeviceSynchronize() != cudaSuccess) return fail("kernel");
  if (sdq_device_status(NULL) != SDQ_OK) return fail("device status");
  for (i = 0; i < 4; ++i) {
    if (cudaMemcpy(oh[i], od[i], sizes[i], cudaMemcpyDeviceToHost) != cudaSuccess)
      return fail("cudaMemcpy to the host");
    if (write_file(dir, names[i], oh[i], sizes[i])) return fail("writing an output");
  }
  /* the host-buffer entry point on the same (pageable) host arrays */
  wsb = sdq_fuse_host_workspace_bytes(M, K, 0);
  if (cudaMalloc(&ws, wsb) != cudaSuccess) return fail("cudaMalloc workspace");
  st = sdq_fuse_host(xh, gh, (int8_t*)oh2[0], (float*)oh2[1], (int8_t*)oh2[2], (float*)oh2[3], M,
                     K, 128, ws, wsb, 0, NULL);
  if (st != SDQ_OK) return fail(sdq_status_string(st));
  if (cudaDeviceSynchronize() != cudaSuccess) return fail("host-buffer call");
  for (i = 0; i < 4; ++i)
    if (memcmp(oh[i], oh2[i], sizes[i]) != 0) return fail("host-buffer entry differs");
  for (i = 0; i < 4; ++i) {
    cudaFree(od[i]);
    free(oh[i]);
    free(oh2[i]);
  }
  cudaFree(xd);
  cudaFree(gd);
  cudaFree(ws);
  free(xh);
  free(gh);
  return 0;
}
#endif

int main(int argc, char** argv) {
  if (argc >= 2 && strcmp(argv[1], "cpu") == 0) return cpu_checks();
#ifdef SDQ_C_CLIENT_GPU
  if (argc == 5 && strcmp(argv[1], "gpu") == 0)
    return cpu_checks() || gpu_run(argv[2], strtoll(argv[3], NULL, 10), strtoll(argv[4], NULL, 10));
#endif
  return fail("usage: sdq_c_client cpu | gpu DIR M K");
}

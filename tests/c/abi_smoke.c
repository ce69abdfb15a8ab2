/*
 * Plain C user of libhadq through include/hadq.h (no Python).
 *
 *   abi_smoke host   checks that need no GPU: version, status strings, buffer
 *                    sizes, argument validation (nothing reaches the device)
 *   abi_smoke gpu    additionally rotates rows of basis vectors on the device:
 *                    e_j . H_n / sqrt(n) is row j of H_n / sqrt(n), whose
 *                    entries are (-1)^popcount(i & j) / sqrt(n); then
 *                    quantizes the same rows to int4 g128, where every group
 *                    has absmax 1/sqrt(n), so every code is +/-7
 *
 * Exit status 0 on success; the first failed check is printed.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime.h>

#include "hadq.h"

static int fails = 0;
#define CHECK(cond, ...)                               \
  do {                                                 \
    if (!(cond)) {                                     \
      fprintf(stderr, "FAILED %s:%d: ", __FILE__, __LINE__); \
      fprintf(stderr, __VA_ARGS__);                    \
      fprintf(stderr, "\n");                           \
      fails++;                                         \
      return 1;                                        \
    }                                                  \
  } while (0)

static int host_checks(void) {
  CHECK(hadq_version() == 200, "version %d", hadq_version());
  CHECK(hadq_get_impl() == HADQ_IMPL_AUTO, "impl %d", (int)hadq_get_impl());
  CHECK(hadq_set_impl((hadq_impl)9) == HADQ_ERR_INVALID_ARG, "bad impl accepted");
  CHECK(strcmp(hadq_status_string(HADQ_OK), "ok") == 0, "status string");
  CHECK(hadq_codes_bytes(4, 1024, HADQ_INT4_SYM) == 2048, "int4 code bytes");
  CHECK(hadq_scales_bytes(4, 1024, HADQ_INT4_SYM, 128) == 64, "int4 scale bytes");
  CHECK(hadq_scales_bytes(4, 1024, HADQ_NVFP4, 16) == 256, "nvfp4 scale bytes");
  /* validation happens on the host before any CUDA call */
  void* fake = (void*)(uintptr_t)0x100000;
  hadq_status st = hadq_rotate_quant(fake, HADQ_BF16, 4, 1024, 0, HADQ_INT4_SYM, 48, fake, fake, NULL);
  CHECK(st == HADQ_ERR_INVALID_ARG, "group 48 gave status %d", (int)st);
  CHECK(strlen(hadq_last_error()) > 0, "no error message");
  st = hadq_rotate(NULL, HADQ_F32, 0, 64, 0, NULL, HADQ_F32, NULL);
  CHECK(st == HADQ_OK, "empty call gave status %d", (int)st);
  st = hadq_rotate(fake, HADQ_F32, 4, 1000, 0, fake, HADQ_F32, NULL);
  CHECK(st == HADQ_ERR_INVALID_ARG, "non-power-of-2 full rotation gave status %d", (int)st);
  return 0;
}

static int popcount_parity(unsigned v) {
  int p = 0;
  while (v) { p ^= 1; v &= v - 1; }
  return p;
}

static int gpu_checks(void) {
  const int64_t rows = 8, n = 1024;
  float* xh = (float*)calloc((size_t)(rows * n), sizeof(float));
  float* yh = (float*)malloc((size_t)(rows * n) * sizeof(float));
  uint8_t* ch = (uint8_t*)malloc((size_t)(rows * n / 2));
  uint16_t* sh = (uint16_t*)malloc((size_t)(rows * n / 128) * 2);
  for (int64_t r = 0; r < rows; ++r) xh[r * n + 37 * r + 5] = 1.0f;   /* row r = e_j, j = 37 r + 5 */
  float *x = NULL, *y = NULL;
  void *codes = NULL, *scales = NULL;
  CHECK(cudaMalloc((void**)&x, rows * n * 4) == cudaSuccess, "cudaMalloc");
  CHECK(cudaMalloc((void**)&y, rows * n * 4) == cudaSuccess, "cudaMalloc");
  CHECK(cudaMalloc(&codes, rows * n / 2) == cudaSuccess, "cudaMalloc");
  CHECK(cudaMalloc(&scales, rows * n / 128 * 2) == cudaSuccess, "cudaMalloc");
  CHECK(cudaMemcpy(x, xh, rows * n * 4, cudaMemcpyHostToDevice) == cudaSuccess, "copy in");
  hadq_status st = hadq_rotate(x, HADQ_F32, rows, n, 0, y, HADQ_F32, NULL);
  CHECK(st == HADQ_OK, "hadq_rotate: %s", hadq_last_error());
  st = hadq_rotate_quant(x, HADQ_F32, rows, n, 0, HADQ_INT4_SYM, 128, codes, scales, NULL);
  CHECK(st == HADQ_OK, "hadq_rotate_quant: %s", hadq_last_error());
  CHECK(cudaDeviceSynchronize() == cudaSuccess, "sync");
  CHECK(cudaMemcpy(yh, y, rows * n * 4, cudaMemcpyDeviceToHost) == cudaSuccess, "copy out");
  CHECK(cudaMemcpy(ch, codes, rows * n / 2, cudaMemcpyDeviceToHost) == cudaSuccess, "copy out");
  const double inv = 1.0 / sqrt((double)n);
  for (int64_t r = 0; r < rows; ++r) {
    const unsigned j = (unsigned)(37 * r + 5);
    for (int64_t i = 0; i < n; ++i) {
      const double want = (popcount_parity((unsigned)i & j) ? -inv : inv);
      CHECK(fabs(yh[r * n + i] - want) < 1e-6, "row %lld element %lld: %g vs %g", (long long)r, (long long)i,
            yh[r * n + i], want);
      const int nib = (ch[(r * n + i) / 2] >> (4 * (i & 1))) & 15;
      const int code = nib >= 8 ? nib - 16 : nib;
      CHECK(code == (want > 0 ? 7 : -7), "code %d at row %lld element %lld", code, (long long)r, (long long)i);
    }
  }
  cudaFree(x); cudaFree(y); cudaFree(codes); cudaFree(scales);
  free(xh); free(yh); free(ch); free(sh);
  return 0;
}

int main(int argc, char** argv) {
  if (host_checks()) return 1;
  if (argc > 1 && strcmp(argv[1], "gpu") == 0 && gpu_checks()) return 1;
  printf("abi_smoke ok (%s)\n", argc > 1 ? argv[1] : "host");
  return fails != 0;
}

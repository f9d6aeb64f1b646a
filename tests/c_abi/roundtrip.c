/* roundtrip.c -- libnvfp4 used from plain C through its C ABI (include/nvfp4.h): device buffers from
 * the CUDA runtime, a ScaleSearch quantize, a dequantize and a Hadamard-16 rotation on the default
 * stream, every output byte compared with the CPU oracle (test infrastructure, linked only here), and
 * the synchronous argument errors.  Prints "ok" and exits 0 on success. */
#include <cuda_runtime.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "nvfp4.h"
#include "nvfp4_ref.h"
#include "seeded.h"

#define CHECK_CUDA(call)                                                         \
  do {                                                                           \
    cudaError_t e_ = (call);                                                     \
    if (e_ != cudaSuccess) {                                                     \
      printf("CUDA error %s at line %d\n", cudaGetErrorString(e_), __LINE__);   \
      return 1;                                                                  \
    }                                                                            \
  } while (0)

#define CHECK_NV(call)                                                                   \
  do {                                                                                   \
    int s_ = (call);                                                                     \
    if (s_ != NVFP4_OK) {                                                                \
      printf("libnvfp4 status %d (%s) at line %d\n", s_, nvfp4_status_str(s_), __LINE__); \
      return 1;                                                                          \
    }                                                                                    \
  } while (0)

static int same_bytes(const void* a, const void* b, size_t n, const char* what) {
  if (memcmp(a, b, n) != 0) {
    const unsigned char *p = a, *q = b;
    size_t i = 0;
    while (p[i] == q[i]) ++i;
    printf("%s differs first at byte %zu (%u vs %u)\n", what, i, p[i], q[i]);
    return 0;
  }
  return 1;
}

int main(void) {
  /* 50 001 blocks: many CTA rounds and a partial last one; an all-zero block and outlier blocks */
  const int64_t nb = 50001, n = 16 * nb;
  float* x = malloc(n * sizeof(float));
  seeded_rng rng = {0x243F6A8885A308D3ull};
  for (int64_t i = 0; i < n; ++i) x[i] = seeded_normal(&rng);
  for (int64_t i = 0; i < n; i += 997) x[i] *= 16.0f;
  for (int i = 0; i < 16; ++i) x[16 * 1234 + i] = 0.0f;

  float *dx, *dg, *dout, *drot;
  uint8_t *dcodes, *dscales;
  CHECK_CUDA(cudaMalloc((void**)&dx, n * sizeof(float)));
  CHECK_CUDA(cudaMalloc((void**)&dout, n * sizeof(float)));
  CHECK_CUDA(cudaMalloc((void**)&drot, n * sizeof(float)));
  CHECK_CUDA(cudaMalloc((void**)&dg, sizeof(float)));
  CHECK_CUDA(cudaMalloc((void**)&dcodes, n / 2));
  CHECK_CUDA(cudaMalloc((void**)&dscales, nb));
  CHECK_CUDA(cudaMemcpy(dx, x, n * sizeof(float), cudaMemcpyHostToDevice));

  CHECK_NV(nvfp4_quantize(dx, n, NVFP4_F32, 16, -2, 6, dcodes, dscales, dg, NULL));
  CHECK_NV(nvfp4_dequantize(dcodes, dscales, dg, n, NVFP4_F32, dout, NULL));
  CHECK_NV(nvfp4_hadamard16(dx, n, NVFP4_F32, drot, NVFP4_F32, NULL));
  CHECK_CUDA(cudaDeviceSynchronize());

  uint8_t* codes = malloc(n / 2);
  uint8_t* scales = malloc(nb);
  float* out = malloc(n * sizeof(float));
  float* rot = malloc(n * sizeof(float));
  float g;
  CHECK_CUDA(cudaMemcpy(codes, dcodes, n / 2, cudaMemcpyDeviceToHost));
  CHECK_CUDA(cudaMemcpy(scales, dscales, nb, cudaMemcpyDeviceToHost));
  CHECK_CUDA(cudaMemcpy(out, dout, n * sizeof(float), cudaMemcpyDeviceToHost));
  CHECK_CUDA(cudaMemcpy(rot, drot, n * sizeof(float), cudaMemcpyDeviceToHost));
  CHECK_CUDA(cudaMemcpy(&g, dg, sizeof(float), cudaMemcpyDeviceToHost));

  uint8_t* rcodes = malloc(n / 2);
  uint8_t* rscales = malloc(nb);
  float* rout = malloc(n * sizeof(float));
  float* rrot = malloc(n * sizeof(float));
  float rg;
  if (ref_quantize(x, n, REF_F32, -2, 6, NULL, rcodes, rscales, &rg, NULL, NULL) != 0 ||
      ref_dequantize(rcodes, rscales, rg, n, REF_F32, rout) != 0 ||
      ref_hadamard16(x, n, REF_F32, rrot, REF_F32) != 0) {
    printf("oracle call failed\n");
    return 1;
  }
  int ok = same_bytes(&g, &rg, sizeof(float), "g") && same_bytes(codes, rcodes, n / 2, "codes") &&
           same_bytes(scales, rscales, nb, "scales") && same_bytes(out, rout, n * sizeof(float), "dequantize") &&
           same_bytes(rot, rrot, n * sizeof(float), "hadamard16");

  /* argument errors come back synchronously and enqueue nothing */
  ok = ok && nvfp4_quantize(dx, 20, NVFP4_F32, 16, -2, 6, dcodes, dscales, dg, NULL) == NVFP4_ERR_SIZE;
  ok = ok && nvfp4_quantize(dx, n, NVFP4_F32, 32, -2, 6, dcodes, dscales, dg, NULL) == NVFP4_ERR_ARG;
  ok = ok && nvfp4_quantize(dx, n, NVFP4_F32, 16, 6, -2, dcodes, dscales, dg, NULL) == NVFP4_ERR_ARG;
  ok = ok && nvfp4_dequantize(dcodes, dscales, NULL, n, NVFP4_F32, dout, NULL) == NVFP4_ERR_ARG;
  ok = ok && strlen(nvfp4_status_str(NVFP4_ERR_SIZE)) > 0;

  cudaFree(dx);
  cudaFree(dout);
  cudaFree(drot);
  cudaFree(dg);
  cudaFree(dcodes);
  cudaFree(dscales);
  free(x);
  free(codes);
  free(scales);
  free(out);
  free(rot);
  free(rcodes);
  free(rscales);
  free(rout);
  free(rrot);
  printf(ok ? "ok\n" : "FAILED\n");
  return ok ? 0 : 1;
}

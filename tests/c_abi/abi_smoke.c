/*
 * abi_smoke.c -- a C caller of libmoe_epilogue.so, using only the public header.
 *
 * Allocates device buffers with the CUDA runtime, calls moe_residual_add and
 * moe_swiglu_clamped_fwd on a small problem, and checks the results against
 * values computed here in plain C on exactly representable inputs:
 *   residual add: e = i, s = 0.5, r = 2  (all exact in fp32)  -> out = i + 2.5
 *   clamped SwiGLU with gate = 0: silu(0) = 0 -> y = +0 whatever up and p are
 * It also checks that a bad argument returns MOE_ERR_LIMIT without a launch.
 * Exit status 0 on success.
 */
#include <stdio.h>
#include <stdlib.h>
#include <cuda_runtime_api.h>

#include "moe_epilogue.h"

#define CHECK(x)                                                                  \
  do {                                                                            \
    int rc_ = (int)(x);                                                           \
    if (rc_ != 0) {                                                               \
      fprintf(stderr, "%s:%d: %s -> %d\n", __FILE__, __LINE__, #x, rc_);          \
      return 1;                                                                   \
    }                                                                             \
  } while (0)

int main(void) {
  const int n = 1000;
  float *e, *s, *r, *o;
  CHECK(cudaMalloc((void**)&e, n * sizeof(float)));
  CHECK(cudaMalloc((void**)&s, n * sizeof(float)));
  CHECK(cudaMalloc((void**)&r, n * sizeof(float)));
  CHECK(cudaMalloc((void**)&o, n * sizeof(float)));
  float* h = (float*)malloc(n * sizeof(float));
  for (int i = 0; i < n; ++i) h[i] = (float)i;
  CHECK(cudaMemcpy(e, h, n * sizeof(float), cudaMemcpyHostToDevice));
  for (int i = 0; i < n; ++i) h[i] = 0.5f;
  CHECK(cudaMemcpy(s, h, n * sizeof(float), cudaMemcpyHostToDevice));
  for (int i = 0; i < n; ++i) h[i] = 2.0f;
  CHECK(cudaMemcpy(r, h, n * sizeof(float), cudaMemcpyHostToDevice));
  CHECK(moe_residual_add(e, s, r, o, n, MOE_FP32, 0));
  CHECK(cudaMemcpy(h, o, n * sizeof(float), cudaMemcpyDeviceToHost));
  for (int i = 0; i < n; ++i)
    if (h[i] != (float)i + 2.5f) {
      fprintf(stderr, "residual add: element %d is %g\n", i, h[i]);
      return 1;
    }

  /* clamped SwiGLU, bf16: rows of [gate = 0 | up = 1.5] -> y = +0 */
  const int rows = 64, inter = 256;
  unsigned short *x, *y;
  float* p;
  CHECK(cudaMalloc((void**)&x, (size_t)rows * 2 * inter * 2));
  CHECK(cudaMalloc((void**)&y, (size_t)rows * inter * 2));
  CHECK(cudaMalloc((void**)&p, rows * sizeof(float)));
  unsigned short* hx = (unsigned short*)malloc((size_t)rows * 2 * inter * 2);
  for (int i = 0; i < rows; ++i)
    for (int j = 0; j < 2 * inter; ++j) hx[i * 2 * inter + j] = j < inter ? 0x0000 : 0x3FC0;
  CHECK(cudaMemcpy(x, hx, (size_t)rows * 2 * inter * 2, cudaMemcpyHostToDevice));
  for (int i = 0; i < rows; ++i) h[i] = 0.25f;
  CHECK(cudaMemcpy(p, h, rows * sizeof(float), cudaMemcpyHostToDevice));
  CHECK(cudaMemset(y, 0xFF, (size_t)rows * inter * 2));
  CHECK(moe_swiglu_clamped_fwd(x, p, y, rows, inter, 2 * inter, inter, 7.0f, MOE_BF16, 0));
  CHECK(cudaMemcpy(hx, y, (size_t)rows * inter * 2, cudaMemcpyDeviceToHost));
  for (int i = 0; i < rows * inter; ++i)
    if (hx[i] != 0x0000) {
      fprintf(stderr, "swiglu: element %d is 0x%04x\n", i, hx[i]);
      return 1;
    }
  if (moe_swiglu_clamped_fwd(x, p, y, rows, inter, 2 * inter, inter, -1.0f, MOE_BF16, 0) !=
      MOE_ERR_LIMIT) {
    fprintf(stderr, "a negative limit was not rejected\n");
    return 1;
  }
  CHECK(cudaDeviceSynchronize());
  printf("abi_smoke: ok (%s)\n", moe_status_string(MOE_OK));
  return 0;
}

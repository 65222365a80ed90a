/*
 * abi_smoke.c -- a C caller of libmoe_epilogue.so, using only the public header.
 *
 * Allocates device buffers with the CUDA runtime, calls moe_residual_add and
 * moe_swiglu_clamped_fwd on a small problem, and checks the results against
 * values computed here in plain C on exactly representable inputs:
 *   residual add: e = i, s = 0.5, r = 2  (all exact in fp32)  -> out = i + 2.5
 *   clamped SwiGLU with gate = 0: silu(0) = 0 -> y = +0 whatever up and p are
 * It also checks that a bad argument returns MOE_ERR_LIMIT without a launch, and
 * runs the rank-order reduce-scatter over three buffers from moe_symm_alloc
 * (exact integers: block q holds (q + 1) * (row * 16 + col + 1), so rank 1's
 * rows 4..7 sum to 6 * (row * 16 + col + 1)), after exporting an IPC handle.
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
  /* rank-order reduce-scatter over three library-allocated buffers */
  {
    enum { W = 3, CAP = 10, HID = 16, LOCAL = 4 };
    void* blocks[W];
    float hb[CAP * HID];
    for (int q = 0; q < W; ++q) {
      CHECK(moe_symm_alloc(CAP * HID * sizeof(float), &blocks[q]));
      for (int i = 0; i < CAP * HID; ++i) hb[i] = (float)((q + 1) * (i + 1));
      CHECK(cudaMemcpy(blocks[q], hb, sizeof(hb), cudaMemcpyHostToDevice));
    }
    unsigned char handle[MOE_IPC_HANDLE_BYTES];
    CHECK(moe_ipc_export(blocks[0], handle));
    void** table;
    int32_t *offs, *ep;
    float* out;
    const int32_t h_offs[W] = {0, 4, 8}, h_ep = CAP;
    CHECK(cudaMalloc((void**)&table, sizeof(blocks)));
    CHECK(cudaMemcpy(table, blocks, sizeof(blocks), cudaMemcpyHostToDevice));
    CHECK(cudaMalloc((void**)&offs, sizeof(h_offs)));
    CHECK(cudaMemcpy(offs, h_offs, sizeof(h_offs), cudaMemcpyHostToDevice));
    CHECK(cudaMalloc((void**)&ep, sizeof(h_ep)));
    CHECK(cudaMemcpy(ep, &h_ep, sizeof(h_ep), cudaMemcpyHostToDevice));
    CHECK(cudaMalloc((void**)&out, LOCAL * HID * sizeof(float)));
    CHECK(moe_ordered_reduce_scatter_v((const void* const*)table, 0, W, 1, offs, ep, CAP, out,
                                       LOCAL, HID, MOE_FP32, MOE_FP32, NULL, 0));
    CHECK(cudaMemcpy(hb, out, LOCAL * HID * sizeof(float), cudaMemcpyDeviceToHost));
    for (int i = 0; i < LOCAL * HID; ++i)
      if (hb[i] != (float)(6 * (4 * HID + i + 1))) {
        fprintf(stderr, "reduce-scatter: element %d is %g\n", i, hb[i]);
        return 1;
      }
    for (int q = 0; q < W; ++q) CHECK(moe_symm_free(blocks[q]));
    CHECK(cudaFree(table));
    CHECK(cudaFree(offs));
    CHECK(cudaFree(ep));
    CHECK(cudaFree(out));
  }
  CHECK(cudaDeviceSynchronize());
  printf("abi_smoke: ok (%s)\n", moe_status_string(MOE_OK));
  return 0;
}

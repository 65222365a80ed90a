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
 * rows 4..7 sum to 6 * (row * 16 + col + 1)), after exporting an IPC handle,
 * and the EP combine over two ranks' fp32 expert rows (token t of rank q's
 * expert e: inverse map entry, rows holding small integers, exact sums).
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
  /* EP combine: 2 ranks x 2 experts, 4 tokens, hidden 8, fp32.  Rank q's
     expert rows: row r holds 100 * q + 10 * r + col.  Token t uses rank 0's
     row t (expert 0) and rank 1's row 3 - t (expert 1); rank 1 owns tokens
     2..3, so out[i] = (10 * t + col) + (100 + 10 * (3 - t) + col). */
  {
    enum { W = 2, E = 2, T = 4, H = 8, ROWS = 4 };
    float hrows[ROWS * H];
    int32_t hinv[T * E];
    float* eo[W];
    int32_t* inv[W];
    for (int q = 0; q < W; ++q) {
      for (int r = 0; r < ROWS; ++r)
        for (int c = 0; c < H; ++c) hrows[r * H + c] = (float)(100 * q + 10 * r + c);
      for (int t = 0; t < T; ++t) {
        hinv[t * E + 0] = q == 0 ? t : -1;
        hinv[t * E + 1] = q == 1 ? 3 - t : -1;
      }
      CHECK(cudaMalloc((void**)&eo[q], sizeof(hrows)));
      CHECK(cudaMemcpy(eo[q], hrows, sizeof(hrows), cudaMemcpyHostToDevice));
      CHECK(cudaMalloc((void**)&inv[q], sizeof(hinv)));
      CHECK(cudaMemcpy(inv[q], hinv, sizeof(hinv), cudaMemcpyHostToDevice));
    }
    void **eo_t, **inv_t;
    int32_t *offs, *ep;
    float* out;
    const int32_t h_offs[W] = {0, 2}, h_ep = T;
    CHECK(cudaMalloc((void**)&eo_t, sizeof(eo)));
    CHECK(cudaMemcpy(eo_t, eo, sizeof(eo), cudaMemcpyHostToDevice));
    CHECK(cudaMalloc((void**)&inv_t, sizeof(inv)));
    CHECK(cudaMemcpy(inv_t, inv, sizeof(inv), cudaMemcpyHostToDevice));
    CHECK(cudaMalloc((void**)&offs, sizeof(h_offs)));
    CHECK(cudaMemcpy(offs, h_offs, sizeof(h_offs), cudaMemcpyHostToDevice));
    CHECK(cudaMalloc((void**)&ep, sizeof(h_ep)));
    CHECK(cudaMemcpy(ep, &h_ep, sizeof(h_ep), cudaMemcpyHostToDevice));
    CHECK(cudaMalloc((void**)&out, 2 * H * sizeof(float)));
    CHECK(moe_unpermute_reduce_scatter((const void* const*)eo_t, MOE_FP32, ROWS,
                                       (const int32_t* const*)inv_t, E, T, ep, W, 1, offs,
                                       MOE_FP32, out, MOE_FP32, 2, H, NULL, 0));
    float ho[2 * H];
    CHECK(cudaMemcpy(ho, out, sizeof(ho), cudaMemcpyDeviceToHost));
    for (int i = 0; i < 2 * H; ++i) {
      const int t = 2 + i / H, c = i % H;
      const float want = (float)((10 * t + c) + (100 + 10 * (3 - t) + c));
      if (ho[i] != want) {
        fprintf(stderr, "EP combine: element %d is %g, want %g\n", i, ho[i], want);
        return 1;
      }
    }
    for (int q = 0; q < W; ++q) {
      CHECK(cudaFree(eo[q]));
      CHECK(cudaFree(inv[q]));
    }
    CHECK(cudaFree(eo_t));
    CHECK(cudaFree(inv_t));
    CHECK(cudaFree(offs));
    CHECK(cudaFree(ep));
    CHECK(cudaFree(out));
  }
  CHECK(cudaDeviceSynchronize());
  printf("abi_smoke: ok (%s)\n", moe_status_string(MOE_OK));
  return 0;
}

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
 * The other hot-path entry points run on inputs whose results are exact too:
 *   clamped SwiGLU backward with gate = 0, up = 1.5, dy = 1, p = 0.25:
 *     d_gate = dy * p * up * silu'(0) = 0.1875, d_up = dy * p * silu(0) = +0,
 *     grad_probs = sum_j dy * silu(0) * up = +0;
 *   router-weight multiply with small integers and p = 0.5 / 0.25 (products
 *     and row sums exact in fp32, and in bf16 where stored);
 *   squared ReLU with probabilities over a padded map (integers -2..3: squares
 *     0, 1, 4, 9; times 0.5), padding rows zeroed, rows past n_used untouched;
 *   fixed-order unpermute of small-integer rows into fp32 (exact sums), one
 *     token past valid_tokens untouched.
 * Exit status 0 on success.
 */
#include <stdio.h>
#include <stdlib.h>
#include <string.h>
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

/* bf16 bits of a float that bf16 represents exactly, and back */
static unsigned short bf16_of(float f) {
  unsigned int u;
  memcpy(&u, &f, 4);
  return (unsigned short)(u >> 16);
}
static float of_bf16(unsigned short b) {
  unsigned int u = (unsigned int)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

static int check_bf16(const char* what, const unsigned short* got, const float* want, int n) {
  for (int i = 0; i < n; ++i)
    if (got[i] != bf16_of(want[i])) {
      fprintf(stderr, "%s: element %d is 0x%04x (%g), want %g\n", what, i, got[i],
              of_bf16(got[i]), want[i]);
      return 1;
    }
  return 0;
}

/* clamped SwiGLU backward, bf16, rows of [gate = 0 | up = 1.5], dy = 1, p = 0.25 */
static int run_swiglu_bwd(void) {
  enum { R = 32, I = 256 };
  unsigned short *x, *gy, *gx;
  float *p, *gp;
  static unsigned short hx[R * 2 * I], hg[R * I];
  static float hp[R], want[R * 2 * I];
  for (int i = 0; i < R; ++i) {
    hp[i] = 0.25f;
    for (int j = 0; j < 2 * I; ++j) {
      hx[i * 2 * I + j] = j < I ? bf16_of(0.0f) : bf16_of(1.5f);
      want[i * 2 * I + j] = j < I ? 0.1875f : 0.0f;
    }
    for (int j = 0; j < I; ++j) hg[i * I + j] = bf16_of(1.0f);
  }
  CHECK(cudaMalloc((void**)&x, sizeof(hx)));
  CHECK(cudaMalloc((void**)&gy, sizeof(hg)));
  CHECK(cudaMalloc((void**)&gx, sizeof(hx)));
  CHECK(cudaMalloc((void**)&p, sizeof(hp)));
  CHECK(cudaMalloc((void**)&gp, sizeof(hp)));
  CHECK(cudaMemcpy(x, hx, sizeof(hx), cudaMemcpyHostToDevice));
  CHECK(cudaMemcpy(gy, hg, sizeof(hg), cudaMemcpyHostToDevice));
  CHECK(cudaMemcpy(p, hp, sizeof(hp), cudaMemcpyHostToDevice));
  CHECK(cudaMemset(gp, 0xFF, sizeof(hp)));
  CHECK(moe_swiglu_clamped_bwd(x, p, gy, gx, gp, R, I, 2 * I, I, 2 * I, 7.0f, MOE_BF16, 0));
  CHECK(cudaMemcpy(hx, gx, sizeof(hx), cudaMemcpyDeviceToHost));
  CHECK(cudaMemcpy(hp, gp, sizeof(hp), cudaMemcpyDeviceToHost));
  if (check_bf16("swiglu bwd grad_x", hx, want, R * 2 * I)) return 1;
  for (int i = 0; i < R; ++i) {
    unsigned int u;
    memcpy(&u, &hp[i], 4);
    if (u != 0u) {
      fprintf(stderr, "swiglu bwd grad_probs[%d] bits 0x%08x, want +0\n", i, u);
      return 1;
    }
  }
  CHECK(cudaFree(x));
  CHECK(cudaFree(gy));
  CHECK(cudaFree(gx));
  CHECK(cudaFree(p));
  CHECK(cudaFree(gp));
  return 0;
}

/* router-weight multiply, forward into bf16 and fp32 and backward with and
   without x, on small integers */
static int run_router_weight(void) {
  enum { R = 24, H = 136 };
  unsigned short *x, *g, *o16, *gx;
  float *p, *o32, *gp;
  static unsigned short hx[R * H], hg[R * H], h16[R * H];
  static float hp[R], h32[R * H], want[R * H], hgp[R];
  for (int i = 0; i < R * H; ++i) {
    hx[i] = bf16_of((float)(i % 7 - 3));
    hg[i] = bf16_of((float)(i % 5 - 2));
  }
  for (int r = 0; r < R; ++r) hp[r] = 0.5f;
  CHECK(cudaMalloc((void**)&x, sizeof(hx)));
  CHECK(cudaMalloc((void**)&g, sizeof(hg)));
  CHECK(cudaMalloc((void**)&o16, sizeof(h16)));
  CHECK(cudaMalloc((void**)&gx, sizeof(h16)));
  CHECK(cudaMalloc((void**)&p, sizeof(hp)));
  CHECK(cudaMalloc((void**)&o32, sizeof(h32)));
  CHECK(cudaMalloc((void**)&gp, sizeof(hgp)));
  CHECK(cudaMemcpy(x, hx, sizeof(hx), cudaMemcpyHostToDevice));
  CHECK(cudaMemcpy(g, hg, sizeof(hg), cudaMemcpyHostToDevice));
  CHECK(cudaMemcpy(p, hp, sizeof(hp), cudaMemcpyHostToDevice));
  CHECK(moe_router_weight_mul_fwd(x, MOE_BF16, p, o16, MOE_BF16, R, H, 0));
  CHECK(moe_router_weight_mul_fwd(x, MOE_BF16, p, o32, MOE_FP32, R, H, 0));
  CHECK(cudaMemcpy(h16, o16, sizeof(h16), cudaMemcpyDeviceToHost));
  CHECK(cudaMemcpy(h32, o32, sizeof(h32), cudaMemcpyDeviceToHost));
  for (int i = 0; i < R * H; ++i) want[i] = (float)(i % 7 - 3) * 0.5f;
  if (check_bf16("router weight fwd (bf16 out)", h16, want, R * H)) return 1;
  for (int i = 0; i < R * H; ++i)
    if (h32[i] != want[i]) {
      fprintf(stderr, "router weight fwd (fp32 out): element %d is %g\n", i, h32[i]);
      return 1;
    }
  /* backward: grad_x = g * 0.25; grad_probs[r] = sum_h g * x (exact integers) */
  for (int r = 0; r < R; ++r) hp[r] = 0.25f;
  CHECK(cudaMemcpy(p, hp, sizeof(hp), cudaMemcpyHostToDevice));
  CHECK(moe_router_weight_mul_bwd(g, MOE_BF16, x, MOE_BF16, p, gx, gp, R, H, 0));
  CHECK(cudaMemcpy(h16, gx, sizeof(h16), cudaMemcpyDeviceToHost));
  CHECK(cudaMemcpy(hgp, gp, sizeof(hgp), cudaMemcpyDeviceToHost));
  for (int i = 0; i < R * H; ++i) want[i] = (float)(i % 5 - 2) * 0.25f;
  if (check_bf16("router weight bwd grad_x", h16, want, R * H)) return 1;
  for (int r = 0; r < R; ++r) {
    long s = 0;
    for (int h = 0; h < H; ++h) s += (long)((r * H + h) % 5 - 2) * ((r * H + h) % 7 - 3);
    if (hgp[r] != (float)s) {
      fprintf(stderr, "router weight bwd grad_probs[%d] is %g, want %ld\n", r, hgp[r], s);
      return 1;
    }
  }
  CHECK(cudaMemset(gx, 0, sizeof(h16)));
  CHECK(moe_router_weight_mul_bwd(g, MOE_BF16, NULL, MOE_BF16, p, gx, NULL, R, H, 0));
  CHECK(cudaMemcpy(h16, gx, sizeof(h16), cudaMemcpyDeviceToHost));
  if (check_bf16("router weight bwd grad_x (x not saved)", h16, want, R * H)) return 1;
  if (moe_router_weight_mul_bwd(g, MOE_BF16, x, MOE_BF16, p, gx, NULL, R, H, 0) != MOE_ERR_NULL) {
    fprintf(stderr, "x without grad_probs was not rejected\n");
    return 1;
  }
  CHECK(cudaFree(x));
  CHECK(cudaFree(g));
  CHECK(cudaFree(o16));
  CHECK(cudaFree(gx));
  CHECK(cudaFree(p));
  CHECK(cudaFree(o32));
  CHECK(cudaFree(gp));
  return 0;
}

/* squared ReLU with probabilities over a padded map: rows 0..9, n_used 8,
   map = {0, 1, -1, 2, 3, -1, 4, 5, 6, 7} (rows 2 and 5 padding), probs 0.5 */
static int run_act_permuted(void) {
  enum { MAXR = 10, W = 40, NUSED = 8, NP = 8 };
  const int32_t hmap[MAXR] = {0, 1, -1, 2, 3, -1, 4, 5, 6, 7};
  const int32_t hn = NUSED;
  static unsigned short hx[MAXR * W], ho[MAXR * W];
  static float hp[NP], want[MAXR * W];
  for (int i = 0; i < NP; ++i) hp[i] = 0.5f;
  for (int i = 0; i < MAXR * W; ++i) hx[i] = bf16_of((float)(i % 6 - 2));
  unsigned short *x, *o;
  int32_t *map, *n, *err;
  float* p;
  CHECK(cudaMalloc((void**)&x, sizeof(hx)));
  CHECK(cudaMalloc((void**)&o, sizeof(ho)));
  CHECK(cudaMalloc((void**)&map, sizeof(hmap)));
  CHECK(cudaMalloc((void**)&n, sizeof(hn)));
  CHECK(cudaMalloc((void**)&err, sizeof(int32_t)));
  CHECK(cudaMalloc((void**)&p, sizeof(hp)));
  CHECK(cudaMemcpy(x, hx, sizeof(hx), cudaMemcpyHostToDevice));
  CHECK(cudaMemcpy(map, hmap, sizeof(hmap), cudaMemcpyHostToDevice));
  CHECK(cudaMemcpy(n, &hn, sizeof(hn), cudaMemcpyHostToDevice));
  CHECK(cudaMemcpy(p, hp, sizeof(hp), cudaMemcpyHostToDevice));
  CHECK(cudaMemset(o, 0xFF, sizeof(ho)));
  CHECK(cudaMemset(err, 0, sizeof(int32_t)));
  CHECK(moe_act_with_probs_permuted(MOE_ACT_SQRELU, x, o, map, n, p, NP, MAXR, W, 1.0f, 1, err,
                                    0));
  CHECK(cudaMemcpy(ho, o, sizeof(ho), cudaMemcpyDeviceToHost));
  int32_t herr = -1;
  CHECK(cudaMemcpy(&herr, err, sizeof(herr), cudaMemcpyDeviceToHost));
  if (herr != 0) {
    fprintf(stderr, "act permuted: error word %d\n", herr);
    return 1;
  }
  for (int r = 0; r < NUSED; ++r)
    for (int c = 0; c < W; ++c) {
      const float v = (float)((r * W + c) % 6 - 2);
      want[r * W + c] = hmap[r] < 0 ? 0.0f : (v > 0 ? v * v : 0.0f) * 0.5f;
    }
  if (check_bf16("act permuted", ho, want, NUSED * W)) return 1;
  for (int i = NUSED * W; i < MAXR * W; ++i)
    if (ho[i] != 0xFFFF) {
      fprintf(stderr, "act permuted: element %d past n_used was written\n", i);
      return 1;
    }
  CHECK(cudaFree(x));
  CHECK(cudaFree(o));
  CHECK(cudaFree(map));
  CHECK(cudaFree(n));
  CHECK(cudaFree(err));
  CHECK(cudaFree(p));
  return 0;
}

/* fixed-order unpermute: 6 expert rows of small integers, 4 tokens x 3 local
   experts, valid_tokens 3 (token 3 untouched), bf16 in, fp32 out */
static int run_unpermute(void) {
  enum { ROWS = 6, T = 4, E = 3, H = 24, VALID = 3 };
  const int32_t hinv[T * E] = {0, -1, 3, 1, 2, -1, -1, -1, -1, 4, 5, 0};
  const int32_t hv = VALID;
  static unsigned short heo[ROWS * H];
  static float ho[T * H];
  for (int r = 0; r < ROWS; ++r)
    for (int c = 0; c < H; ++c) heo[r * H + c] = bf16_of((float)(10 * r + c % 9 - 4));
  unsigned short* eo;
  int32_t *inv, *v;
  float* o;
  CHECK(cudaMalloc((void**)&eo, sizeof(heo)));
  CHECK(cudaMalloc((void**)&inv, sizeof(hinv)));
  CHECK(cudaMalloc((void**)&v, sizeof(hv)));
  CHECK(cudaMalloc((void**)&o, sizeof(ho)));
  CHECK(cudaMemcpy(eo, heo, sizeof(heo), cudaMemcpyHostToDevice));
  CHECK(cudaMemcpy(inv, hinv, sizeof(hinv), cudaMemcpyHostToDevice));
  CHECK(cudaMemcpy(v, &hv, sizeof(hv), cudaMemcpyHostToDevice));
  for (int i = 0; i < T * H; ++i) ho[i] = -7.0f;
  CHECK(cudaMemcpy(o, ho, sizeof(ho), cudaMemcpyHostToDevice));
  CHECK(moe_unpermute_ordered(eo, MOE_BF16, ROWS, inv, v, o, MOE_FP32, T, H, E, NULL, 0));
  CHECK(cudaMemcpy(ho, o, sizeof(ho), cudaMemcpyDeviceToHost));
  for (int t = 0; t < T; ++t)
    for (int c = 0; c < H; ++c) {
      float want = -7.0f;                       /* token 3: untouched */
      if (t < VALID) {
        want = 0.0f;
        for (int e = 0; e < E; ++e)
          if (hinv[t * E + e] >= 0) want += (float)(10 * hinv[t * E + e] + c % 9 - 4);
      }
      if (ho[t * H + c] != want) {
        fprintf(stderr, "unpermute: token %d col %d is %g, want %g\n", t, c, ho[t * H + c],
                want);
        return 1;
      }
    }
  CHECK(cudaFree(eo));
  CHECK(cudaFree(inv));
  CHECK(cudaFree(v));
  CHECK(cudaFree(o));
  return 0;
}

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
  if (run_swiglu_bwd() || run_router_weight() || run_act_permuted() || run_unpermute()) return 1;
  CHECK(cudaDeviceSynchronize());
  printf("abi_smoke: ok (%s)\n", moe_status_string(MOE_OK));
  return 0;
}

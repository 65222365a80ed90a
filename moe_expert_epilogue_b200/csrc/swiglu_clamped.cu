// swiglu_clamped.cu -- clamped, probability-weighted SwiGLU, forward and
// one-pass backward (nemo_automodel.components.moe.swiglu_triton: module
// docstring, _swiglu_clamped_fwd_kernel, _swiglu_clamped_bwd_kernel).
//
//   y      = silu(clamp(g, max=L)) * clamp(u, -L, L) * p          fp32, one bf16 rounding
//   d_gate = dy * p * uc * silu'(gc)  on g <= L        (torch.clamp's inclusive masks)
//   d_up   = dy * p * silu(gc)        on -L <= u <= L
//   d_p    = sum_j dy * silu(gc) * uc
//
// Forward: a flat, persistent, grid-stride stream over 8-column chunks: per
// chunk two 16-byte loads (gate, up) and one 16-byte store.  Backward: a
// persistent loop over groups of rows; W threads own one row (one warp for the
// vectorised path), walk its chunks with a fixed column assignment, write
// d_gate / d_up straight into the two halves of grad_x and reduce the row's
// probability gradient with a fixed tree (per-thread partials in column order,
// warp butterfly, warps in index order).  No barrier is needed when W = 32, so
// every warp streams independently with its next loads already in flight.
#include "common.cuh"
#include "launch.cuh"

namespace moe {
namespace {

struct FwdMath {
  float L;
  __device__ __forceinline__ float operator()(float g, float u, float p) const {
    const float gc = clamp_max(g, L);
    const float uc = clamp_sym(u, L);
    const float s = gc * sigmoid(gc);
    return (s * uc) * p;
  }
};

struct BwdOut {
  float d_gate, d_up, t;
};

__device__ __forceinline__ BwdOut bwd_math(float g, float u, float dy, float p, float L) {
  const float gc = clamp_max(g, L);
  const float uc = clamp_sym(u, L);
  const float sg = sigmoid(gc);
  const float s = gc * sg;
  const float a = dy * p;
  const float dsilu = sg * (1.0f + gc * (1.0f - sg));
  BwdOut o;
  o.d_gate = (g <= L) ? (a * uc) * dsilu : 0.0f;
  o.d_up = (u >= -L && u <= L) ? a * s : 0.0f;
  o.t = dy * (s * uc);
  return o;
}

// ------------------------------------------------------------------ forward

template <int U>
__global__ void __launch_bounds__(kThreads)
swiglu_fwd_vec(const uint16_t* __restrict__ x, const float* __restrict__ probs,
               uint16_t* __restrict__ y, int64_t rows, int64_t inter, int64_t ld_x,
               int64_t ld_y, float L) {
  const int64_t cpr = inter / kVec;
  const int64_t total = rows * cpr;
  const int64_t S = (int64_t)gridDim.x * kThreads;
  int64_t q = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  if (q >= total) return;
  RowCursor cur(q, S, cpr);
  const FwdMath f{L};
  for (; q < total; q += U * S) {
    uint4 gw[U], uw[U];
    float p[U];
    uint16_t* dst[U];
#pragma unroll
    for (int k = 0; k < U; ++k) {
      if (q + k * S < total) {
        const uint16_t* src = x + cur.r * ld_x + cur.c * kVec;
        gw[k] = ld_stream(src);
        uw[k] = ld_stream(src + inter);
        p[k] = __ldg(probs + cur.r);
        dst[k] = y + cur.r * ld_y + cur.c * kVec;
      }
      cur.advance();
    }
#pragma unroll
    for (int k = 0; k < U; ++k) {
      if (q + k * S < total) {
        float g[8], u[8], o[8];
        unpack_bf16x8(gw[k], g);
        unpack_bf16x8(uw[k], u);
#pragma unroll
        for (int i = 0; i < 8; ++i) o[i] = f(g[i], u[i], p[k]);
        store8<BF16>(dst[k], o);
      }
    }
  }
}

// Warp-per-row forward for rows of at least 64 chunks: a warp owns one row at
// a time, loads the row's probability once and streams its chunks lane,
// lane + 32, ... with U chunks' loads in flight per lane.
template <int U>
__global__ void __launch_bounds__(kThreads)
swiglu_fwd_rows(const uint16_t* __restrict__ x, const float* __restrict__ probs,
                uint16_t* __restrict__ y, int64_t rows, int64_t inter, int64_t ld_x,
                int64_t ld_y, float L) {
  const int64_t cpr = inter / kVec;
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = (int64_t)gridDim.x * (kThreads / 32);
  const FwdMath f{L};
  for (int64_t r = (int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5); r < rows;
       r += nwarps) {
    const float p = __ldg(probs + r);
    const uint16_t* xr = x + r * ld_x;
    uint16_t* yr = y + r * ld_y;
    for (int64_t c0 = lane; c0 < cpr; c0 += 32 * U) {
      uint4 gw[U], uw[U];
#pragma unroll
      for (int k = 0; k < U; ++k) {
        const int64_t c = c0 + 32 * k;
        if (c < cpr) {
          gw[k] = ld_stream(xr + c * kVec);
          uw[k] = ld_stream(xr + inter + c * kVec);
        }
      }
#pragma unroll
      for (int k = 0; k < U; ++k) {
        const int64_t c = c0 + 32 * k;
        if (c < cpr) {
          float g[8], u[8], o[8];
          unpack_bf16x8(gw[k], g);
          unpack_bf16x8(uw[k], u);
#pragma unroll
          for (int i = 0; i < 8; ++i) o[i] = f(g[i], u[i], p);
          store8<BF16>(yr + c * kVec, o);
        }
      }
    }
  }
}

// Element-granular forward: any inter, leading dimensions and alignment.
__global__ void __launch_bounds__(kThreads)
swiglu_fwd_scalar(const uint16_t* __restrict__ x, const float* __restrict__ probs,
                  uint16_t* __restrict__ y, int64_t rows, int64_t inter, int64_t ld_x,
                  int64_t ld_y, float L) {
  const int64_t total = rows * inter;
  const int64_t S = (int64_t)gridDim.x * kThreads;
  int64_t q = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  if (q >= total) return;
  RowCursor cur(q, S, inter);
  const FwdMath f{L};
  for (; q < total; q += S, cur.advance()) {
    const uint16_t* src = x + cur.r * ld_x + cur.c;
    const float g = load1<BF16>(src), u = load1<BF16>(src + inter);
    store1<BF16>(y + cur.r * ld_y + cur.c, f(g, u, __ldg(probs + cur.r)));
  }
}

// ------------------------------------------------------------------ backward

// W threads per row (a multiple of 32), kThreads / W rows per CTA iteration.
// red[] is double-buffered so one __syncthreads per iteration suffices: a
// buffer is rewritten two iterations later, after every reader has passed
// the intervening barrier.
template <int W>
__device__ __forceinline__ float row_reduce(float acc, float (*red)[kThreads / 32], int parity) {
  acc = warp_sum(acc);
  if constexpr (W == 32) {
    return acc;
  } else {
    if ((threadIdx.x & 31) == 0) red[parity][threadIdx.x >> 5] = acc;
    __syncthreads();
    const int first = (threadIdx.x / W) * (W / 32);
    float s = 0.0f;
#pragma unroll
    for (int w = 0; w < W / 32; ++w) s += red[parity][first + w];
    return s;
  }
}

#ifndef MOE_SWIGLU_BWD_MIN_BLOCKS
#define MOE_SWIGLU_BWD_MIN_BLOCKS 1
#endif

template <int W, int U>
__global__ void __launch_bounds__(kThreads, MOE_SWIGLU_BWD_MIN_BLOCKS)
swiglu_bwd_vec(const uint16_t* __restrict__ x, const float* __restrict__ probs,
               const uint16_t* __restrict__ gy, uint16_t* __restrict__ gx,
               float* __restrict__ gp, int64_t rows, int64_t inter, int64_t ld_x,
               int64_t ld_gy, int64_t ld_gx, float L) {
  constexpr int G = kThreads / W;
  __shared__ float red[2][kThreads / 32];
  const int sub = threadIdx.x / W, lane = threadIdx.x % W;
  const int64_t cpr = inter / kVec;
  int parity = 0;
  for (int64_t r0 = (int64_t)blockIdx.x * G; r0 < rows; r0 += (int64_t)gridDim.x * G) {
    const int64_t r = r0 + sub;
    float acc = 0.0f;
    if (r < rows) {
      const float p = __ldg(probs + r);
      const uint16_t* xr = x + r * ld_x;
      const uint16_t* gyr = gy + r * ld_gy;
      uint16_t* gxr = gx + r * ld_gx;
      for (int64_t c0 = lane; c0 < cpr; c0 += (int64_t)U * W) {
        uint4 gw[U], uw[U], dw[U];
#pragma unroll
        for (int k = 0; k < U; ++k) {
          const int64_t c = c0 + (int64_t)k * W;
          if (c < cpr) {
            gw[k] = ld_stream(xr + c * kVec);
            uw[k] = ld_stream(xr + inter + c * kVec);
            dw[k] = ld_stream(gyr + c * kVec);
          }
        }
#pragma unroll
        for (int k = 0; k < U; ++k) {
          const int64_t c = c0 + (int64_t)k * W;
          if (c < cpr) {
            float g[8], u[8], d[8], og[8], ou[8];
            unpack_bf16x8(gw[k], g);
            unpack_bf16x8(uw[k], u);
            unpack_bf16x8(dw[k], d);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const BwdOut o = bwd_math(g[i], u[i], d[i], p, L);
              og[i] = o.d_gate;
              ou[i] = o.d_up;
              acc += o.t;
            }
            store8<BF16>(gxr + c * kVec, og);
            store8<BF16>(gxr + inter + c * kVec, ou);
          }
        }
      }
    }
    const float s = row_reduce<W>(acc, red, parity);
    if (r < rows && lane == 0) gp[r] = s;
    parity ^= 1;
  }
}

template <int W>
__global__ void __launch_bounds__(kThreads)
swiglu_bwd_scalar(const uint16_t* __restrict__ x, const float* __restrict__ probs,
                  const uint16_t* __restrict__ gy, uint16_t* __restrict__ gx,
                  float* __restrict__ gp, int64_t rows, int64_t inter, int64_t ld_x,
                  int64_t ld_gy, int64_t ld_gx, float L) {
  constexpr int G = kThreads / W;
  __shared__ float red[2][kThreads / 32];
  const int sub = threadIdx.x / W, lane = threadIdx.x % W;
  int parity = 0;
  for (int64_t r0 = (int64_t)blockIdx.x * G; r0 < rows; r0 += (int64_t)gridDim.x * G) {
    const int64_t r = r0 + sub;
    float acc = 0.0f;
    if (r < rows) {
      const float p = __ldg(probs + r);
      for (int64_t j = lane; j < inter; j += W) {
        const float g = load1<BF16>(x + r * ld_x + j);
        const float u = load1<BF16>(x + r * ld_x + inter + j);
        const float d = load1<BF16>(gy + r * ld_gy + j);
        const BwdOut o = bwd_math(g, u, d, p, L);
        store1<BF16>(gx + r * ld_gx + j, o.d_gate);
        store1<BF16>(gx + r * ld_gx + inter + j, o.d_up);
        acc += o.t;
      }
    }
    const float s = row_reduce<W>(acc, red, parity);
    if (r < rows && lane == 0) gp[r] = s;
    parity ^= 1;
  }
}

// Threads per row: the smallest of 32/64/128/256 that covers the row's work
// units (chunks or elements), so short rows do not idle a whole CTA.  The
// choice depends on the row length only, never on the number of rows.
inline int threads_per_row(int64_t units) {
  if (units <= 32) return 32;
  if (units <= 64) return 64;
  if (units <= 128) return 128;
  return 256;
}

template <class K>
int launch_persistent(K kernel, int64_t useful_blocks, cudaStream_t stream, const uint16_t* x,
                      const float* probs, const uint16_t* gy, uint16_t* gx, float* gp,
                      int64_t rows, int64_t inter, int64_t ld_x, int64_t ld_gy, int64_t ld_gx,
                      float L) {
  int grid;
  if (int rc = persistent_grid((const void*)kernel, 0, useful_blocks, &grid)) return rc;
  kernel<<<grid, kThreads, 0, stream>>>(x, probs, gy, gx, gp, rows, inter, ld_x, ld_gy, ld_gx,
                                        L);
  return check_launch();
}

}  // namespace

// Tuning knobs (compile-time).  kFwdUnroll: chunks whose loads a thread issues
// before it computes any of them.  kBwdRowThreads: threads that own one row in
// the backward (0: the smallest of 32/64/128/256 covering the row's chunks);
// it fixes the grad_probs summation tree together with the row length.
// kBwdUnroll: chunks per thread loaded ahead in the backward.
#ifndef MOE_SWIGLU_FWD_UNROLL
#define MOE_SWIGLU_FWD_UNROLL 2
#endif
#ifndef MOE_SWIGLU_FWD_ROW_UNROLL
#define MOE_SWIGLU_FWD_ROW_UNROLL 8
#endif
#ifndef MOE_SWIGLU_FWD_ROWS
#define MOE_SWIGLU_FWD_ROWS 1
#endif
#ifndef MOE_SWIGLU_BWD_ROW_THREADS
#define MOE_SWIGLU_BWD_ROW_THREADS 32
#endif
#ifndef MOE_SWIGLU_BWD_UNROLL
#define MOE_SWIGLU_BWD_UNROLL 4
#endif
constexpr int kFwdUnroll = MOE_SWIGLU_FWD_UNROLL;
constexpr int kFwdRowUnroll = MOE_SWIGLU_FWD_ROW_UNROLL;
constexpr bool kFwdRows = MOE_SWIGLU_FWD_ROWS != 0;
constexpr int kBwdRowThreads = MOE_SWIGLU_BWD_ROW_THREADS;
constexpr int kBwdUnroll = MOE_SWIGLU_BWD_UNROLL;

int launch_swiglu_clamped_fwd(const uint16_t* x, const float* probs, uint16_t* y, int64_t rows,
                              int64_t inter, int64_t ld_x, int64_t ld_y, float limit,
                              cudaStream_t stream) {
  const bool vec = inter % kVec == 0 && ld_x % kVec == 0 && ld_y % kVec == 0 && aligned16(x) &&
                   aligned16(y);
  int grid;
  if (vec && kFwdRows && inter / kVec >= 64) {
    auto k = swiglu_fwd_rows<kFwdRowUnroll>;
    if (int rc = persistent_grid((const void*)k, 0, (rows + kThreads / 32 - 1) / (kThreads / 32),
                                 &grid))
      return rc;
    k<<<grid, kThreads, 0, stream>>>(x, probs, y, rows, inter, ld_x, ld_y, limit);
  } else if (vec) {
    const int64_t units = rows * (inter / kVec);
    auto k = swiglu_fwd_vec<kFwdUnroll>;
    if (int rc = persistent_grid((const void*)k, 0,
                                 (units + kThreads * kFwdUnroll - 1) / (kThreads * kFwdUnroll),
                                 &grid))
      return rc;
    k<<<grid, kThreads, 0, stream>>>(x, probs, y, rows, inter, ld_x, ld_y, limit);
  } else {
    const int64_t units = rows * inter;
    if (int rc = persistent_grid((const void*)swiglu_fwd_scalar, 0,
                                 (units + kThreads - 1) / kThreads, &grid))
      return rc;
    swiglu_fwd_scalar<<<grid, kThreads, 0, stream>>>(x, probs, y, rows, inter, ld_x, ld_y,
                                                     limit);
  }
  return check_launch();
}

int launch_swiglu_clamped_bwd(const uint16_t* x, const float* probs, const uint16_t* grad_y,
                              uint16_t* grad_x, float* grad_probs, int64_t rows, int64_t inter,
                              int64_t ld_x, int64_t ld_gy, int64_t ld_gx, float limit,
                              cudaStream_t stream) {
  const bool vec = inter % kVec == 0 && ld_x % kVec == 0 && ld_gy % kVec == 0 &&
                   ld_gx % kVec == 0 && aligned16(x) && aligned16(grad_y) && aligned16(grad_x);
  const int W = (vec && kBwdRowThreads) ? kBwdRowThreads
                                        : threads_per_row(vec ? inter / kVec : inter);
  const int64_t blocks = (rows + kThreads / W - 1) / (kThreads / W);
#define MOE_BWD_ARGS stream, x, probs, grad_y, grad_x, grad_probs, rows, inter, ld_x, ld_gy, ld_gx, limit
  if (vec) {
    switch (W) {
      case 32: return launch_persistent(swiglu_bwd_vec<32, kBwdUnroll>, blocks, MOE_BWD_ARGS);
      case 64: return launch_persistent(swiglu_bwd_vec<64, kBwdUnroll>, blocks, MOE_BWD_ARGS);
      case 128: return launch_persistent(swiglu_bwd_vec<128, kBwdUnroll>, blocks, MOE_BWD_ARGS);
      default: return launch_persistent(swiglu_bwd_vec<256, kBwdUnroll>, blocks, MOE_BWD_ARGS);
    }
  }
  switch (W) {
    case 32: return launch_persistent(swiglu_bwd_scalar<32>, blocks, MOE_BWD_ARGS);
    case 64: return launch_persistent(swiglu_bwd_scalar<64>, blocks, MOE_BWD_ARGS);
    case 128: return launch_persistent(swiglu_bwd_scalar<128>, blocks, MOE_BWD_ARGS);
    default: return launch_persistent(swiglu_bwd_scalar<256>, blocks, MOE_BWD_ARGS);
  }
#undef MOE_BWD_ARGS
}

}  // namespace moe

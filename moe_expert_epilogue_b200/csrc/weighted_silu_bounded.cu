// weighted_silu_bounded.cu -- device-bounded weighted SwiGLU
// (core.inference.moe.batch_invariant: _weighted_silu_mul_bounded_kernel,
// weighted_silu_mul_bounded).
//
//   out[r, j] = bf16( silu(gate) * up * weights[r] ),  gate = y[r, j], up = y[r, half_n + j]
//
// fp32 math, one rounding, for every flat output element r * half_n + j below
// the device-resident bound (live_rows * half_n); elements at or past it are
// neither read nor written.  The grid is a fixed persistent one (CUDA-graph
// safe as the bound changes) whose size cannot change any bit: each element's
// instruction sequence is the same whichever thread computes it.  Rows of a
// multiple of 16 columns with 32-byte aligned bases take the flat kernel
// (threads stride over 16-column chunks); other layouts give one warp one row
// at a time.  Either way the one row the bound may cut is finished
// element-wise.
#include "common.cuh"
#include "launch.cuh"

namespace moe {
namespace {

__device__ __forceinline__ float weighted_silu(float g, float u, float w) {
  const float s = g * sigmoid(g);
  return (s * u) * w;
}

template <int U, bool VEC>
__global__ void __launch_bounds__(kThreads)
weighted_silu_bounded_kernel(const uint16_t* __restrict__ y, const float* __restrict__ w,
                             uint16_t* __restrict__ out, const int64_t* __restrict__ bound_p,
                             int64_t rows, int64_t half_n, int32_t* err) {
  pdl_prologue();
  int64_t bound = __ldg(bound_p);
  const int64_t total = rows * half_n;
  if (bound < 0 || bound > total) {
    if (blockIdx.x == 0 && threadIdx.x == 0) flag_error(err, MOE_DEVERR_COUNT);
    bound = bound < 0 ? 0 : total;
  }
  const int64_t live = (bound + half_n - 1) / half_n;     // rows with at least one element
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = (int64_t)gridDim.x * (kThreads / 32);
  for (int64_t r = (int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5); r < live;
       r += nwarps) {
    const int64_t limit = min(half_n, bound - r * half_n);  // elements of this row
    const float wr = __ldg(w + r);
    const uint16_t* yr = y + r * 2 * half_n;
    uint16_t* orow = out + r * half_n;
    if (VEC && limit == half_n) {
      const int64_t cpr = half_n / kVec;
      for (int64_t c0 = lane; c0 < cpr; c0 += 32 * U) {
        uint4 gw[U], uw[U];
#pragma unroll
        for (int k = 0; k < U; ++k) {
          const int64_t c = c0 + 32 * k;
          if (c < cpr) {
            gw[k] = ld_stream(yr + c * kVec);
            uw[k] = ld_stream(yr + half_n + c * kVec);
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
            for (int i = 0; i < 8; ++i) o[i] = weighted_silu(g[i], u[i], wr);
            store8<BF16>(orow + c * kVec, o);
          }
        }
      }
    } else {
      for (int64_t j = lane; j < limit; j += 32)
        orow[j] = f32_to_bf16(weighted_silu(load1<BF16>(yr + j), load1<BF16>(yr + half_n + j), wr));
    }
  }
}

// Flat form (half_n % 16 == 0, 32-byte aligned bases): threads stride over the
// 16-column chunks of the rows that lie wholly below the bound in row-major
// order (one 32-byte load of each half, one 32-byte store per chunk); the
// elements of the one row the bound cuts go element-wise to the grid's first
// threads.
__global__ void __launch_bounds__(kThreads)
weighted_silu_bounded_flat(const uint16_t* __restrict__ y, const float* __restrict__ w,
                           uint16_t* __restrict__ out, const int64_t* __restrict__ bound_p,
                           int64_t rows, int64_t half_n, int32_t* err) {
  pdl_prologue();
  int64_t bound = __ldg(bound_p);
  const int64_t total = rows * half_n;
  if (bound < 0 || bound > total) {
    if (blockIdx.x == 0 && threadIdx.x == 0) flag_error(err, MOE_DEVERR_COUNT);
    bound = bound < 0 ? 0 : total;
  }
  const int64_t full = bound / half_n;                    // rows wholly below the bound
  const int64_t cpr = half_n / 16;
  const int64_t chunks = full * cpr;
  const int64_t S = (int64_t)gridDim.x * kThreads;
  const int64_t t0 = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  if (t0 < chunks) {
    RowCursor cur(t0, S, cpr);
    for (int64_t q = t0; q < chunks; q += S, cur.advance()) {
      const uint16_t* yr = y + cur.r * 2 * half_n + cur.c * 16;
      const u4x2 gw = ld_stream32(yr);
      const u4x2 uw = ld_stream32(yr + half_n);
      const float wr = __ldg(w + cur.r);
      float o[2][8];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        float g[8], u[8];
        unpack_bf16x8(h ? gw.hi : gw.lo, g);
        unpack_bf16x8(h ? uw.hi : uw.lo, u);
#pragma unroll
        for (int i = 0; i < 8; ++i) o[h][i] = weighted_silu(g[i], u[i], wr);
      }
      st_stream32(out + cur.r * half_n + cur.c * 16, pack8<BF16>(o[0]), pack8<BF16>(o[1]));
    }
  }
  const int64_t cut = bound - full * half_n;              // elements of row `full`
  for (int64_t j = t0; j < cut; j += S) {
    const uint16_t* yr = y + full * 2 * half_n;
    out[full * half_n + j] =
        f32_to_bf16(weighted_silu(load1<BF16>(yr + j), load1<BF16>(yr + half_n + j), __ldg(w + full)));
  }
}

}  // namespace

#ifndef MOE_BOUNDED_UNROLL
#define MOE_BOUNDED_UNROLL 4
#endif
// The flat form at 4 CTAs per SM: measured on B200 at 65536 rows x half_n
// 1536, all live, 90.5 us against 97.4-98.1 with the warp-per-row kernel
// (3 / 6 CTAs per SM: 103.5 / 112.9).
#ifndef MOE_BOUNDED_FLAT
#define MOE_BOUNDED_FLAT 1
#endif
#ifndef MOE_BOUNDED_FLAT_CTAS
#define MOE_BOUNDED_FLAT_CTAS 4
#endif

int launch_weighted_silu_mul_bounded(const uint16_t* y, const float* weights, uint16_t* out,
                                     const int64_t* bound_elems, int64_t rows, int64_t half_n,
                                     int32_t num_programs, int32_t* dev_err,
                                     cudaStream_t stream) {
  const bool vec = half_n % kVec == 0 && aligned16(y) && aligned16(out);
  if (MOE_BOUNDED_FLAT && half_n % 16 == 0 && aligned32(y) && aligned32(out)) {
    int grid = num_programs;
    if (grid <= 0) {
      int sms = 0;
      if (int rc = device_sm_count(&sms)) return rc;
      const int64_t useful = (rows * (half_n / 16) + kThreads - 1) / kThreads;
      int64_t g = (int64_t)sms * MOE_BOUNDED_FLAT_CTAS;
      if (useful < g) g = useful;
      grid = (int)(g < 1 ? 1 : g);
    }
    launch_kernel(weighted_silu_bounded_flat, grid, 0, stream, y, weights, out, bound_elems, rows,
                  half_n, dev_err);
    return check_launch();
  }
  auto k = vec ? weighted_silu_bounded_kernel<MOE_BOUNDED_UNROLL, true>
               : weighted_silu_bounded_kernel<1, false>;
  int grid;
  if (num_programs > 0) {
    grid = num_programs;
  } else if (int rc = persistent_grid((const void*)k, 0, (rows + kThreads / 32 - 1) / (kThreads / 32),
                                      &grid)) {
    return rc;
  }
  launch_kernel(k, grid, 0, stream, y, weights, out, bound_elems, rows, half_n, dev_err);
  return check_launch();
}

}  // namespace moe

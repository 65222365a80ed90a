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
// instruction sequence is the same whichever warp computes it.  One warp owns
// one row at a time; the one row the bound may cut is finished element-wise.
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

}  // namespace

#ifndef MOE_BOUNDED_UNROLL
#define MOE_BOUNDED_UNROLL 4
#endif

int launch_weighted_silu_mul_bounded(const uint16_t* y, const float* weights, uint16_t* out,
                                     const int64_t* bound_elems, int64_t rows, int64_t half_n,
                                     int32_t num_programs, int32_t* dev_err,
                                     cudaStream_t stream) {
  const bool vec = half_n % kVec == 0 && aligned16(y) && aligned16(out);
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

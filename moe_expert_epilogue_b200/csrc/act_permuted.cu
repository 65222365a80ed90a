// act_permuted.cu -- batch-invariant activation with router probabilities
// over an expert-grouped, alignment-padded row layout
// (core.inference.moe.batch_invariant: _squared_relu_with_probs_kernel,
// squared_relu_with_probs, _swiglu_with_probs_kernel, swiglu_with_probs).
//
//   SQRELU:        out = bf16( bf16(relu(x)^2) * p )     the square is materialised in bf16
//   SQRELU_CLAMP:  z = s * tanh(x / s); out = bf16( relu(z)^2 * p )   fp32 throughout
//   SWIGLU:        out = bf16( silu(gate) * up * p )     gate | up halves of the row
//
// p = probs[permutation_map[r]].  Rows r < *n_used with a negative map entry
// are alignment padding: zero-filled when zero_padding is set, otherwise not
// touched.  Rows r >= *n_used are neither read nor written.  The kernel is a
// fixed persistent grid striding over (row, 8-column chunk) pairs up to the
// device-resident bound, so a captured graph stays valid as n_used changes,
// and every output element is computed by the same instruction sequence
// whatever the grid (batch invariance).
#include "common.cuh"
#include "launch.cuh"

namespace moe {
namespace {

constexpr int kUnroll = 2;

template <int ACT>
__device__ __forceinline__ float act_one(float a, float b, float p, float scale) {
  if constexpr (ACT == MOE_ACT_SQRELU) {
    const float rl = a < 0.0f ? 0.0f : a;                 // relu, NaN kept
    return round_to<BF16>(rl * rl) * p;
  } else if constexpr (ACT == MOE_ACT_SQRELU_CLAMP) {
    const float z = scale * tanhf(__fdiv_rn(a, scale));
    const float rl = z < 0.0f ? 0.0f : z;
    return (rl * rl) * p;
  } else {
    const float s = a * sigmoid(a);
    return (s * b) * p;
  }
}

// Reads the live-row bound, clamps it to [0, max_rows] and reports a bad one.
__device__ __forceinline__ int64_t live_rows(const int32_t* n_used, int64_t max_rows,
                                             int32_t* err) {
  int64_t n = __ldg(n_used);
  if (n < 0 || n > max_rows) {
    if (blockIdx.x == 0 && threadIdx.x == 0) flag_error(err, MOE_DEVERR_COUNT);
    n = n < 0 ? 0 : max_rows;
  }
  return n;
}

template <int ACT, bool VEC>
__global__ void __launch_bounds__(kThreads)
act_permuted_kernel(const uint16_t* __restrict__ x, uint16_t* __restrict__ out,
                    const int32_t* __restrict__ pmap, const int32_t* __restrict__ n_used,
                    const float* __restrict__ probs, int64_t num_probs, int64_t max_rows,
                    int64_t width, float scale, int zero_padding, int32_t* err) {
  const int64_t rows = live_rows(n_used, max_rows, err);
  constexpr int64_t unit = VEC ? kVec : 1;
  const int64_t upr = width / unit;                      // units per row
  const int64_t in_w = ACT == MOE_ACT_SWIGLU ? 2 * width : width;
  const int64_t total = rows * upr;
  const int64_t S = (int64_t)gridDim.x * kThreads;
  int64_t q = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  if (q >= total) return;
  RowCursor cur(q, S, upr);
  constexpr int U = VEC ? kUnroll : 1;
  for (; q < total; q += U * S) {
    uint4 a[U], b[U];
    float p[U];
    int64_t r[U], c[U];
    int state[U];  // 0: nothing, 1: compute, 2: write zeros
#pragma unroll
    for (int k = 0; k < U; ++k) {
      state[k] = 0;
      r[k] = cur.r;
      c[k] = cur.c;
      if (q + k * S < total) {
        const int32_t m = __ldg(pmap + cur.r);
        if (m < 0) {
          state[k] = zero_padding ? 2 : 0;
        } else if (m >= num_probs) {
          flag_error(err, MOE_DEVERR_MAP);
        } else {
          state[k] = 1;
          p[k] = __ldg(probs + m);
          const uint16_t* src = x + cur.r * in_w + cur.c * unit;
          if constexpr (VEC) {
            a[k] = ld_stream(src);
            if constexpr (ACT == MOE_ACT_SWIGLU) b[k] = ld_stream(src + width);
          } else {
            a[k].x = __ldg(src);
            if constexpr (ACT == MOE_ACT_SWIGLU) b[k].x = __ldg(src + width);
          }
        }
      }
      cur.advance();
    }
#pragma unroll
    for (int k = 0; k < U; ++k) {
      uint16_t* dst = out + r[k] * width + c[k] * unit;
      if (state[k] == 2) {
        if constexpr (VEC) st_stream(dst, make_uint4(0u, 0u, 0u, 0u));
        else *dst = 0;
      } else if (state[k] == 1) {
        if constexpr (VEC) {
          float av[8], bv[8], o[8];
          unpack_bf16x8(a[k], av);
          if constexpr (ACT == MOE_ACT_SWIGLU) unpack_bf16x8(b[k], bv);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            o[i] = act_one<ACT>(av[i], ACT == MOE_ACT_SWIGLU ? bv[i] : 0.0f, p[k], scale);
          store8<BF16>(dst, o);
        } else {
          const float av = __uint_as_float(a[k].x << 16);
          const float bv = ACT == MOE_ACT_SWIGLU ? __uint_as_float(b[k].x << 16) : 0.0f;
          *dst = f32_to_bf16(act_one<ACT>(av, bv, p[k], scale));
        }
      }
    }
  }
}

template <int ACT, bool VEC>
int launch_act(const uint16_t* x, uint16_t* out, const int32_t* pmap, const int32_t* n_used,
               const float* probs, int64_t num_probs, int64_t max_rows, int64_t width,
               float scale, int zero_padding, int32_t* err, cudaStream_t stream) {
  auto k = act_permuted_kernel<ACT, VEC>;
  const int64_t units = max_rows * (VEC ? width / kVec : width);
  const int64_t per_block = (int64_t)kThreads * (VEC ? kUnroll : 1);
  int grid;
  if (int rc = persistent_grid((const void*)k, 0, (units + per_block - 1) / per_block, &grid))
    return rc;
  k<<<grid, kThreads, 0, stream>>>(x, out, pmap, n_used, probs, num_probs, max_rows, width,
                                   scale, zero_padding, err);
  return check_launch();
}

}  // namespace

int launch_act_with_probs_permuted(moe_act act, const uint16_t* x, uint16_t* out,
                                   const int32_t* permutation_map, const int32_t* n_used,
                                   const float* probs, int64_t num_probs, int64_t max_rows,
                                   int64_t width, float clamp_scale, int zero_padding,
                                   int32_t* dev_err, cudaStream_t stream) {
  const bool vec = width % kVec == 0 && aligned16(x) && aligned16(out);
#define MOE_ACT_ARGS x, out, permutation_map, n_used, probs, num_probs, max_rows, width, \
                     clamp_scale, zero_padding, dev_err, stream
  switch (act) {
    case MOE_ACT_SQRELU:
      return vec ? launch_act<MOE_ACT_SQRELU, true>(MOE_ACT_ARGS)
                 : launch_act<MOE_ACT_SQRELU, false>(MOE_ACT_ARGS);
    case MOE_ACT_SQRELU_CLAMP:
      return vec ? launch_act<MOE_ACT_SQRELU_CLAMP, true>(MOE_ACT_ARGS)
                 : launch_act<MOE_ACT_SQRELU_CLAMP, false>(MOE_ACT_ARGS);
    default:
      return vec ? launch_act<MOE_ACT_SWIGLU, true>(MOE_ACT_ARGS)
                 : launch_act<MOE_ACT_SWIGLU, false>(MOE_ACT_ARGS);
  }
#undef MOE_ACT_ARGS
}

}  // namespace moe

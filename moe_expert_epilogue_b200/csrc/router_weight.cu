// router_weight.cu -- router-weight multiply in fp32, forward and backward
// (nemo_automodel.components.moe.optimized_ops: _rw_fwd_core, _rw_bwd_x_core,
// _rw_bwd_probs_core, _RouterWeightMulFunction).
//
//   fwd:  out    = (x.float() * p).to(out_dtype)             one multiply, one rounding
//   bwd:  grad_x = (g.float() * p).to(x_dtype)               one multiply, one rounding
//         grad_p = sum_h g.float() * x.float()               fp32 row reduction
//
// The forward and the x-only backward are flat grid-stride streams over
// 8-element chunks (an fp32 side 32-byte aligned moves each chunk with one
// 32-byte access; 16-bit input into fp32 output takes one 16-byte load and one
// 32-byte store per chunk).  The backward with the probability gradient walks
// rows like the SwiGLU backward: W threads per row, fixed column assignment,
// fixed reduction tree, no fp32 intermediate ever leaves the registers (16-bit
// rows with 32-byte alignment: 16-column chunks, otherwise 8).
#include <type_traits>

#include "common.cuh"
#include "launch.cuh"

namespace moe {
namespace {

// Chunks whose loads a thread issues before computing any of them: kUnroll in
// the backward with the probability gradient (two inputs per chunk), and
// kScaleUnroll 16-byte chunks in the one-input flat stream (halved for fp32
// inputs, whose chunks are 32 bytes).  Measured on B200 at [16384, 7168]:
// the forward 81.3 us with 2 chunks, 79.1 with 6, 75.8 with 8.
#ifndef MOE_RW_UNROLL
#define MOE_RW_UNROLL 2
#endif
#ifndef MOE_RW_SCALE_UNROLL
#define MOE_RW_SCALE_UNROLL 8
#endif
#ifndef MOE_RW_F32OUT_UNROLL
#define MOE_RW_F32OUT_UNROLL 4
#endif
// The backward with the probability gradient takes 32-byte loads for 16-bit
// g and x (rows of a multiple of 16 columns, 32-byte aligned): 4 chunks per
// thread in flight, 128 threads per 7168-wide row, 2 CTAs per SM.  Measured on
// B200 at [16384, 7168] bf16, back to back: 105.7-106.1 us against 111.7 with
// the 16-byte row kernel (grad_x identical); 2 chunks per thread at 4 / 3 / 2
// CTAs per SM: 109.3-109.7 / 108.1-108.2 / 123.7-123.9; 1 chunk: 111.8-112.0.
#ifndef MOE_RW_WIDE
#define MOE_RW_WIDE 1
#endif
#ifndef MOE_RW_WIDE_U
#define MOE_RW_WIDE_U 4
#endif
#ifndef MOE_RW_WIDE_CTAS
#define MOE_RW_WIDE_CTAS 0
#endif
constexpr int kUnroll = MOE_RW_UNROLL;
template <class DI>
constexpr int scale_unroll() { return MOE_RW_SCALE_UNROLL * 2 / DI::kBytes; }

// Routing probabilities may be bf16, fp16 or fp32 (widened exactly); the
// probability gradient is rounded to their dtype.  Once per row, so a runtime
// switch is free.
__device__ __forceinline__ float load_prob(const void* p, int dt, int64_t i) {
  if (dt == MOE_BF16) return __uint_as_float((uint32_t)__ldg(static_cast<const uint16_t*>(p) + i) << 16);
  if (dt == MOE_FP16) return f16_to_f32(__ldg(static_cast<const uint16_t*>(p) + i));
  return __ldg(static_cast<const float*>(p) + i);
}
// The same with the dtype fixed at compile time, for the flat streams that
// look a probability up per chunk.  Measured on B200 at [16384, 7168] bf16:
// with 16-bit probabilities the runtime switch inside the unrolled loop costs
// the forward 103-104 us against 77 with the dtype fixed; with fp32
// probabilities the runtime form is the faster one (80.6-80.9 us against
// 81.8-82.0), so PDT < 0 keeps it.
template <int PDT>
__device__ __forceinline__ float load_prob_t(const void* p, int p_dt, int64_t i) {
  if constexpr (PDT < 0) return load_prob(p, p_dt, i);
  else if constexpr (PDT == MOE_BF16)
    return __uint_as_float((uint32_t)__ldg(static_cast<const uint16_t*>(p) + i) << 16);
  else if constexpr (PDT == MOE_FP16)
    return f16_to_f32(__ldg(static_cast<const uint16_t*>(p) + i));
  else
    return __ldg(static_cast<const float*>(p) + i);
}
__device__ __forceinline__ void store_prob(void* p, int dt, int64_t i, float v) {
  if (dt == MOE_BF16) static_cast<uint16_t*>(p)[i] = f32_to_bf16(v);
  else if (dt == MOE_FP16) static_cast<uint16_t*>(p)[i] = f32_to_f16(v);
  else static_cast<float*>(p)[i] = v;
}

// out[r, :] = cast(in[r, :] * p[r]) over a [rows, cpr] chunk grid.
template <class DI, class DO, int PDT, bool A32 = false>
__global__ void __launch_bounds__(kThreads)
scale_rows_vec(const typename DI::T* __restrict__ in, const void* __restrict__ probs, int p_dt,
               typename DO::T* __restrict__ out, int64_t rows, int64_t hidden) {
  pdl_prologue();
  const int64_t cpr = hidden / kVec;
  const int64_t total = rows * cpr;
  const int64_t S = (int64_t)gridDim.x * kThreads;
  int64_t q = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  if (q >= total) return;
  RowCursor cur(q, S, cpr);
  constexpr int U = scale_unroll<DI>();
  for (; q < total; q += U * S) {
    Raw8<DI> raw[U];
    float p[U];
    int64_t off[U];
#pragma unroll
    for (int k = 0; k < U; ++k) {
      if (q + k * S < total) {
        off[k] = cur.r * hidden + cur.c * kVec;
        raw[k] = load8a<DI, A32>(in + off[k]);
        p[k] = load_prob_t<PDT>(probs, p_dt, cur.r);
      }
      cur.advance();
    }
#pragma unroll
    for (int k = 0; k < U; ++k) {
      if (q + k * S < total) {
        float v[8];
        widen8<DI>(raw[k], v);
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = v[i] * p[k];
        store8a<DO, A32>(out + off[k], v);
      }
    }
  }
}

// A 16-bit input scaled into fp32: units of 4 elements, so that a warp's
// 8-byte loads cover 256 contiguous bytes and its 16-byte stores 512 (with
// 8-element units each fp32 store instruction would cover every other 16
// bytes of a 1 KB span).  U units' loads in flight per thread.
template <class DI, int U, int PDT>
__global__ void __launch_bounds__(kThreads)
scale_rows_to_f32(const uint16_t* __restrict__ in, const void* __restrict__ probs, int p_dt,
                  float* __restrict__ out, int64_t rows, int64_t hidden) {
  pdl_prologue();
  const int64_t upr = hidden / 4;
  const int64_t total = rows * upr;
  const int64_t S = (int64_t)gridDim.x * kThreads;
  int64_t q = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  if (q >= total) return;
  RowCursor cur(q, S, upr);
  for (; q < total; q += U * S) {
    uint2 raw[U];
    float p[U];
    int64_t off[U];
#pragma unroll
    for (int k = 0; k < U; ++k) {
      if (q + k * S < total) {
        off[k] = cur.r * hidden + cur.c * 4;
        asm("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
            : "=r"(raw[k].x), "=r"(raw[k].y)
            : "l"(in + off[k]));
        p[k] = load_prob_t<PDT>(probs, p_dt, cur.r);
      }
      cur.advance();
    }
#pragma unroll
    for (int k = 0; k < U; ++k) {
      if (q + k * S < total) {
        float v[4];
        if constexpr (std::is_same<DI, BF16>::value) {
          v[0] = bf16_lo(raw[k].x); v[1] = bf16_hi(raw[k].x);
          v[2] = bf16_lo(raw[k].y); v[3] = bf16_hi(raw[k].y);
        } else {
          v[0] = f16_to_f32((uint16_t)(raw[k].x & 0xffffu)); v[1] = f16_to_f32((uint16_t)(raw[k].x >> 16));
          v[2] = f16_to_f32((uint16_t)(raw[k].y & 0xffffu)); v[3] = f16_to_f32((uint16_t)(raw[k].y >> 16));
        }
        st_stream(out + off[k], make_uint4(__float_as_uint(v[0] * p[k]), __float_as_uint(v[1] * p[k]),
                                           __float_as_uint(v[2] * p[k]), __float_as_uint(v[3] * p[k])));
      }
    }
  }
}

template <class DI, class DO>
__global__ void __launch_bounds__(kThreads)
scale_rows_scalar(const typename DI::T* __restrict__ in, const void* __restrict__ probs,
                  int p_dt, typename DO::T* __restrict__ out, int64_t rows, int64_t hidden) {
  pdl_prologue();
  const int64_t total = rows * hidden;
  const int64_t S = (int64_t)gridDim.x * kThreads;
  int64_t q = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  if (q >= total) return;
  RowCursor cur(q, S, hidden);
  for (; q < total; q += S, cur.advance())
    store1<DO>(out + q, load1<DI>(in + q) * load_prob(probs, p_dt, cur.r));
}

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

// Backward with the probability gradient.  VEC selects 8-element chunks
// (hidden % 8 == 0, 16-byte aligned) or single elements.
template <class DG, class DX, int W, bool VEC>
__global__ void __launch_bounds__(kThreads)
rw_bwd_rows(const typename DG::T* __restrict__ g, const typename DX::T* __restrict__ x,
            const void* __restrict__ probs, int p_dt, typename DX::T* __restrict__ gx,
            void* __restrict__ gp, int64_t rows, int64_t hidden) {
  pdl_prologue();
  constexpr int G = kThreads / W;
  __shared__ float red[2][kThreads / 32];
  const int sub = threadIdx.x / W, lane = threadIdx.x % W;
  int parity = 0;
  for (int64_t r0 = (int64_t)blockIdx.x * G; r0 < rows; r0 += (int64_t)gridDim.x * G) {
    const int64_t r = r0 + sub;
    float acc = 0.0f;
    if (r < rows) {
      const float p = load_prob(probs, p_dt, r);
      const int64_t base = r * hidden;
      if constexpr (VEC) {
        const int64_t cpr = hidden / kVec;
        for (int64_t c0 = lane; c0 < cpr; c0 += (int64_t)kUnroll * W) {
          Raw8<DG> rg[kUnroll];
          Raw8<DX> rx[kUnroll];
#pragma unroll
          for (int k = 0; k < kUnroll; ++k) {
            const int64_t c = c0 + (int64_t)k * W;
            if (c < cpr) {
              rg[k] = load8<DG>(g + base + c * kVec);
              rx[k] = load8<DX>(x + base + c * kVec);
            }
          }
#pragma unroll
          for (int k = 0; k < kUnroll; ++k) {
            const int64_t c = c0 + (int64_t)k * W;
            if (c < cpr) {
              float gv[8], xv[8], o[8];
              widen8<DG>(rg[k], gv);
              widen8<DX>(rx[k], xv);
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                o[i] = gv[i] * p;
                acc += gv[i] * xv[i];
              }
              store8<DX>(gx + base + c * kVec, o);
            }
          }
        }
      } else {
        for (int64_t j = lane; j < hidden; j += W) {
          const float gv = load1<DG>(g + base + j);
          store1<DX>(gx + base + j, gv * p);
          acc += gv * load1<DX>(x + base + j);
        }
      }
    }
    const float s = row_reduce<W>(acc, red, parity);
    if (r < rows && lane == 0) store_prob(gp, p_dt, r, s);
    parity ^= 1;
  }
}

// Backward with the probability gradient, 16-bit g and x, rows of a multiple
// of 16 columns with 32-byte aligned bases: 32-byte loads and stores, U chunks
// per thread in flight, W threads per row; each thread sums its columns in
// order, then the fixed tree -- a fixed order for a given row length.
template <class DG, class DX, int W, int U>
__global__ void __launch_bounds__(kThreads)
rw_bwd_wide(const uint16_t* __restrict__ g, const uint16_t* __restrict__ x,
            const void* __restrict__ probs, int p_dt, uint16_t* __restrict__ gx,
            void* __restrict__ gp, int64_t rows, int64_t hidden) {
  pdl_prologue();
  constexpr int G = kThreads / W;
  __shared__ float red[2][kThreads / 32];
  const int sub = threadIdx.x / W, lane = threadIdx.x % W;
  const int64_t cpr = hidden / 16;
  int parity = 0;
  for (int64_t r0 = (int64_t)blockIdx.x * G; r0 < rows; r0 += (int64_t)gridDim.x * G) {
    const int64_t r = r0 + sub;
    float acc = 0.0f;
    if (r < rows) {
      const float p = load_prob(probs, p_dt, r);
      const int64_t base = r * hidden;
      for (int64_t c0 = lane; c0 < cpr; c0 += (int64_t)U * W) {
        u4x2 rg[U], rx[U];
#pragma unroll
        for (int k = 0; k < U; ++k) {
          const int64_t c = c0 + (int64_t)k * W;
          if (c < cpr) {
            rg[k] = ld_stream32(g + base + c * 16);
            rx[k] = ld_stream32(x + base + c * 16);
          }
        }
#pragma unroll
        for (int k = 0; k < U; ++k) {
          const int64_t c = c0 + (int64_t)k * W;
          if (c < cpr) {
            float o[2][8];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              Raw8<DG> a;
              Raw8<DX> b;
              a.w[0] = h ? rg[k].hi : rg[k].lo;
              b.w[0] = h ? rx[k].hi : rx[k].lo;
              float gv[8], xv[8];
              widen8<DG>(a, gv);
              widen8<DX>(b, xv);
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                o[h][i] = gv[i] * p;
                acc += gv[i] * xv[i];
              }
            }
            st_stream32(gx + base + c * 16, pack8<DX>(o[0]), pack8<DX>(o[1]));
          }
        }
      }
    }
    const float sum = row_reduce<W>(acc, red, parity);
    if (r < rows && lane == 0) store_prob(gp, p_dt, r, sum);
    parity ^= 1;
  }
}

inline int threads_per_row(int64_t units) {
  if (units <= 32) return 32;
  if (units <= 64) return 64;
  if (units <= 128) return 128;
  return 256;
}

// A 16-bit input scaled into fp32 with 8-element units: one 16-byte load and
// one 32-byte store per unit (32-byte aligned output), U units per thread.
template <class DI, int U, int PDT>
__global__ void __launch_bounds__(kThreads)
scale_rows_to_f32_wide(const uint16_t* __restrict__ in, const void* __restrict__ probs, int p_dt,
                       float* __restrict__ out, int64_t rows, int64_t hidden) {
  pdl_prologue();
  const int64_t upr = hidden / kVec;
  const int64_t total = rows * upr;
  const int64_t S = (int64_t)gridDim.x * kThreads;
  int64_t q = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  if (q >= total) return;
  RowCursor cur(q, S, upr);
  for (; q < total; q += U * S) {
    Raw8<DI> raw[U];
    float p[U];
    int64_t off[U];
#pragma unroll
    for (int k = 0; k < U; ++k) {
      if (q + k * S < total) {
        off[k] = cur.r * hidden + cur.c * kVec;
        raw[k] = load8<DI>(reinterpret_cast<const typename DI::T*>(in) + off[k]);
        p[k] = load_prob_t<PDT>(probs, p_dt, cur.r);
      }
      cur.advance();
    }
#pragma unroll
    for (int k = 0; k < U; ++k) {
      if (q + k * S < total) {
        float v[8];
        widen8<DI>(raw[k], v);
        st_stream32(out + off[k],
                    make_uint4(__float_as_uint(v[0] * p[k]), __float_as_uint(v[1] * p[k]),
                               __float_as_uint(v[2] * p[k]), __float_as_uint(v[3] * p[k])),
                    make_uint4(__float_as_uint(v[4] * p[k]), __float_as_uint(v[5] * p[k]),
                               __float_as_uint(v[6] * p[k]), __float_as_uint(v[7] * p[k])));
      }
    }
  }
}

// Measured on B200 at [16384, 7168] bf16 -> fp32: 121.3-121.4 us with 2 units
// per thread (4 / 8: 121.5-121.6 / 122.4-122.5) against 124.4 with the
// 4-element units below.
#ifndef MOE_RW_F32OUT_WIDE
#define MOE_RW_F32OUT_WIDE 1
#endif
#ifndef MOE_RW_F32OUT_WIDE_U
#define MOE_RW_F32OUT_WIDE_U 2
#endif
// fp32 input or output sides with 32-byte alignment: one 32-byte access per
// 8-element chunk.  Measured on B200 at [16384, 7168], fp32 grad_out into bf16
// grad_x (x not saved): 112.8-113.0 us against 117.7.
#ifndef MOE_RW_F32_WIDE
#define MOE_RW_F32_WIDE 1
#endif

template <class DI, class DO, int PDT>
int launch_scale_t(const void* in, const void* probs, int p_dt, void* out, int64_t rows,
                   int64_t hidden, cudaStream_t stream) {
  const auto* i = static_cast<const typename DI::T*>(in);
  auto* o = static_cast<typename DO::T*>(out);
  int grid;
  if constexpr (DI::kBytes == 2 && DO::kBytes == 4) {
    if (MOE_RW_F32OUT_WIDE && hidden % kVec == 0 && aligned32(out) && aligned16(in)) {
      constexpr int U = MOE_RW_F32OUT_WIDE_U;
      auto k = scale_rows_to_f32_wide<DI, U, PDT>;
      const int64_t units = rows * (hidden / kVec);
      if (int rc = persistent_grid((const void*)k, 0, (units + kThreads * U - 1) / (kThreads * U),
                                   &grid))
        return rc;
      launch_kernel(k, grid, 0, stream, static_cast<const uint16_t*>(in), probs, p_dt,
                    static_cast<float*>(out), rows, hidden);
      return check_launch();
    }
    if (hidden % 4 == 0 && aligned16(out) && (reinterpret_cast<uintptr_t>(in) & 7u) == 0) {
      constexpr int U = MOE_RW_F32OUT_UNROLL;
      auto k = scale_rows_to_f32<DI, U, PDT>;
      const int64_t units = rows * (hidden / 4);
      if (int rc = persistent_grid((const void*)k, 0, (units + kThreads * U - 1) / (kThreads * U),
                                   &grid))
        return rc;
      launch_kernel(k, grid, 0, stream, static_cast<const uint16_t*>(in), probs, p_dt,
                    static_cast<float*>(out), rows, hidden);
      return check_launch();
    }
  }
  if (hidden % kVec == 0 && aligned16(in) && aligned16(out)) {
    // fp32 sides with 32-byte alignment take one 32-byte access per chunk
    const bool a32 = MOE_RW_F32_WIDE && (DI::kBytes == 4 || DO::kBytes == 4) &&
                     (DI::kBytes != 4 || aligned32(in)) && (DO::kBytes != 4 || aligned32(out));
    auto k = a32 ? scale_rows_vec<DI, DO, PDT, true> : scale_rows_vec<DI, DO, PDT, false>;
    const int64_t units = rows * (hidden / kVec);
    if (int rc = persistent_grid((const void*)k, 0,
                                 (units + kThreads * scale_unroll<DI>() - 1) /
                                     (kThreads * scale_unroll<DI>()),
                                 &grid))
      return rc;
    launch_kernel(k, grid, 0, stream, i, probs, p_dt, o, rows, hidden);
  } else {
    auto k = scale_rows_scalar<DI, DO>;
    if (int rc = persistent_grid((const void*)k, 0, (rows * hidden + kThreads - 1) / kThreads,
                                 &grid))
      return rc;
    launch_kernel(k, grid, 0, stream, i, probs, p_dt, o, rows, hidden);
  }
  return check_launch();
}

template <class DI, class DO>
int launch_scale(const void* in, const void* probs, int p_dt, void* out, int64_t rows,
                 int64_t hidden, cudaStream_t stream) {
  switch (p_dt) {
    case MOE_BF16:
      return launch_scale_t<DI, DO, MOE_BF16>(in, probs, p_dt, out, rows, hidden, stream);
    case MOE_FP16:
      return launch_scale_t<DI, DO, MOE_FP16>(in, probs, p_dt, out, rows, hidden, stream);
    default:
      return launch_scale_t<DI, DO, -1>(in, probs, p_dt, out, rows, hidden, stream);
  }
}

template <class DG, class DX, int W, bool VEC>
int launch_rows(const void* g, const void* x, const void* probs, int p_dt, void* gx, void* gp,
                int64_t rows, int64_t hidden, cudaStream_t stream) {
  auto k = rw_bwd_rows<DG, DX, W, VEC>;
  int grid;
  const int64_t blocks = (rows + kThreads / W - 1) / (kThreads / W);
  if (int rc = persistent_grid((const void*)k, 0, blocks, &grid)) return rc;
  launch_kernel(k, grid, 0, stream, static_cast<const typename DG::T*>(g),
                                   static_cast<const typename DX::T*>(x), probs, p_dt,
                                   static_cast<typename DX::T*>(gx), gp, rows, hidden);
  return check_launch();
}

template <class DG, class DX, int W>
int launch_wide(const void* g, const void* x, const void* probs, int p_dt, void* gx, void* gp,
                int64_t rows, int64_t hidden, cudaStream_t stream) {
  auto k = rw_bwd_wide<DG, DX, W, MOE_RW_WIDE_U>;
  int grid;
  const int64_t blocks = (rows + kThreads / W - 1) / (kThreads / W);
  if (int rc = persistent_grid((const void*)k, 0, blocks, &grid)) return rc;
  if (MOE_RW_WIDE_CTAS > 0) {
    int sms = 0;
    if (int rc = device_sm_count(&sms)) return rc;
    if ((int64_t)sms * MOE_RW_WIDE_CTAS < grid) grid = sms * MOE_RW_WIDE_CTAS;
  }
  launch_kernel(k, grid, 0, stream, static_cast<const uint16_t*>(g),
                static_cast<const uint16_t*>(x), probs, p_dt, static_cast<uint16_t*>(gx), gp,
                rows, hidden);
  return check_launch();
}

template <class DG, class DX>
int launch_bwd_with_probs(const void* g, const void* x, const void* probs, int p_dt, void* gx,
                          void* gp, int64_t rows, int64_t hidden, cudaStream_t stream) {
  if constexpr (DG::kBytes == 2 && DX::kBytes == 2) {
    if (MOE_RW_WIDE && hidden % 16 == 0 && aligned32(g) && aligned32(x) && aligned32(gx)) {
      const int W = threads_per_row(hidden / 16 / MOE_RW_WIDE_U);
      switch (W) {
        case 32: return launch_wide<DG, DX, 32>(g, x, probs, p_dt, gx, gp, rows, hidden, stream);
        case 64: return launch_wide<DG, DX, 64>(g, x, probs, p_dt, gx, gp, rows, hidden, stream);
        case 128: return launch_wide<DG, DX, 128>(g, x, probs, p_dt, gx, gp, rows, hidden, stream);
        default: return launch_wide<DG, DX, 256>(g, x, probs, p_dt, gx, gp, rows, hidden, stream);
      }
    }
  }
  const bool vec = hidden % kVec == 0 && aligned16(g) && aligned16(x) && aligned16(gx);
  const int W = threads_per_row(vec ? hidden / kVec : hidden);
#define MOE_RW_ARGS g, x, probs, p_dt, gx, gp, rows, hidden, stream
  if (vec) {
    switch (W) {
      case 32: return launch_rows<DG, DX, 32, true>(MOE_RW_ARGS);
      case 64: return launch_rows<DG, DX, 64, true>(MOE_RW_ARGS);
      case 128: return launch_rows<DG, DX, 128, true>(MOE_RW_ARGS);
      default: return launch_rows<DG, DX, 256, true>(MOE_RW_ARGS);
    }
  }
  switch (W) {
    case 32: return launch_rows<DG, DX, 32, false>(MOE_RW_ARGS);
    case 64: return launch_rows<DG, DX, 64, false>(MOE_RW_ARGS);
    case 128: return launch_rows<DG, DX, 128, false>(MOE_RW_ARGS);
    default: return launch_rows<DG, DX, 256, false>(MOE_RW_ARGS);
  }
#undef MOE_RW_ARGS
}

// Dispatch a (dtype, dtype) pair to a template taking two storage tags.
template <template <class, class> class F, class... A>
int dispatch2(moe_dtype a, moe_dtype b, A... args) {
#define MOE_CASE_B(TA)                                                   \
  switch (b) {                                                           \
    case MOE_BF16: return F<TA, BF16>::run(args...);                     \
    case MOE_FP16: return F<TA, F16>::run(args...);                      \
    default: return F<TA, F32>::run(args...);                            \
  }
  switch (a) {
    case MOE_BF16: MOE_CASE_B(BF16)
    case MOE_FP16: MOE_CASE_B(F16)
    default: MOE_CASE_B(F32)
  }
#undef MOE_CASE_B
}

template <class DI, class DO> struct Fwd {
  static int run(const void* x, const void* p, int p_dt, void* out, int64_t rows, int64_t hidden,
                 cudaStream_t s) {
    return launch_scale<DI, DO>(x, p, p_dt, out, rows, hidden, s);
  }
};

template <class DG, class DX> struct Bwd {
  static int run(const void* g, const void* x, const void* p, int p_dt, void* gx, void* gp,
                 int64_t rows, int64_t hidden, cudaStream_t s) {
    if (x == nullptr) return launch_scale<DG, DX>(g, p, p_dt, gx, rows, hidden, s);
    return launch_bwd_with_probs<DG, DX>(g, x, p, p_dt, gx, gp, rows, hidden, s);
  }
};

}  // namespace

int launch_router_weight_fwd(const void* x, moe_dtype x_dt, const void* probs, moe_dtype p_dt,
                             void* out, moe_dtype out_dt, int64_t rows, int64_t hidden,
                             cudaStream_t stream) {
  return dispatch2<Fwd>(x_dt, out_dt, x, probs, (int)p_dt, out, rows, hidden, stream);
}

int launch_router_weight_bwd(const void* grad_out, moe_dtype g_dt, const void* x,
                             moe_dtype x_dt, const void* probs, moe_dtype p_dt, void* grad_x,
                             void* grad_probs, int64_t rows, int64_t hidden,
                             cudaStream_t stream) {
  return dispatch2<Bwd>(g_dt, x_dt, grad_out, x, probs, (int)p_dt, grad_x, grad_probs, rows,
                        hidden, stream);
}

}  // namespace moe

// residual_add.cu -- fused MoE residual add
// (core.fusions.fused_moe_residual_add: module docstring, _moe_residual_add_kernel,
// fused_moe_residual_add).
//
//   out = residual + round_dt(expert_output + shared_expert_output)
//
// Both adds in fp32, each result rounded to the activation dtype, so the
// output is bit-identical to the two unfused adds.  One flat grid-stride
// stream: for 16-bit types with 32-byte aligned bases three 32-byte loads and
// one 32-byte store per 16 elements; for fp32 with 32-byte aligned bases the
// same per 8 elements; otherwise three 16-byte loads and one 16-byte store
// per 8 elements (two of each for fp32).  In place (out ==
// residual) is safe: every element is read and written by the same thread,
// load before store, and the residual is read through the coherent path
// (never the read-only one).
#include "common.cuh"
#include "launch.cuh"

namespace moe {
namespace {

constexpr int kUnroll = 2;

template <class D>
__device__ __forceinline__ float add_pair(float e, float s, float r) {
  return r + round_to<D>(e + s);
}

template <class D, bool A32 = false>
__global__ void __launch_bounds__(kThreads)
residual_add_vec(const typename D::T* e, const typename D::T* s, const typename D::T* r,
                 typename D::T* out, int64_t numel) {
  pdl_prologue();
  const int64_t chunks = numel / kVec;
  const int64_t S = (int64_t)gridDim.x * kThreads;
  const int64_t t0 = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  for (int64_t q = t0; q < chunks; q += kUnroll * S) {
    Raw8<D> re[kUnroll], rs[kUnroll], rr[kUnroll];
#pragma unroll
    for (int k = 0; k < kUnroll; ++k) {
      const int64_t c = q + k * S;
      if (c < chunks) {
        re[k] = load8a<D, A32>(e + c * kVec);
        rs[k] = load8a<D, A32>(s + c * kVec);
        rr[k] = load8a<D, A32, false>(r + c * kVec);  // r may alias out
      }
    }
#pragma unroll
    for (int k = 0; k < kUnroll; ++k) {
      const int64_t c = q + k * S;
      if (c < chunks) {
        float ve[8], vs[8], vr[8], o[8];
        widen8<D>(re[k], ve);
        widen8<D>(rs[k], vs);
        widen8<D>(rr[k], vr);
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
          float t0 = ve[i] + vs[i], t1 = ve[i + 1] + vs[i + 1];
          round2<D>(t0, t1);                            // the expert sum, rounded to D
          o[i] = vr[i] + t0;
          o[i + 1] = vr[i + 1] + t1;
        }
        store8a<D, A32>(out + c * kVec, o);
      }
    }
  }
  // ragged tail (numel % 8 elements): the first threads of the grid
  const int64_t tail = chunks * kVec + t0;
  if (tail < numel)
    store1<D>(out + tail, add_pair<D>(load1<D>(e + tail), load1<D>(s + tail), load1c<D>(r + tail)));
}

// 16-bit types, 32-byte aligned bases: 16 elements per chunk (three 32-byte
// loads, one 32-byte store), U chunks per thread, grid strides apart.
template <class D, int U>
__global__ void __launch_bounds__(kThreads)
residual_add_wide(const uint16_t* e, const uint16_t* s, const uint16_t* r, uint16_t* out,
                  int64_t numel) {
  pdl_prologue();
  const int64_t chunks = numel / 16;
  const int64_t S = (int64_t)gridDim.x * kThreads;
  const int64_t t0 = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  for (int64_t q = t0; q < chunks; q += U * S) {
    u4x2 re[U], rs[U], rr[U];
#pragma unroll
    for (int k = 0; k < U; ++k) {
      const int64_t c = q + k * S;
      if (c < chunks) {
        re[k] = ld_stream32(e + c * 16);
        rs[k] = ld_stream32(s + c * 16);
        rr[k] = ld_coherent32(r + c * 16);              // r may alias out
      }
    }
#pragma unroll
    for (int k = 0; k < U; ++k) {
      const int64_t c = q + k * S;
      if (c < chunks) {
        float o[2][8];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          Raw8<D> a, b, c8;
          a.w[0] = h ? re[k].hi : re[k].lo;
          b.w[0] = h ? rs[k].hi : rs[k].lo;
          c8.w[0] = h ? rr[k].hi : rr[k].lo;
          float ve[8], vs[8], vr[8];
          widen8<D>(a, ve);
          widen8<D>(b, vs);
          widen8<D>(c8, vr);
#pragma unroll
          for (int i = 0; i < 8; i += 2) {
            float t0 = ve[i] + vs[i], t1 = ve[i + 1] + vs[i + 1];
            round2<D>(t0, t1);
            o[h][i] = vr[i] + t0;
            o[h][i + 1] = vr[i + 1] + t1;
          }
        }
        st_stream32(out + c * 16, pack8<D>(o[0]), pack8<D>(o[1]));
      }
    }
  }
  const int64_t tail = chunks * 16 + t0;                  // numel % 16 elements
  if (tail < numel)
    store1<D>(out + tail, add_pair<D>(load1<D>(e + tail), load1<D>(s + tail), load1c<D>(r + tail)));
}

// The 32-byte form runs 2 chunks per thread at 2 CTAs per SM.  Measured on
// B200 at [32768, 7168] bf16, back to back: 270.0 us against 297.1 with the
// 16-byte stream at full occupancy (same bits); 1 chunk at 2 / 4 / 8 CTAs per
// SM: 338.5 / 275.7 / 279.6; 2 chunks at 1 / 3: 304.5 / 279.7; 3 chunks at 2:
// 278.6; 4 chunks at 1 / 2: 271.5 / 280.4.
#ifndef MOE_RES_WIDE
#define MOE_RES_WIDE 1
#endif
// fp32 with 32-byte aligned bases: one 32-byte access per 8-element chunk.
// Measured on B200 at [32768, 7168] fp32: 540.8-541.1 us against 594.8-594.9
// with two 16-byte accesses (chained after the router-weight forward: 793
// against 885).
#ifndef MOE_RES_F32_WIDE
#define MOE_RES_F32_WIDE 1
#endif
#ifndef MOE_RES_WIDE_U
#define MOE_RES_WIDE_U 2
#endif
#ifndef MOE_RES_WIDE_CTAS
#define MOE_RES_WIDE_CTAS 2
#endif

template <class D>
__global__ void __launch_bounds__(kThreads)
residual_add_scalar(const typename D::T* e, const typename D::T* s, const typename D::T* r,
                    typename D::T* out, int64_t numel) {
  pdl_prologue();
  const int64_t S = (int64_t)gridDim.x * kThreads;
  for (int64_t i = (int64_t)blockIdx.x * kThreads + threadIdx.x; i < numel; i += S)
    store1<D>(out + i, add_pair<D>(load1<D>(e + i), load1<D>(s + i), load1c<D>(r + i)));
}

template <class D>
int launch(const void* e, const void* s, const void* r, void* out, int64_t numel,
           cudaStream_t stream) {
  using T = typename D::T;
  const bool vec = aligned16(e) && aligned16(s) && aligned16(r) && aligned16(out);
  int grid;
  if constexpr (D::kBytes == 2) {
    if (MOE_RES_WIDE && aligned32(e) && aligned32(s) && aligned32(r) && aligned32(out)) {
      constexpr int U = MOE_RES_WIDE_U;
      auto k = residual_add_wide<D, U>;
      const int64_t chunks = numel / 16;
      const int64_t per_block = (int64_t)kThreads * U;
      if (int rc = persistent_grid((const void*)k, 0,
                                   chunks > 0 ? (chunks + per_block - 1) / per_block : 1, &grid))
        return rc;
      if (MOE_RES_WIDE_CTAS > 0) {
        int sms = 0;
        if (int rc = device_sm_count(&sms)) return rc;
        if ((int64_t)sms * MOE_RES_WIDE_CTAS < grid) grid = sms * MOE_RES_WIDE_CTAS;
      }
      launch_kernel(k, grid, 0, stream, static_cast<const uint16_t*>(e),
                    static_cast<const uint16_t*>(s), static_cast<const uint16_t*>(r),
                    static_cast<uint16_t*>(out), numel);
      return check_launch();
    }
  }
  if (vec) {
    const bool a32 = D::kBytes == 4 && MOE_RES_F32_WIDE && aligned32(e) && aligned32(s) &&
                     aligned32(r) && aligned32(out);
    auto k = a32 ? residual_add_vec<D, true> : residual_add_vec<D, false>;
    const int64_t chunks = numel / kVec;
    const int64_t per_block = (int64_t)kThreads * kUnroll;
    if (int rc = persistent_grid((const void*)k, 0, chunks > 0 ? (chunks + per_block - 1) / per_block : 1,
                                 &grid))
      return rc;
    launch_kernel(k, grid, 0, stream, static_cast<const T*>(e), static_cast<const T*>(s),
                                     static_cast<const T*>(r), static_cast<T*>(out), numel);
  } else {
    auto k = residual_add_scalar<D>;
    if (int rc = persistent_grid((const void*)k, 0, (numel + kThreads - 1) / kThreads, &grid))
      return rc;
    launch_kernel(k, grid, 0, stream, static_cast<const T*>(e), static_cast<const T*>(s),
                                     static_cast<const T*>(r), static_cast<T*>(out), numel);
  }
  return check_launch();
}

}  // namespace

int launch_residual_add(const void* e, const void* s, const void* r, void* out, int64_t numel,
                        moe_dtype dt, cudaStream_t stream) {
  switch (dt) {
    case MOE_BF16: return launch<BF16>(e, s, r, out, numel, stream);
    case MOE_FP16: return launch<F16>(e, s, r, out, numel, stream);
    default: return launch<F32>(e, s, r, out, numel, stream);
  }
}

}  // namespace moe

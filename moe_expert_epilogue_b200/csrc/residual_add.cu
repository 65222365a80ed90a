// residual_add.cu -- fused MoE residual add
// (core.fusions.fused_moe_residual_add: module docstring, _moe_residual_add_kernel,
// fused_moe_residual_add).
//
//   out = residual + round_dt(expert_output + shared_expert_output)
//
// Both adds in fp32, each result rounded to the activation dtype, so the
// output is bit-identical to the two unfused adds.  One flat grid-stride
// stream: three 16-byte loads and one 16-byte store per 8 elements (two of
// each for fp32).  In place (out == residual) is safe: every element is read
// and written by the same thread, load before store, and the residual is
// read through the coherent path (never the read-only one).
#include "common.cuh"
#include "launch.cuh"

namespace moe {
namespace {

constexpr int kUnroll = 2;

template <class D>
__device__ __forceinline__ float add_pair(float e, float s, float r) {
  return r + round_to<D>(e + s);
}

template <class D>
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
        re[k] = load8<D>(e + c * kVec);
        rs[k] = load8<D>(s + c * kVec);
        rr[k] = load8<D, false>(r + c * kVec);  // r may alias out
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
        store8<D>(out + c * kVec, o);
      }
    }
  }
  // ragged tail (numel % 8 elements): the first threads of the grid
  const int64_t tail = chunks * kVec + t0;
  if (tail < numel)
    store1<D>(out + tail, add_pair<D>(load1<D>(e + tail), load1<D>(s + tail), load1c<D>(r + tail)));
}

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
  if (vec) {
    auto k = residual_add_vec<D>;
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

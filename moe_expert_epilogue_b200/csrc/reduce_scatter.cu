// reduce_scatter.cu -- rank-order reduce-scatter of variable token rows
// (core.inference.moe.batch_invariant: ordered_reduce_scatter_v,
// _ordered_reduce_scatter_v_kernel).
//
// Every rank holds, at the same byte offset of a buffer that this GPU can
// address (its own memory, or a peer's memory mapped into this process), a
// row-major [capacity_rows, hidden] block of partial results for the tokens of
// all ranks.  This rank's output row t is the source row
// rank_token_offset[rank] + t, summed over the ranks in rank order in fp32,
//     acc = x_0;  acc = acc + x_1;  ...;  acc = acc + x_{world-1},
// and rounded once to the output dtype: the bits do not depend on the grid,
// the batch or which rank's data arrives first.
//
// The rank's rows are one contiguous block in every buffer, so the kernel is a
// single flat stream over local_tokens * hidden elements: per 8 elements, one
// 16-byte load from each rank (kGroup ranks' loads in flight at a time), the
// in-order sum, one 16-byte store.  Peer data is read with plain loads (no TMA, no cluster
// multicast), and the kernel never waits on another rank: the caller orders
// the launch after every rank's inputs are complete and before any rank
// overwrites them.
#include "common.cuh"
#include "launch.cuh"

namespace moe {
namespace {

// Measured on B200 (8 ranks' bf16 blocks of 8192 x 4096 on one GPU, and 2, 4
// and 8 ranks at other sizes): one vector per thread with 4 ranks' loads in
// flight (47 registers, 5 CTAs per SM) beats deeper per-thread batches (2
// vectors x 8 ranks: 150 registers, 1 CTA per SM) by 1.5-3x; parallelism
// across warps hides the latency better than depth within a thread here.
#ifndef MOE_RS_GROUP
#define MOE_RS_GROUP 4
#endif
#ifndef MOE_RS_UNROLL
#define MOE_RS_UNROLL 1
#endif
#ifndef MOE_RS_MIN_BLOCKS
#define MOE_RS_MIN_BLOCKS 0
#endif

constexpr int kMaxWorld = 64;             // ranks per reduce-scatter (kept in shared memory)
constexpr int kGroup = MOE_RS_GROUP;      // ranks whose loads are in flight together
constexpr int kUnroll = MOE_RS_UNROLL;    // vectors per thread and iteration

// Output rows [t_lo, t_hi) have their source row inside the data; the rest are
// neither read nor written and set MOE_DEVERR_COUNT.
struct RowRange {
  int64_t src0;      // source element index of output element 0 (may be negative)
  int64_t lo, hi;    // valid output elements
};

__device__ __forceinline__ RowRange valid_range(const int32_t* offs, int rank,
                                                const int32_t* ep_tokens, int64_t capacity,
                                                int64_t local, int64_t hidden, int32_t* err) {
  const int64_t first = __ldg(offs + rank);
  const int64_t ep = __ldg(ep_tokens);
  const int64_t avail = ep < 0 ? 0 : (ep > capacity ? capacity : ep);
  int64_t t_lo = first < 0 ? -first : 0;
  int64_t t_hi = avail - first < local ? avail - first : local;
  if (t_lo > local) t_lo = local;
  if (t_hi < t_lo) t_hi = t_lo;
  const bool bad = ep < 0 || ep > capacity || t_lo > 0 || t_hi < local;
  if (bad && blockIdx.x == 0 && threadIdx.x == 0) flag_error(err, MOE_DEVERR_COUNT);
  return {first * hidden, t_lo * hidden, t_hi * hidden};
}

// Reads the world's input bases (buffer + byte offset) into shared memory;
// true when every one of them is 16-byte aligned.
template <class DI>
__device__ __forceinline__ bool load_bases(const void* const* bufs, int64_t byte_off, int world,
                                           const typename DI::T** src) {
  int misaligned = 0;
  for (int q = threadIdx.x; q < world; q += blockDim.x) {
    const char* b = static_cast<const char*>(bufs[q]) + byte_off;
    misaligned |= (int)(reinterpret_cast<uintptr_t>(b) & 15);
    src[q] = reinterpret_cast<const typename DI::T*>(b);
  }
  return __syncthreads_or(misaligned) == 0;
}

// One element at a time, ranks summed in order (any alignment).
template <class DI, class DO>
__device__ __forceinline__ void rs_elements(const typename DI::T* const* src, const RowRange& R,
                                            int world, typename DO::T* out) {
  const int64_t S = (int64_t)gridDim.x * kThreads;
  for (int64_t e = R.lo + (int64_t)blockIdx.x * kThreads + threadIdx.x; e < R.hi; e += S) {
    const int64_t i = R.src0 + e;
    float acc = load1<DI>(src[0] + i);
    for (int q = 1; q < world; ++q) acc = acc + load1<DI>(src[q] + i);
    store1<DO>(out + e, acc);
  }
}

// Vector path: hidden % 8 == 0 and out and the byte offset 16-byte aligned;
// a buffer base that is not 16-byte aligned sends the whole grid down the
// element path instead.
template <class DI, class DO>
__global__ void __launch_bounds__(kThreads, MOE_RS_MIN_BLOCKS)
rs_vec(const void* const* __restrict__ bufs, int64_t byte_off, int world, int rank,
       const int32_t* __restrict__ offs, const int32_t* __restrict__ ep_tokens, int64_t capacity,
       typename DO::T* __restrict__ out, int64_t local, int64_t hidden, int32_t* err) {
  using TI = typename DI::T;
  __shared__ const TI* src[kMaxWorld];
  pdl_prologue();
  const RowRange R = valid_range(offs, rank, ep_tokens, capacity, local, hidden, err);
  if (!load_bases<DI>(bufs, byte_off, world, src)) {
    rs_elements<DI, DO>(src, R, world, out);
    return;
  }
  const int64_t c_lo = R.lo / kVec, c_hi = R.hi / kVec;
  const int64_t S = (int64_t)gridDim.x * kThreads;
  for (int64_t c0 = c_lo + (int64_t)blockIdx.x * kThreads + threadIdx.x; c0 < c_hi;
       c0 += kUnroll * S) {
    float acc[kUnroll][8];
    for (int q0 = 0; q0 < world; q0 += kGroup) {
      Raw8<DI> r[kUnroll][kGroup];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int64_t c = c0 + u * S;
#pragma unroll
        for (int k = 0; k < kGroup; ++k)
          if (c < c_hi && q0 + k < world) r[u][k] = load8<DI>(src[q0 + k] + (R.src0 + c * kVec));
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
#pragma unroll
        for (int k = 0; k < kGroup; ++k) {
          if (q0 + k < world) {
            float x[8];
            widen8<DI>(r[u][k], x);
            if (q0 + k == 0) {
#pragma unroll
              for (int i = 0; i < 8; ++i) acc[u][i] = x[i];
            } else {
#pragma unroll
              for (int i = 0; i < 8; ++i) acc[u][i] = acc[u][i] + x[i];
            }
          }
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int64_t c = c0 + u * S;
      if (c < c_hi) store8<DO>(out + c * kVec, acc[u]);
    }
  }
}

template <class DI, class DO>
__global__ void __launch_bounds__(kThreads)
rs_scalar(const void* const* __restrict__ bufs, int64_t byte_off, int world, int rank,
          const int32_t* __restrict__ offs, const int32_t* __restrict__ ep_tokens,
          int64_t capacity, typename DO::T* __restrict__ out, int64_t local, int64_t hidden,
          int32_t* err) {
  __shared__ const typename DI::T* src[kMaxWorld];
  pdl_prologue();
  const RowRange R = valid_range(offs, rank, ep_tokens, capacity, local, hidden, err);
  load_bases<DI>(bufs, byte_off, world, src);
  rs_elements<DI, DO>(src, R, world, out);
}

template <class DI, class DO>
int launch(const void* const* bufs, int64_t byte_off, int world, int rank, const int32_t* offs,
           const int32_t* ep_tokens, int64_t capacity, void* out, int64_t local, int64_t hidden,
           bool vec, int32_t* err, cudaStream_t stream) {
  using TO = typename DO::T;
  const int64_t n = local * hidden;
  int grid;
  if (vec) {
    auto k = rs_vec<DI, DO>;
    const int64_t per_block = (int64_t)kThreads * kUnroll * kVec;
    if (int rc = persistent_grid((const void*)k, 0, (n + per_block - 1) / per_block, &grid))
      return rc;
    {
      // the fewest CTAs that keep every thread's iteration count the same: no
      // partial last round of a few threads (one launch per rank is short, so
      // that round is a visible share of it; measured 65.8 -> 63.4 us for 8
      // ranks' blocks of 4096 tokens x 4096, neutral at larger sizes)
      const int64_t units = n / kVec, per = (int64_t)grid * kThreads * kUnroll;
      const int64_t iters = (units + per - 1) / per;
      const int64_t g = (units + iters * kThreads * kUnroll - 1) / (iters * kThreads * kUnroll);
      grid = (int)(g < 1 ? 1 : g);
    }
    launch_kernel(k, grid, 0, stream, bufs, byte_off, world, rank, offs, ep_tokens, capacity,
                  static_cast<TO*>(out), local, hidden, err);
  } else {
    auto k = rs_scalar<DI, DO>;
    if (int rc = persistent_grid((const void*)k, 0, (n + kThreads - 1) / kThreads, &grid))
      return rc;
    launch_kernel(k, grid, 0, stream, bufs, byte_off, world, rank, offs, ep_tokens, capacity,
                  static_cast<TO*>(out), local, hidden, err);
  }
  return check_launch();
}

template <class DI>
int dispatch_out(moe_dtype out_dt, const void* const* bufs, int64_t byte_off, int world, int rank,
                 const int32_t* offs, const int32_t* ep_tokens, int64_t capacity, void* out,
                 int64_t local, int64_t hidden, bool vec, int32_t* err, cudaStream_t stream) {
  switch (out_dt) {
    case MOE_BF16:
      return launch<DI, BF16>(bufs, byte_off, world, rank, offs, ep_tokens, capacity, out, local,
                              hidden, vec, err, stream);
    case MOE_FP16:
      return launch<DI, F16>(bufs, byte_off, world, rank, offs, ep_tokens, capacity, out, local,
                             hidden, vec, err, stream);
    default:
      return launch<DI, F32>(bufs, byte_off, world, rank, offs, ep_tokens, capacity, out, local,
                             hidden, vec, err, stream);
  }
}

}  // namespace

int max_reduce_scatter_world() { return kMaxWorld; }

int launch_ordered_reduce_scatter_v(const void* const* bufs, int64_t byte_off, int world, int rank,
                                    const int32_t* offs, const int32_t* ep_tokens,
                                    int64_t capacity, void* out, int64_t local, int64_t hidden,
                                    moe_dtype in_dt, moe_dtype out_dt, int32_t* err,
                                    cudaStream_t stream) {
  const bool vec = hidden % kVec == 0 && aligned16(out) && byte_off % 16 == 0;
  switch (in_dt) {
    case MOE_BF16:
      return dispatch_out<BF16>(out_dt, bufs, byte_off, world, rank, offs, ep_tokens, capacity,
                                out, local, hidden, vec, err, stream);
    case MOE_FP16:
      return dispatch_out<F16>(out_dt, bufs, byte_off, world, rank, offs, ep_tokens, capacity,
                               out, local, hidden, vec, err, stream);
    default:
      return dispatch_out<F32>(out_dt, bufs, byte_off, world, rank, offs, ep_tokens, capacity,
                               out, local, hidden, vec, err, stream);
  }
}

}  // namespace moe

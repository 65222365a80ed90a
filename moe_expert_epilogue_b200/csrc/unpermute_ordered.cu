// unpermute_ordered.cu -- token-local, batch-invariant unpermute
// (core.inference.moe.batch_invariant: _unpermute_tokens_in_expert_order_kernel,
// unpermute_tokens_in_expert_order).
//
//   out[t, :] = cast( ((+0 + eo[row_0, :]) + eo[row_1, :]) + ... )
//
// where row_0, row_1, ... are the inverse-map entries of token t in
// increasing local expert id.  fp32 sequential adds, no atomics: the bits of
// a token depend only on that token's rows, never on the grid or the batch.
//
// For E <= 64 a warp owns one (token, column range) item at a time and
// compacts the token's inverse-map row itself (unpermute_warp); otherwise one
// CTA owns one token at a time (persistent loop up to the device-resident
// valid_tokens) and warp 0 compacts a token's inverse-map row into an ordered
// list of live rows in shared memory, one token ahead.  Either way the
// compaction (ballot + popc) keeps the increasing-expert order, and every
// thread issues the loads of up to 8 contributing rows of its chunk (8 or 16
// columns) before it adds them in list order.
#include "common.cuh"
#include "launch.cuh"
#include "rowlist.cuh"

namespace moe {
namespace {

// contributing rows loaded before they are summed: 128 bytes per thread in flight
template <class DI> constexpr int kBatch = DI::kBytes == 4 ? 4 : 8;
// the same for the 32-byte loads of 16-bit inputs (256 bytes per thread)
#ifndef MOE_UNPERMUTE_WIDE_BATCH
#define MOE_UNPERMUTE_WIDE_BATCH 8
#endif

// The CTA walks tokens t = blockIdx.x, + gridDim.x, ...  Row lists are
// double-buffered and built one token ahead by warp 0: at the top of an
// iteration warp 0 issues the loads of the NEXT token's inverse-map row (for
// E <= 64: two entries per lane, into registers), gathers its own share of the
// current token, and only then compacts the next list, so the map latency hides
// behind the gathers.  One barrier per token: it publishes the list built in
// the previous iteration and retires the buffer about to be rebuilt.
template <class DI, class DO, bool VEC, bool SMALL_E>
__global__ void __launch_bounds__(kThreads)
unpermute_kernel(const typename DI::T* __restrict__ eo, int64_t max_rows,
                 const int32_t* __restrict__ inv, const int32_t* __restrict__ valid_tokens,
                 typename DO::T* __restrict__ out, int64_t tokens, int64_t hidden, int E,
                 int32_t* err) {
  pdl_prologue();
  extern __shared__ int32_t s_list[];  // [2][E]
  __shared__ int s_count[2];
  int64_t n = __ldg(valid_tokens);
  if (n < 0 || n > tokens) {
    if (blockIdx.x == 0 && threadIdx.x == 0) flag_error(err, MOE_DEVERR_COUNT);
    n = n < 0 ? 0 : tokens;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int64_t t = blockIdx.x;
  if (t >= n) return;                                   // CTA-uniform
  if (warp == 0) {
    const int c = compact_row(inv + t * E, E, max_rows, s_list, err, lane);
    if (lane == 0) s_count[0] = c;
  }
  for (int parity = 0; t < n; t += gridDim.x, parity ^= 1) {
    __syncthreads();
    const int32_t* list = s_list + parity * E;
    const int count = s_count[parity];
    const int64_t t_next = t + gridDim.x;
    const bool build = warp == 0 && t_next < n;         // warp-uniform
    int32_t p0 = -1, p1 = -1;
    if (SMALL_E && build) {
      const int32_t* nrow = inv + t_next * E;
      if (lane < E) p0 = __ldg(nrow + lane);
      if (lane + 32 < E) p1 = __ldg(nrow + lane + 32);
    }
    if constexpr (VEC) {
      const int64_t cpr = hidden / kVec;
      for (int64_t c = threadIdx.x; c < cpr; c += kThreads) {
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
        for (int j0 = 0; j0 < count; j0 += kBatch<DI>) {
          Raw8<DI> raw[kBatch<DI>];
#pragma unroll
          for (int j = 0; j < kBatch<DI>; ++j)
            if (j0 + j < count) raw[j] = load8<DI>(eo + (int64_t)list[j0 + j] * hidden + c * kVec);
#pragma unroll
          for (int j = 0; j < kBatch<DI>; ++j) {
            if (j0 + j < count) {
              float v[8];
              widen8<DI>(raw[j], v);
#pragma unroll
              for (int i = 0; i < 8; ++i) acc[i] = acc[i] + v[i];
            }
          }
        }
        store8<DO>(out + t * hidden + c * kVec, acc);
      }
    } else {
      for (int64_t h = threadIdx.x; h < hidden; h += kThreads) {
        float acc = 0.0f;
        for (int j = 0; j < count; ++j) acc = acc + load1<DI>(eo + (int64_t)list[j] * hidden + h);
        store1<DO>(out + t * hidden + h, acc);
      }
    }
    if (build) {
      int32_t* next = s_list + (parity ^ 1) * E;
      const int c = SMALL_E ? compact_pair(p0, p1, max_rows, next, err, lane)
                            : compact_row(inv + t_next * E, E, max_rows, next, err, lane);
      if (lane == 0) s_count[parity ^ 1] = c;
    }
  }
}

// Barrier-free variant for E <= 64 (the unpermute counterpart of the fused
// epilogue's): a warp owns one work item -- a token and one of SPLIT equal
// column ranges of its hidden dimension -- compacts the token's inverse-map
// row itself (entries loaded during the previous item) into its own list, and
// never waits for the other warps.  CH is the columns per lane per load: 8
// (16 bytes) or, for 16-bit inputs, 16 (32 bytes).
#ifndef MOE_UNPERMUTE_MIN_BLOCKS
#define MOE_UNPERMUTE_MIN_BLOCKS 0
#endif
#if MOE_UNPERMUTE_MIN_BLOCKS > 0
#define MOE_UNPERMUTE_MIN_BLOCKS_ATTR __launch_bounds__(kThreads, MOE_UNPERMUTE_MIN_BLOCKS)
#else
#define MOE_UNPERMUTE_MIN_BLOCKS_ATTR __launch_bounds__(kThreads)
#endif

template <class DI, class DO, int SPLIT, int CH>
__global__ void MOE_UNPERMUTE_MIN_BLOCKS_ATTR
unpermute_warp(const typename DI::T* __restrict__ eo, int64_t max_rows,
               const int32_t* __restrict__ inv, const int32_t* __restrict__ valid_tokens,
               typename DO::T* __restrict__ out, int64_t tokens, int64_t hidden, int E,
               int32_t* err) {
  pdl_prologue();
  __shared__ int32_t s_list[kThreads / 32][64];
  int64_t n = __ldg(valid_tokens);
  if (n < 0 || n > tokens) {
    if (blockIdx.x == 0 && threadIdx.x == 0) flag_error(err, MOE_DEVERR_COUNT);
    n = n < 0 ? 0 : tokens;
  }
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t nwarps = (int64_t)gridDim.x * (kThreads / 32);
  const int64_t items = n * SPLIT;
  const int64_t cpr = hidden / CH;
  const int64_t cpi = (cpr + SPLIT - 1) / SPLIT;
  int32_t* list = s_list[warp];
  int64_t it = (int64_t)blockIdx.x * (kThreads / 32) + warp;
  if (it >= items) return;                                 // warp-uniform
  int32_t p0, p1;
  {
    const int32_t* row = inv + (it / SPLIT) * E;
    p0 = lane < E ? __ldg(row + lane) : -1;
    p1 = lane + 32 < E ? __ldg(row + lane + 32) : -1;
  }
  constexpr int B = kBatch<DI>;
  constexpr int WB = MOE_UNPERMUTE_WIDE_BATCH;
  for (; it < items; it += nwarps) {
    const int64_t t = it / SPLIT;
    __syncwarp();
    const int count = compact_pair(p0, p1, max_rows, list, err, lane);
    __syncwarp();
    const int64_t itn = it + nwarps;
    if (itn < items) {
      const int32_t* row = inv + (itn / SPLIT) * E;
      p0 = lane < E ? __ldg(row + lane) : -1;
      p1 = lane + 32 < E ? __ldg(row + lane + 32) : -1;
    }
    const int64_t c_end = min(cpr, (it % SPLIT + 1) * cpi);
    for (int64_t c = (it % SPLIT) * cpi + lane; c < c_end; c += 32) {
      if constexpr (CH == 8) {
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
        for (int j0 = 0; j0 < count; j0 += B) {
          Raw8<DI> raw[B];
#pragma unroll
          for (int j = 0; j < B; ++j)
            if (j0 + j < count) raw[j] = load8<DI>(eo + (int64_t)list[j0 + j] * hidden + c * kVec);
#pragma unroll
          for (int j = 0; j < B; ++j) {
            if (j0 + j < count) {
              float v[8];
              widen8<DI>(raw[j], v);
#pragma unroll
              for (int i = 0; i < 8; ++i) acc[i] = acc[i] + v[i];
            }
          }
        }
        store8<DO>(out + t * hidden + c * kVec, acc);
      } else {
        // 16 columns of a 16-bit input per 32-byte load
        float lo[8], hi[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) lo[i] = hi[i] = 0.0f;
        for (int j0 = 0; j0 < count; j0 += WB) {
          u4x2 raw[WB];
#pragma unroll
          for (int j = 0; j < WB; ++j)
            if (j0 + j < count) raw[j] = ld_stream32(eo + (int64_t)list[j0 + j] * hidden + c * 16);
#pragma unroll
          for (int j = 0; j < WB; ++j) {
            if (j0 + j < count) {
              Raw8<DI> a, b;
              a.w[0] = raw[j].lo;
              b.w[0] = raw[j].hi;
              float va[8], vb[8];
              widen8<DI>(a, va);
              widen8<DI>(b, vb);
#pragma unroll
              for (int i = 0; i < 8; ++i) {
                lo[i] = lo[i] + va[i];
                hi[i] = hi[i] + vb[i];
              }
            }
          }
        }
        typename DO::T* o = out + t * hidden + c * 16;
        if constexpr (DO::kBytes == 2) {
          st_stream32(o, pack8<DO>(lo), pack8<DO>(hi));
        } else {
          store8<DO>(o, lo);
          store8<DO>(o + 8, hi);
        }
      }
    }
  }
}

#ifndef MOE_UNPERMUTE_WARP_ITEMS
#define MOE_UNPERMUTE_WARP_ITEMS 1
#endif
// 16-bit inputs with hidden % 16 == 0 and 32-byte aligned bases take 32-byte
// loads (16 columns per lane, all of a token's rows in flight) with items of
// two lane rounds.  Measured on B200 at 8192 tokens x top-8 of 64, hidden
// 4096, bf16: 94.4 us against 105.7 with 16-byte loads, bit-identical (items
// of 1 / 4 rounds: 95.1 / 95.2; 4 rows in flight: 95.2-95.8).
#ifndef MOE_UNPERMUTE_WIDE
#define MOE_UNPERMUTE_WIDE 1
#endif
#ifndef MOE_UNPERMUTE_WIDE_ROUNDS
#define MOE_UNPERMUTE_WIDE_ROUNDS 2
#endif

template <class DI, class DO, int CH>
int launch_unpermute_warp(const void* eo, int64_t max_rows, const int32_t* inv,
                          const int32_t* valid_tokens, void* out, int64_t tokens, int64_t hidden,
                          int E, int32_t* err, cudaStream_t stream, int rounds) {
  const int64_t cpr = hidden / CH;
  const int64_t per = cpr / (32 * rounds);
  const int split = per >= 8 ? 8 : per >= 4 ? 4 : per >= 2 ? 2 : 1;
  auto k = split == 8 ? unpermute_warp<DI, DO, 8, CH> : split == 4 ? unpermute_warp<DI, DO, 4, CH>
         : split == 2 ? unpermute_warp<DI, DO, 2, CH> : unpermute_warp<DI, DO, 1, CH>;
  int grid;
  const int64_t warps = tokens * split;
  if (int rc = persistent_grid((const void*)k, 0, (warps + kThreads / 32 - 1) / (kThreads / 32),
                               &grid))
    return rc;
  launch_kernel(k, grid, 0, stream, static_cast<const typename DI::T*>(eo), max_rows, inv,
                valid_tokens, static_cast<typename DO::T*>(out), tokens, hidden, E, err);
  return check_launch();
}

template <class DI, class DO>
int launch_unpermute(const void* eo, int64_t max_rows, const int32_t* inv,
                     const int32_t* valid_tokens, void* out, int64_t tokens, int64_t hidden,
                     int E, int32_t* err, cudaStream_t stream) {
  const bool vec = hidden % kVec == 0 && aligned16(eo) && aligned16(out);
  if constexpr (DI::kBytes == 2) {
    if (MOE_UNPERMUTE_WIDE && MOE_UNPERMUTE_WARP_ITEMS && E <= 64 && hidden % 16 == 0 &&
        aligned32(eo) && aligned32(out))
      return launch_unpermute_warp<DI, DO, 16>(eo, max_rows, inv, valid_tokens, out, tokens,
                                               hidden, E, err, stream, MOE_UNPERMUTE_WIDE_ROUNDS);
  }
  if (MOE_UNPERMUTE_WARP_ITEMS && vec && E <= 64)
    return launch_unpermute_warp<DI, DO, 8>(eo, max_rows, inv, valid_tokens, out, tokens, hidden,
                                            E, err, stream, 4);
  const size_t smem = 2 * (size_t)E * sizeof(int32_t);
  auto k = vec ? (E <= 64 ? unpermute_kernel<DI, DO, true, true> : unpermute_kernel<DI, DO, true, false>)
              : (E <= 64 ? unpermute_kernel<DI, DO, false, true>
                         : unpermute_kernel<DI, DO, false, false>);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute((const void*)k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return cuda_fail(e);
  }
  int grid;
  if (int rc = persistent_grid((const void*)k, smem, tokens > 0 ? tokens : 1, &grid)) return rc;
  launch_kernel(k, grid, smem, stream, static_cast<const typename DI::T*>(eo), max_rows, inv,
                                      valid_tokens, static_cast<typename DO::T*>(out), tokens,
                                      hidden, E, err);
  return check_launch();
}

template <class DI>
int dispatch_out(moe_dtype out_dt, const void* eo, int64_t max_rows, const int32_t* inv,
                 const int32_t* vt, void* out, int64_t tokens, int64_t hidden, int E,
                 int32_t* err, cudaStream_t s) {
  switch (out_dt) {
    case MOE_BF16: return launch_unpermute<DI, BF16>(eo, max_rows, inv, vt, out, tokens, hidden, E, err, s);
    case MOE_FP16: return launch_unpermute<DI, F16>(eo, max_rows, inv, vt, out, tokens, hidden, E, err, s);
    default: return launch_unpermute<DI, F32>(eo, max_rows, inv, vt, out, tokens, hidden, E, err, s);
  }
}

}  // namespace

int launch_unpermute_ordered(const void* expert_output, moe_dtype in_dt, int64_t max_rows,
                             const int32_t* inverse_map, const int32_t* valid_tokens,
                             void* out, moe_dtype out_dt, int64_t tokens, int64_t hidden,
                             int32_t num_local_experts, int32_t* dev_err,
                             cudaStream_t stream) {
  switch (in_dt) {
    case MOE_BF16:
      return dispatch_out<BF16>(out_dt, expert_output, max_rows, inverse_map, valid_tokens, out,
                                tokens, hidden, num_local_experts, dev_err, stream);
    case MOE_FP16:
      return dispatch_out<F16>(out_dt, expert_output, max_rows, inverse_map, valid_tokens, out,
                               tokens, hidden, num_local_experts, dev_err, stream);
    default:
      return dispatch_out<F32>(out_dt, expert_output, max_rows, inverse_map, valid_tokens, out,
                               tokens, hidden, num_local_experts, dev_err, stream);
  }
}

}  // namespace moe

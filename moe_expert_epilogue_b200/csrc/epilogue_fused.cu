// epilogue_fused.cu -- the MoE epilogue chain in one pass:
//   router-weight multiply (nemo_automodel.components.moe.optimized_ops,
//     _rw_fwd_core, applied to the expert-grouped rows with their permuted
//     probabilities),
//   fixed-order unpermute (core.inference.moe.batch_invariant,
//     _unpermute_tokens_in_expert_order_kernel),
//   residual + (routed + shared) add (core.fusions.fused_moe_residual_add).
//
// Bit-identical to the three materialised steps, because every rounding of the
// chain is kept in registers:
//   w_j    = round_dt(eo[row_j, :] * row_probs[row_j])        step 1, per row
//   routed = round_dt(((+0 + w_0) + w_1) + ...)               step 2, fp32, rows in
//                                                              increasing expert order
//   out    = round_dt(residual + round_dt(routed + shared))   step 3
// The chain reads every expert row, the shared output and the residual once and
// writes out once; the two [tokens, hidden] intermediates and the weighted copy
// of the expert rows never reach memory.  The step-1 product is an explicitly
// rounded multiply (__fmul_rn), so it is never fused into the step-2 add, for
// fp32 as for the 16-bit types.
//
// Structure: the unpermute's -- a warp per (token, column range) with its own
// row list for E <= 64 (below), else one CTA per token at a time with row
// lists compacted one token ahead by warp 0 and one barrier per token; each
// thread gathers the rows of its chunk (and the rows' probabilities, which
// stay in L1) with the shared and residual chunks in flight beside them.
#include "common.cuh"
#include "launch.cuh"
#include "rowlist.cuh"

namespace moe {
namespace {

template <class D> constexpr int kRowsAhead = 4;

template <class D, bool VEC, bool SMALL_E>
__global__ void __launch_bounds__(kThreads)
epilogue_fused_kernel(const typename D::T* __restrict__ eo, const float* __restrict__ row_probs,
                      int64_t max_rows, const int32_t* __restrict__ inv,
                      const int32_t* __restrict__ valid_tokens,
                      const typename D::T* __restrict__ shared, const typename D::T* residual,
                      typename D::T* out, int64_t tokens, int64_t hidden, int E, int32_t* err) {
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
  constexpr int B = kRowsAhead<D>;
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
    const int64_t base = t * hidden;
    if constexpr (VEC) {
      const int64_t cpr = hidden / kVec;
      for (int64_t c = threadIdx.x; c < cpr; c += kThreads) {
        const Raw8<D> rs = load8<D>(shared + base + c * kVec);
        const Raw8<D> rr = load8<D, false>(residual + base + c * kVec);  // may alias out
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
        for (int j0 = 0; j0 < count; j0 += B) {
          Raw8<D> raw[B];
          float p[B];
#pragma unroll
          for (int j = 0; j < B; ++j) {
            if (j0 + j < count) {
              const int64_t row = list[j0 + j];
              raw[j] = load8<D>(eo + row * hidden + c * kVec);
              p[j] = __ldg(row_probs + row);
            }
          }
#pragma unroll
          for (int j = 0; j < B; ++j) {
            if (j0 + j < count) {
              float v[8];
              widen8<D>(raw[j], v);
#pragma unroll
              for (int i = 0; i < 8; i += 2) {
                float w0 = __fmul_rn(v[i], p[j]), w1 = __fmul_rn(v[i + 1], p[j]);
                round2<D>(w0, w1);                      // step 1's rounding, two at a time
                acc[i] = acc[i] + w0;
                acc[i + 1] = acc[i + 1] + w1;
              }
            }
          }
        }
        float vs[8], vr[8];
        widen8<D>(rs, vs);
        widen8<D>(rr, vr);
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
          round2<D>(acc[i], acc[i + 1]);                // step 2's rounding
          float t0 = acc[i] + vs[i], t1 = acc[i + 1] + vs[i + 1];
          round2<D>(t0, t1);                            // step 3's first rounding
          acc[i] = vr[i] + t0;
          acc[i + 1] = vr[i + 1] + t1;
        }
        store8<D>(out + base + c * kVec, acc);
      }
    } else {
      for (int64_t h = threadIdx.x; h < hidden; h += kThreads) {
        float acc = 0.0f;
        for (int j = 0; j < count; ++j) {
          const int64_t row = list[j];
          acc = acc + round_to<D>(__fmul_rn(load1<D>(eo + row * hidden + h), __ldg(row_probs + row)));
        }
        const float s = load1<D>(shared + base + h), r = load1c<D>(residual + base + h);
        store1<D>(out + base + h, r + round_to<D>(round_to<D>(acc) + s));
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

// Barrier-free variant for E <= 64: a warp owns one work item -- a token and
// one of SPLIT equal column ranges of its hidden dimension -- at a time.  The
// warp compacts the token's inverse-map row itself (two entries per lane,
// already loaded during the previous item) into its own shared-memory list,
// so warps never wait for each other; items = tokens * SPLIT keep the load
// balanced across the persistent grid.
// CH is the columns per lane per load.  With 16-byte loads (CH = 8) more
// resident warps hide the gather latency better than more rows in flight per
// warp: 4 rows at 4 CTAs per SM (64 registers) for the 16-bit types, measured
// 122.5 us against 127.6 (8 rows, 3 CTAs) and 138 (8 rows, the compiler's 102
// registers, 2 CTAs) at 8192 tokens x top-8, hidden 4096; fp32 keeps 3 CTAs (4
// would spill).  16-bit types with hidden % 16 == 0 and 32-byte aligned bases
// take 32-byte loads (CH = 16): 4 rows in flight at 2 CTAs per SM, 119.5 us
// against 122.6 on the same shape, bit-identical (2 rows at 3 CTAs: 124.1).
template <class D> constexpr int kFusedMinBlocks = D::kBytes == 4 ? 3 : 4;
#ifndef MOE_FUSED_WIDE
#define MOE_FUSED_WIDE 1
#endif
#ifndef MOE_FUSED_WIDE_ROWS
#define MOE_FUSED_WIDE_ROWS 4
#endif
#ifndef MOE_FUSED_WIDE_MIN_BLOCKS
#define MOE_FUSED_WIDE_MIN_BLOCKS 2
#endif
#ifndef MOE_FUSED_WIDE_ROUNDS
#define MOE_FUSED_WIDE_ROUNDS 4
#endif

template <class D, int SPLIT, int CH>
__global__ void __launch_bounds__(kThreads, CH == 16 ? MOE_FUSED_WIDE_MIN_BLOCKS : kFusedMinBlocks<D>)
epilogue_fused_warp(const typename D::T* __restrict__ eo, const float* __restrict__ row_probs,
                    int64_t max_rows, const int32_t* __restrict__ inv,
                    const int32_t* __restrict__ valid_tokens,
                    const typename D::T* __restrict__ shared, const typename D::T* residual,
                    typename D::T* out, int64_t tokens, int64_t hidden, int E, int32_t* err) {
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
  const int64_t cpi = (cpr + SPLIT - 1) / SPLIT;          // chunks per item
  int32_t* list = s_list[warp];
  int64_t it = (int64_t)blockIdx.x * (kThreads / 32) + warp;
  if (it >= items) return;                                 // warp-uniform
  int32_t p0, p1;
  {
    const int32_t* row = inv + (it / SPLIT) * E;
    p0 = lane < E ? __ldg(row + lane) : -1;
    p1 = lane + 32 < E ? __ldg(row + lane + 32) : -1;
  }
  constexpr int B = kRowsAhead<D>;
  constexpr int WB = MOE_FUSED_WIDE_ROWS;
  for (; it < items; it += nwarps) {
    const int64_t t = it / SPLIT;
    __syncwarp();                                          // the previous list is consumed
    const int count = compact_pair(p0, p1, max_rows, list, err, lane);
    __syncwarp();
    const int64_t itn = it + nwarps;
    if (itn < items) {                                     // next item's entries, in flight
      const int32_t* row = inv + (itn / SPLIT) * E;
      p0 = lane < E ? __ldg(row + lane) : -1;
      p1 = lane + 32 < E ? __ldg(row + lane + 32) : -1;
    }
    const int64_t base = t * hidden;
    const int64_t c_end = min(cpr, (it % SPLIT + 1) * cpi);
    for (int64_t c = (it % SPLIT) * cpi + lane; c < c_end; c += 32) {
      if constexpr (CH == 8) {
        const Raw8<D> rs = load8<D>(shared + base + c * kVec);
        const Raw8<D> rr = load8<D, false>(residual + base + c * kVec);  // may alias out
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
        for (int j0 = 0; j0 < count; j0 += B) {
          Raw8<D> raw[B];
          float p[B];
#pragma unroll
          for (int j = 0; j < B; ++j) {
            if (j0 + j < count) {
              const int64_t row = list[j0 + j];
              raw[j] = load8<D>(eo + row * hidden + c * kVec);
              p[j] = __ldg(row_probs + row);
            }
          }
#pragma unroll
          for (int j = 0; j < B; ++j) {
            if (j0 + j < count) {
              float v[8];
              widen8<D>(raw[j], v);
#pragma unroll
              for (int i = 0; i < 8; i += 2) {
                float w0 = __fmul_rn(v[i], p[j]), w1 = __fmul_rn(v[i + 1], p[j]);
                round2<D>(w0, w1);
                acc[i] = acc[i] + w0;
                acc[i + 1] = acc[i + 1] + w1;
              }
            }
          }
        }
        float vs[8], vr[8];
        widen8<D>(rs, vs);
        widen8<D>(rr, vr);
#pragma unroll
        for (int i = 0; i < 8; i += 2) {
          round2<D>(acc[i], acc[i + 1]);
          float t0 = acc[i] + vs[i], t1 = acc[i + 1] + vs[i + 1];
          round2<D>(t0, t1);
          acc[i] = vr[i] + t0;
          acc[i + 1] = vr[i + 1] + t1;
        }
        store8<D>(out + base + c * kVec, acc);
      } else {
        // 16 columns per lane: 32-byte loads and store (16-bit types)
        const u4x2 rs = ld_stream32(shared + base + c * 16);
        const u4x2 rr = ld_coherent32(residual + base + c * 16);   // may alias out
        float acc[2][8];
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[h][i] = 0.0f;
        for (int j0 = 0; j0 < count; j0 += WB) {
          u4x2 raw[WB];
          float p[WB];
#pragma unroll
          for (int j = 0; j < WB; ++j) {
            if (j0 + j < count) {
              const int64_t row = list[j0 + j];
              raw[j] = ld_stream32(eo + row * hidden + c * 16);
              p[j] = __ldg(row_probs + row);
            }
          }
#pragma unroll
          for (int j = 0; j < WB; ++j) {
            if (j0 + j < count) {
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                Raw8<D> r8;
                r8.w[0] = h ? raw[j].hi : raw[j].lo;
                float v[8];
                widen8<D>(r8, v);
#pragma unroll
                for (int i = 0; i < 8; i += 2) {
                  float w0 = __fmul_rn(v[i], p[j]), w1 = __fmul_rn(v[i + 1], p[j]);
                  round2<D>(w0, w1);
                  acc[h][i] = acc[h][i] + w0;
                  acc[h][i + 1] = acc[h][i + 1] + w1;
                }
              }
            }
          }
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          Raw8<D> s8, r8;
          s8.w[0] = h ? rs.hi : rs.lo;
          r8.w[0] = h ? rr.hi : rr.lo;
          float vs[8], vr[8];
          widen8<D>(s8, vs);
          widen8<D>(r8, vr);
#pragma unroll
          for (int i = 0; i < 8; i += 2) {
            round2<D>(acc[h][i], acc[h][i + 1]);
            float t0 = acc[h][i] + vs[i], t1 = acc[h][i + 1] + vs[i + 1];
            round2<D>(t0, t1);
            acc[h][i] = vr[i] + t0;
            acc[h][i + 1] = vr[i + 1] + t1;
          }
        }
        st_stream32(out + base + c * 16, pack8<D>(acc[0]), pack8<D>(acc[1]));
      }
    }
  }
}

#ifndef MOE_FUSED_WARP_ITEMS
#define MOE_FUSED_WARP_ITEMS 1
#endif

template <class D, int CH>
auto fused_warp_for(int split) {
  return split == 8 ? epilogue_fused_warp<D, 8, CH> : split == 4 ? epilogue_fused_warp<D, 4, CH>
       : split == 2 ? epilogue_fused_warp<D, 2, CH> : epilogue_fused_warp<D, 1, CH>;
}

template <class D>
int launch(const void* eo, const float* row_probs, int64_t max_rows, const int32_t* inv,
           const int32_t* valid_tokens, const void* shared, const void* residual, void* out,
           int64_t tokens, int64_t hidden, int E, int32_t* err, cudaStream_t stream) {
  using T = typename D::T;
  const bool vec = hidden % kVec == 0 && aligned16(eo) && aligned16(shared) &&
                   aligned16(residual) && aligned16(out);
  bool wide = false;
  if constexpr (D::kBytes == 2)
    wide = MOE_FUSED_WIDE && hidden % 16 == 0 && aligned32(eo) && aligned32(shared) &&
           aligned32(residual) && aligned32(out);
  if (MOE_FUSED_WARP_ITEMS && vec && E <= 64) {
    // SPLIT: items per token, the largest power of two <= chunks per row / (32 x rounds)
    const int64_t per = wide ? hidden / 16 / (32 * MOE_FUSED_WIDE_ROUNDS) : hidden / kVec / 128;
    const int split = per >= 8 ? 8 : per >= 4 ? 4 : per >= 2 ? 2 : 1;
    auto k = fused_warp_for<D, 8>(split);
    if constexpr (D::kBytes == 2)
      if (wide) k = fused_warp_for<D, 16>(split);
    int grid;
    const int64_t warps = tokens * split;
    if (int rc = persistent_grid((const void*)k, 0, (warps + kThreads / 32 - 1) / (kThreads / 32),
                                 &grid))
      return rc;
    launch_kernel(k, grid, 0, stream, static_cast<const T*>(eo), row_probs, max_rows, inv,
                                     valid_tokens, static_cast<const T*>(shared),
                                     static_cast<const T*>(residual), static_cast<T*>(out),
                                     tokens, hidden, E, err);
    return check_launch();
  }
  const size_t smem = 2 * (size_t)E * sizeof(int32_t);
  auto k = vec ? (E <= 64 ? epilogue_fused_kernel<D, true, true>
                          : epilogue_fused_kernel<D, true, false>)
               : (E <= 64 ? epilogue_fused_kernel<D, false, true>
                          : epilogue_fused_kernel<D, false, false>);
  int grid;
  if (int rc = persistent_grid((const void*)k, smem, tokens > 0 ? tokens : 1, &grid)) return rc;
  launch_kernel(k, grid, smem, stream, static_cast<const T*>(eo), row_probs, max_rows, inv,
                                      valid_tokens, static_cast<const T*>(shared),
                                      static_cast<const T*>(residual), static_cast<T*>(out),
                                      tokens, hidden, E, err);
  return check_launch();
}

}  // namespace

int launch_epilogue_fused(const void* expert_output, const float* row_probs, int64_t max_rows,
                          const int32_t* inverse_map, const int32_t* valid_tokens,
                          const void* shared_expert_output, const void* residual, void* out,
                          int64_t tokens, int64_t hidden, int32_t num_local_experts,
                          moe_dtype dt, int32_t* dev_err, cudaStream_t stream) {
#define MOE_FUSED_ARGS expert_output, row_probs, max_rows, inverse_map, valid_tokens, \
                       shared_expert_output, residual, out, tokens, hidden, num_local_experts, \
                       dev_err, stream
  switch (dt) {
    case MOE_BF16: return launch<BF16>(MOE_FUSED_ARGS);
    case MOE_FP16: return launch<F16>(MOE_FUSED_ARGS);
    default: return launch<F32>(MOE_FUSED_ARGS);
  }
#undef MOE_FUSED_ARGS
}

}  // namespace moe

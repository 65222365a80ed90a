// swiglu_clamped.cu -- clamped, probability-weighted SwiGLU, forward and
// one-pass backward (nemo_automodel.components.moe.swiglu_triton: module
// docstring, _swiglu_clamped_fwd_kernel, _swiglu_clamped_bwd_kernel,
// _SUPPORTED_DTYPES = bf16, fp16, fp32).
//
//   y      = silu(clamp(g, max=L)) * clamp(u, -L, L) * p          fp32, one rounding to x.dtype
//   d_gate = dy * p * uc * silu'(gc)  on g <= L        (torch.clamp's inclusive masks)
//   d_up   = dy * p * silu(gc)        on -L <= u <= L
//   d_p    = sum_j dy * silu(gc) * uc
//
// Forward: TMA-staged.  One CTA per SM; a producer thread copies whole rows
// (gate | up, one cp.async.bulk each) into a ring of S shared-memory stages
// (16, or 8 for rows too long for 16 -- fp32 rows of more than 1592 columns),
// and 8 consumer warps compute rows out of shared memory, writing y straight
// to global memory -- S rows (up to ~200 KB) in flight per SM without holding
// them in registers (measured at rows 65536, inter 2048: 4 % faster than the
// register-staged kernel in bf16, 14 % in fp32).  Rows too long even for 8
// stages: one warp per row (warps stride over the rows), the row's
// probability loaded once, U chunks of 8 columns per lane in flight (two
// loads each: gate, up), one 16-byte store per chunk (two for fp32); a flat
// grid-stride variant serves rows shorter than 64 chunks.  Backward: W threads
// own one row (one warp for the vectorised path), walk its chunks with a fixed
// column assignment, write d_gate / d_up straight into the two halves of
// grad_x and reduce the row's probability gradient with a fixed tree
// (per-thread partials in column order, warp butterfly, warps in index
// order).  No barrier is needed when W = 32, so every warp streams
// independently with its next loads already in flight.
#include "common.cuh"
#include "launch.cuh"
#include "tma.cuh"

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
  // The inclusive masks as equalities: g <= L exactly when min(g, L) == g, and
  // -L <= u <= L exactly when the clamped u equals u (a NaN compares unequal on
  // both sides).  One compare per mask; measured 208.3 us against 209.9 with
  // the range compares (65536 x 2048 bf16, same bits).
  o.d_gate = (gc == g) ? (a * uc) * dsilu : 0.0f;
  o.d_up = (uc == u) ? a * s : 0.0f;
  o.t = dy * (s * uc);
  return o;
}

// ------------------------------------------------------------------ forward

#ifndef MOE_SWIGLU_FWD_MIN_BLOCKS
#define MOE_SWIGLU_FWD_MIN_BLOCKS 0
#endif
#if MOE_SWIGLU_FWD_MIN_BLOCKS > 0
#define MOE_SWIGLU_FWD_MIN_BLOCKS_ATTR __launch_bounds__(kThreads, MOE_SWIGLU_FWD_MIN_BLOCKS)
#else
#define MOE_SWIGLU_FWD_MIN_BLOCKS_ATTR __launch_bounds__(kThreads)
#endif

template <class D, int U>
__global__ void MOE_SWIGLU_FWD_MIN_BLOCKS_ATTR
swiglu_fwd_rows(const typename D::T* __restrict__ x, const float* __restrict__ probs,
                typename D::T* __restrict__ y, int64_t rows, int64_t inter, int64_t ld_x,
                int64_t ld_y, float L) {
  pdl_prologue();
  const int64_t cpr = inter / kVec;
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = (int64_t)gridDim.x * (kThreads / 32);
  const FwdMath f{L};
  for (int64_t r = (int64_t)blockIdx.x * (kThreads / 32) + (threadIdx.x >> 5); r < rows;
       r += nwarps) {
    const float p = __ldg(probs + r);
    const typename D::T* xr = x + r * ld_x;
    typename D::T* yr = y + r * ld_y;
    for (int64_t c0 = lane; c0 < cpr; c0 += 32 * U) {
      Raw8<D> gw[U], uw[U];
#pragma unroll
      for (int k = 0; k < U; ++k) {
        const int64_t c = c0 + 32 * k;
        if (c < cpr) {
          gw[k] = load8<D>(xr + c * kVec);
          uw[k] = load8<D>(xr + inter + c * kVec);
        }
      }
#pragma unroll
      for (int k = 0; k < U; ++k) {
        const int64_t c = c0 + 32 * k;
        if (c < cpr) {
          float g[8], u[8], o[8];
          widen8<D>(gw[k], g);
          widen8<D>(uw[k], u);
#pragma unroll
          for (int i = 0; i < 8; ++i) o[i] = f(g[i], u[i], p);
          store8<D>(yr + c * kVec, o);
        }
      }
    }
  }
}

// Errors recorded by the kernels of this file that wait on barriers (bits
// MOE_DEVERR_*), per device, when the caller gives no error word of its own;
// read and cleared by moe_device_errors().
__device__ int32_t g_device_errors;

constexpr int kTmaConsumers = 8;
constexpr int kTmaThreads = 32 * (kTmaConsumers + 1);
constexpr size_t kTmaSmemMax = 200 * 1024;

// TMA-staged forward.  Row k of the CTA (r = blockIdx.x + k * gridDim.x) goes
// to stage k % S and to consumer warp k % C; since C divides S, every stage is
// filled and emptied by one consumer in order, so a stage has at most one fill
// outstanding and the barrier parities are unambiguous.  full[s] completes a
// phase when the producer's arrival and the row's bytes are in; empty[s] when
// the consumer has read the row.  Every wait is bounded: a consumer's wait for
// its row and the producer's wait for a free stage give up after `wait_cycles`
// SM cycles; the waiting warp then ORs MOE_DEVERR_TIMEOUT into `err` (the
// caller's word, else g_device_errors) and stops, and the producer waits
// (bounded again, kWaitCycles) for every copy it issued before its CTA exits,
// so no copy is left in flight on the normal timeout path.
//
// STALL (tests of that failure path only): the producer neither arrives on
// nor copies into the stage of row `stall_row`, so that row's consumer waits
// for a phase that never completes and times out; nothing is left in flight
// (the drain skips the fill that was never issued).
template <class D, int S, bool STALL>
__global__ void __launch_bounds__(kTmaThreads, 1)
swiglu_fwd_tma(const typename D::T* __restrict__ x, const float* __restrict__ probs,
               typename D::T* __restrict__ y, int64_t rows, int64_t inter, int64_t ld_x,
               int64_t ld_y, float L, int32_t* err, long long wait_cycles, int64_t stall_row) {
  static_assert(S % kTmaConsumers == 0, "each stage must belong to one consumer warp");
  pdl_prologue();
  using T = typename D::T;
  extern __shared__ __align__(128) uint8_t smem[];
  int32_t* const errw = err ? err : &g_device_errors;
  const uint32_t stage_bytes = (uint32_t)(2 * inter * sizeof(T));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (size_t)S * stage_bytes);
  uint64_t* empty = full + S;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      tma::mbar_init(&full[s], 1);
      tma::mbar_init(&empty[s], 1);
    }
    tma::mbar_init_fence();
  }
  __syncthreads();
  const int64_t my_rows = rows > blockIdx.x ? (rows - 1 - blockIdx.x) / gridDim.x + 1 : 0;
  // the CTA-local index of the row that is never filled (STALL only)
  const int64_t k_stall = (STALL && stall_row >= 0 && stall_row % gridDim.x == blockIdx.x)
                              ? stall_row / gridDim.x : -1;
  if (warp == 0) {                                        // producer
    if (lane != 0) return;
    int64_t k = 0;
    for (; k < my_rows; ++k) {
      const int s = (int)(k % S);
      const uint32_t n = (uint32_t)(k / S);
      if (n > 0 && !tma::mbar_wait(&empty[s], (n - 1) & 1, wait_cycles)) {
        atomicOr(errw, MOE_DEVERR_TIMEOUT);
        break;
      }
      if (STALL && k == k_stall) continue;
      const int64_t r = blockIdx.x + k * gridDim.x;
      tma::mbar_arrive_expect_tx(&full[s], stage_bytes);
      tma::bulk_load(smem + (size_t)s * stage_bytes, x + r * ld_x, stage_bytes, &full[s]);
    }
    for (int s = 0; s < S && s < k; ++s) {                // drain every issued copy
      int64_t last = s + ((k - 1 - s) / S) * S;
      if (STALL && last == k_stall) last -= S;            // that fill was never issued
      if (last < 0) continue;
      if (!tma::mbar_wait(&full[s], (uint32_t)(last / S) & 1))
        atomicOr(errw, MOE_DEVERR_TIMEOUT);
    }
    return;
  }
  const int cw = warp - 1;                                // consumers
  const int64_t cpr = inter / kVec;
  const FwdMath f{L};
  for (int64_t k = cw; k < my_rows; k += kTmaConsumers) {
    const int s = (int)(k % S);
    // every lane polls; the warp gives up as one if any lane did (a phase that
    // completes just as the limit passes cannot split the warp)
    const bool ok = tma::mbar_wait(&full[s], (uint32_t)(k / S) & 1, wait_cycles);
    if (!__all_sync(0xffffffffu, ok)) {
      if (lane == 0) atomicOr(errw, MOE_DEVERR_TIMEOUT);
      return;
    }
    const int64_t r = blockIdx.x + k * gridDim.x;
    const float p = __ldg(probs + r);
    const T* st = reinterpret_cast<const T*>(smem + (size_t)s * stage_bytes);
    T* yr = y + r * ld_y;
    for (int64_t c = lane; c < cpr; c += 32) {
      float g[8], u[8], o[8];
      widen8<D>(tma::lds8<D>(st + c * kVec), g);
      widen8<D>(tma::lds8<D>(st + inter + c * kVec), u);
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = f(g[i], u[i], p);
      store8<D>(yr + c * kVec, o);
    }
    __syncwarp();                                          // every lane has read the stage
    if (lane == 0) tma::mbar_arrive(&empty[s]);
  }
}

// Stages of the TMA ring for rows of `inter` columns of T: 16, or 8 for
// longer rows, or 0 when even 8 do not fit.
#ifndef MOE_SWIGLU_FWD_STAGES
#define MOE_SWIGLU_FWD_STAGES 16
#endif
constexpr int kTmaStagesMax = MOE_SWIGLU_FWD_STAGES;   // 16 or 24
static_assert(kTmaStagesMax == 16 || kTmaStagesMax == 24, "16 or 24 ring stages");

template <class T>
int tma_stages(int64_t inter) {
  const size_t stage = (size_t)2 * inter * sizeof(T);
  if (kTmaStagesMax > 16 && kTmaStagesMax * stage + 16 * kTmaStagesMax <= kTmaSmemMax)
    return kTmaStagesMax;
  return 16 * stage + 256 <= kTmaSmemMax ? 16 : 8 * stage + 128 <= kTmaSmemMax ? 8 : 0;
}

// Launches the TMA-staged forward with `grid` CTAs (one per SM at most).
template <class D, bool STALL>
int launch_fwd_tma(const typename D::T* x, const float* probs, typename D::T* y, int64_t rows,
                   int64_t inter, int64_t ld_x, int64_t ld_y, float limit, int grid,
                   int32_t* err, long long wait_cycles, int64_t stall_row,
                   cudaStream_t stream) {
  using T = typename D::T;
  const int S = tma_stages<T>(inter);
  auto k = S == kTmaStagesMax ? swiglu_fwd_tma<D, kTmaStagesMax, STALL>
          : S == 16          ? swiglu_fwd_tma<D, 16, STALL>
                             : swiglu_fwd_tma<D, 8, STALL>;
  const size_t smem = (size_t)S * 2 * inter * sizeof(T) + 2 * (size_t)S * sizeof(uint64_t);
  if (int rc = ensure_smem_limit((const void*)k, kTmaSmemMax)) return rc;
  launch_kernel_block(k, grid, kTmaThreads, smem, stream, x, probs, y, rows, inter, ld_x, ld_y,
                      limit, err, wait_cycles, stall_row);
  return check_launch();
}

// Flat grid-stride forward over (row, chunk) pairs, for short rows.
template <class D, int U>
__global__ void __launch_bounds__(kThreads)
swiglu_fwd_vec(const typename D::T* __restrict__ x, const float* __restrict__ probs,
               typename D::T* __restrict__ y, int64_t rows, int64_t inter, int64_t ld_x,
               int64_t ld_y, float L) {
  pdl_prologue();
  const int64_t cpr = inter / kVec;
  const int64_t total = rows * cpr;
  const int64_t S = (int64_t)gridDim.x * kThreads;
  int64_t q = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  if (q >= total) return;
  RowCursor cur(q, S, cpr);
  const FwdMath f{L};
  for (; q < total; q += U * S) {
    Raw8<D> gw[U], uw[U];
    float p[U];
    typename D::T* dst[U];
#pragma unroll
    for (int k = 0; k < U; ++k) {
      if (q + k * S < total) {
        const typename D::T* src = x + cur.r * ld_x + cur.c * kVec;
        gw[k] = load8<D>(src);
        uw[k] = load8<D>(src + inter);
        p[k] = __ldg(probs + cur.r);
        dst[k] = y + cur.r * ld_y + cur.c * kVec;
      }
      cur.advance();
    }
#pragma unroll
    for (int k = 0; k < U; ++k) {
      if (q + k * S < total) {
        float g[8], u[8], o[8];
        widen8<D>(gw[k], g);
        widen8<D>(uw[k], u);
#pragma unroll
        for (int i = 0; i < 8; ++i) o[i] = f(g[i], u[i], p[k]);
        store8<D>(dst[k], o);
      }
    }
  }
}

// Element-granular forward: any inter, leading dimensions and alignment.
template <class D>
__global__ void __launch_bounds__(kThreads)
swiglu_fwd_scalar(const typename D::T* __restrict__ x, const float* __restrict__ probs,
                  typename D::T* __restrict__ y, int64_t rows, int64_t inter, int64_t ld_x,
                  int64_t ld_y, float L) {
  pdl_prologue();
  const int64_t total = rows * inter;
  const int64_t S = (int64_t)gridDim.x * kThreads;
  int64_t q = (int64_t)blockIdx.x * kThreads + threadIdx.x;
  if (q >= total) return;
  RowCursor cur(q, S, inter);
  const FwdMath f{L};
  for (; q < total; q += S, cur.advance()) {
    const typename D::T* src = x + cur.r * ld_x + cur.c;
    const float g = load1<D>(src), u = load1<D>(src + inter);
    store1<D>(y + cur.r * ld_y + cur.c, f(g, u, __ldg(probs + cur.r)));
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
#define MOE_SWIGLU_BWD_MIN_BLOCKS 0
#endif
#if MOE_SWIGLU_BWD_MIN_BLOCKS > 0
#define MOE_SWIGLU_BWD_MIN_BLOCKS_ATTR __launch_bounds__(kThreads, MOE_SWIGLU_BWD_MIN_BLOCKS)
#else
#define MOE_SWIGLU_BWD_MIN_BLOCKS_ATTR __launch_bounds__(kThreads)
#endif

// An 8-element chunk of D: one 16-byte access for the 16-bit types; two for
// fp32, or one 32-byte access when A32 (32-byte aligned fp32 rows).
template <class D, bool A32>
__device__ __forceinline__ Raw8<D> load_chunk(const typename D::T* p) {
  if constexpr (A32) {
    const u4x2 v = ld_stream32(p);
    Raw8<D> r;
    r.w[0] = v.lo;
    r.w[1] = v.hi;
    return r;
  } else {
    return load8<D>(p);
  }
}
template <class D, bool A32>
__device__ __forceinline__ void store_chunk(typename D::T* p, const float (&v)[8]) {
  if constexpr (A32) {
    st_stream32(p, make_uint4(__float_as_uint(v[0]), __float_as_uint(v[1]), __float_as_uint(v[2]),
                              __float_as_uint(v[3])),
                make_uint4(__float_as_uint(v[4]), __float_as_uint(v[5]), __float_as_uint(v[6]),
                           __float_as_uint(v[7])));
  } else {
    store8<D>(p, v);
  }
}

template <class D, int W, int U, bool A32 = false>
__global__ void MOE_SWIGLU_BWD_MIN_BLOCKS_ATTR
swiglu_bwd_vec(const typename D::T* __restrict__ x, const float* __restrict__ probs,
               const typename D::T* __restrict__ gy, typename D::T* __restrict__ gx,
               float* __restrict__ gp, int64_t rows, int64_t inter, int64_t ld_x,
               int64_t ld_gy, int64_t ld_gx, float L) {
  pdl_prologue();
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
      const typename D::T* xr = x + r * ld_x;
      const typename D::T* gyr = gy + r * ld_gy;
      typename D::T* gxr = gx + r * ld_gx;
      for (int64_t c0 = lane; c0 < cpr; c0 += (int64_t)U * W) {
        Raw8<D> gw[U], uw[U], dw[U];
#pragma unroll
        for (int k = 0; k < U; ++k) {
          const int64_t c = c0 + (int64_t)k * W;
          if (c < cpr) {
            gw[k] = load_chunk<D, A32>(xr + c * kVec);
            uw[k] = load_chunk<D, A32>(xr + inter + c * kVec);
            dw[k] = load_chunk<D, A32>(gyr + c * kVec);
          }
        }
#pragma unroll
        for (int k = 0; k < U; ++k) {
          const int64_t c = c0 + (int64_t)k * W;
          if (c < cpr) {
            float g[8], u[8], d[8], og[8], ou[8];
            widen8<D>(gw[k], g);
            widen8<D>(uw[k], u);
            widen8<D>(dw[k], d);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              const BwdOut o = bwd_math(g[i], u[i], d[i], p, L);
              og[i] = o.d_gate;
              ou[i] = o.d_up;
              acc += o.t;
            }
            store_chunk<D, A32>(gxr + c * kVec, og);
            store_chunk<D, A32>(gxr + inter + c * kVec, ou);
          }
        }
      }
    }
    const float s = row_reduce<W>(acc, red, parity);
    if (r < rows && lane == 0) gp[r] = s;
    parity ^= 1;
  }
}

template <class D, int W>
__global__ void __launch_bounds__(kThreads)
swiglu_bwd_scalar(const typename D::T* __restrict__ x, const float* __restrict__ probs,
                  const typename D::T* __restrict__ gy, typename D::T* __restrict__ gx,
                  float* __restrict__ gp, int64_t rows, int64_t inter, int64_t ld_x,
                  int64_t ld_gy, int64_t ld_gx, float L) {
  pdl_prologue();
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
        const float g = load1<D>(x + r * ld_x + j);
        const float u = load1<D>(x + r * ld_x + inter + j);
        const float d = load1<D>(gy + r * ld_gy + j);
        const BwdOut o = bwd_math(g, u, d, p, L);
        store1<D>(gx + r * ld_gx + j, o.d_gate);
        store1<D>(gx + r * ld_gx + inter + j, o.d_up);
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

// Tuning knobs (compile-time).  Unrolls are chunks whose loads a thread issues
// before it computes any of them, given for 16-bit types (fp32 chunks are twice
// the bytes and use half).  MOE_SWIGLU_BWD_ROW_THREADS: threads that own one
// row in the vectorised backward (0: as the element-wise path, the smallest of
// 32/64/128/256 covering the row); with the row length it fixes the grad_probs
// summation tree.
#ifndef MOE_SWIGLU_FWD_UNROLL
#define MOE_SWIGLU_FWD_UNROLL 2
#endif
#ifndef MOE_SWIGLU_FWD_TMA
#define MOE_SWIGLU_FWD_TMA 1
#endif
#ifndef MOE_SWIGLU_FWD_ROW_UNROLL
#define MOE_SWIGLU_FWD_ROW_UNROLL 8
#endif
#ifndef MOE_SWIGLU_BWD_ROW_THREADS
#define MOE_SWIGLU_BWD_ROW_THREADS 32
#endif
// fp32 rows that are 32-byte aligned take one 32-byte access per 8-element
// chunk, 4 chunks per lane in flight (141 registers, one CTA per SM).
// Measured on B200 at 65536 x 2048 fp32: 394.2 us against 457.2 with two
// 16-byte accesses per chunk (2 chunks per lane), 431.2-431.7 / 423.8-424.1
// with 2 / 3 chunks of 32 bytes.
#ifndef MOE_SWIGLU_BWD_F32_WIDE
#define MOE_SWIGLU_BWD_F32_WIDE 1
#endif
#ifndef MOE_SWIGLU_BWD_F32_UNROLL
#define MOE_SWIGLU_BWD_F32_UNROLL 4
#endif
#ifndef MOE_SWIGLU_BWD_UNROLL
#define MOE_SWIGLU_BWD_UNROLL 4
#endif
template <class D>
constexpr int unroll_for(int u16) { return D::kBytes == 4 ? (u16 + 1) / 2 : u16; }
constexpr int kBwdRowThreads = MOE_SWIGLU_BWD_ROW_THREADS;

template <class D>
int fwd(const void* xv, const float* probs, void* yv, int64_t rows, int64_t inter, int64_t ld_x,
        int64_t ld_y, float limit, int32_t* err, cudaStream_t stream) {
  using T = typename D::T;
  const T* x = static_cast<const T*>(xv);
  T* y = static_cast<T*>(yv);
  const bool vec = inter % kVec == 0 && ld_x % kVec == 0 && ld_y % kVec == 0 && aligned16(x) &&
                   aligned16(y);
  int grid;
  if (MOE_SWIGLU_FWD_TMA && vec && inter / kVec >= 64 && tma_stages<T>(inter) > 0) {
    int sms = 0;
    if (int rc = device_sm_count(&sms)) return rc;
    grid = (int)(rows < sms ? rows : sms);
    return launch_fwd_tma<D, false>(x, probs, y, rows, inter, ld_x, ld_y, limit, grid, err,
                                    tma::kWaitCycles, -1, stream);
  }
  if (vec && inter / kVec >= 64) {
    auto k = swiglu_fwd_rows<D, unroll_for<D>(MOE_SWIGLU_FWD_ROW_UNROLL)>;
    if (int rc = persistent_grid((const void*)k, 0, (rows + kThreads / 32 - 1) / (kThreads / 32),
                                 &grid))
      return rc;
    launch_kernel(k, grid, 0, stream, x, probs, y, rows, inter, ld_x, ld_y, limit);
  } else if (vec) {
    constexpr int U = unroll_for<D>(MOE_SWIGLU_FWD_UNROLL);
    auto k = swiglu_fwd_vec<D, U>;
    const int64_t units = rows * (inter / kVec);
    if (int rc = persistent_grid((const void*)k, 0, (units + kThreads * U - 1) / (kThreads * U),
                                 &grid))
      return rc;
    launch_kernel(k, grid, 0, stream, x, probs, y, rows, inter, ld_x, ld_y, limit);
  } else {
    auto k = swiglu_fwd_scalar<D>;
    if (int rc = persistent_grid((const void*)k, 0, (rows * inter + kThreads - 1) / kThreads,
                                 &grid))
      return rc;
    launch_kernel(k, grid, 0, stream, x, probs, y, rows, inter, ld_x, ld_y, limit);
  }
  return check_launch();
}

template <class K, class T>
int launch_bwd(K kernel, int W, cudaStream_t stream, const T* x, const float* probs, const T* gy,
               T* gx, float* gp, int64_t rows, int64_t inter, int64_t ld_x, int64_t ld_gy,
               int64_t ld_gx, float L) {
  int grid;
  const int64_t blocks = (rows + kThreads / W - 1) / (kThreads / W);
  if (int rc = persistent_grid((const void*)kernel, 0, blocks, &grid)) return rc;
  launch_kernel(kernel, grid, 0, stream, x, probs, gy, gx, gp, rows, inter, ld_x, ld_gy, ld_gx, L);
  return check_launch();
}

template <class D>
int bwd(const void* xv, const float* probs, const void* gyv, void* gxv, float* gp, int64_t rows,
        int64_t inter, int64_t ld_x, int64_t ld_gy, int64_t ld_gx, float limit,
        cudaStream_t stream) {
  using T = typename D::T;
  const T* x = static_cast<const T*>(xv);
  const T* gy = static_cast<const T*>(gyv);
  T* gx = static_cast<T*>(gxv);
  const bool vec = inter % kVec == 0 && ld_x % kVec == 0 && ld_gy % kVec == 0 &&
                   ld_gx % kVec == 0 && aligned16(x) && aligned16(gy) && aligned16(gx);
  const int W = (vec && kBwdRowThreads) ? kBwdRowThreads
                                        : threads_per_row(vec ? inter / kVec : inter);
  constexpr int U = unroll_for<D>(MOE_SWIGLU_BWD_UNROLL);
#define MOE_BWD_ARGS stream, x, probs, gy, gx, gp, rows, inter, ld_x, ld_gy, ld_gx, limit
  if constexpr (D::kBytes == 4) {
    const bool a32 = MOE_SWIGLU_BWD_F32_WIDE && vec && W == 32 && (inter * 4) % 32 == 0 &&
                     (ld_x * 4) % 32 == 0 && (ld_gy * 4) % 32 == 0 && (ld_gx * 4) % 32 == 0 &&
                     aligned32(x) && aligned32(gy) && aligned32(gx);
    if (a32) return launch_bwd(swiglu_bwd_vec<D, 32, MOE_SWIGLU_BWD_F32_UNROLL, true>, 32,
                               MOE_BWD_ARGS);
  }
  if (vec) {
    switch (W) {
      case 32: return launch_bwd(swiglu_bwd_vec<D, 32, U>, 32, MOE_BWD_ARGS);
      case 64: return launch_bwd(swiglu_bwd_vec<D, 64, U>, 64, MOE_BWD_ARGS);
      case 128: return launch_bwd(swiglu_bwd_vec<D, 128, U>, 128, MOE_BWD_ARGS);
      default: return launch_bwd(swiglu_bwd_vec<D, 256, U>, 256, MOE_BWD_ARGS);
    }
  }
  switch (W) {
    case 32: return launch_bwd(swiglu_bwd_scalar<D, 32>, 32, MOE_BWD_ARGS);
    case 64: return launch_bwd(swiglu_bwd_scalar<D, 64>, 64, MOE_BWD_ARGS);
    case 128: return launch_bwd(swiglu_bwd_scalar<D, 128>, 128, MOE_BWD_ARGS);
    default: return launch_bwd(swiglu_bwd_scalar<D, 256>, 256, MOE_BWD_ARGS);
  }
#undef MOE_BWD_ARGS
}

}  // namespace

int launch_swiglu_clamped_fwd(const void* x, const float* probs, void* y, int64_t rows,
                              int64_t inter, int64_t ld_x, int64_t ld_y, float limit,
                              moe_dtype dt, int32_t* dev_err, cudaStream_t stream) {
  switch (dt) {
    case MOE_BF16: return fwd<BF16>(x, probs, y, rows, inter, ld_x, ld_y, limit, dev_err, stream);
    case MOE_FP16: return fwd<F16>(x, probs, y, rows, inter, ld_x, ld_y, limit, dev_err, stream);
    default: return fwd<F32>(x, probs, y, rows, inter, ld_x, ld_y, limit, dev_err, stream);
  }
}

int tma_forward_applies(int64_t inter, moe_dtype dt) {
  if (inter % kVec != 0 || inter / kVec < 64) return 0;
  return dt == MOE_FP32 ? tma_stages<float>(inter) > 0 : tma_stages<uint16_t>(inter) > 0;
}

int launch_swiglu_fwd_stalled(const void* x, const float* probs, void* y, int64_t rows,
                              int64_t inter, float limit, moe_dtype dt, int grid,
                              int64_t stall_row, long long wait_cycles, int32_t* dev_err,
                              cudaStream_t stream) {
  if (dt == MOE_BF16)
    return launch_fwd_tma<BF16, true>(static_cast<const uint16_t*>(x), probs,
                                      static_cast<uint16_t*>(y), rows, inter, 2 * inter, inter,
                                      limit, grid, dev_err, wait_cycles, stall_row, stream);
  return launch_fwd_tma<F16, true>(static_cast<const uint16_t*>(x), probs,
                                   static_cast<uint16_t*>(y), rows, inter, 2 * inter, inter,
                                   limit, grid, dev_err, wait_cycles, stall_row, stream);
}

int launch_swiglu_clamped_bwd(const void* x, const float* probs, const void* grad_y,
                              void* grad_x, float* grad_probs, int64_t rows, int64_t inter,
                              int64_t ld_x, int64_t ld_gy, int64_t ld_gx, float limit,
                              moe_dtype dt, cudaStream_t stream) {
  switch (dt) {
    case MOE_BF16:
      return bwd<BF16>(x, probs, grad_y, grad_x, grad_probs, rows, inter, ld_x, ld_gy, ld_gx,
                       limit, stream);
    case MOE_FP16:
      return bwd<F16>(x, probs, grad_y, grad_x, grad_probs, rows, inter, ld_x, ld_gy, ld_gx,
                      limit, stream);
    default:
      return bwd<F32>(x, probs, grad_y, grad_x, grad_probs, rows, inter, ld_x, ld_gy, ld_gx,
                      limit, stream);
  }
}

}  // namespace moe

extern "C" int moe_device_errors(int32_t* bits, int clear) {
  if (!bits) return MOE_ERR_NULL;
  cudaError_t e = cudaMemcpyFromSymbol(bits, moe::g_device_errors, sizeof(int32_t));
  if (e != cudaSuccess) return moe::cuda_fail(e);
  if (clear) {
    const int32_t zero = 0;
    e = cudaMemcpyToSymbol(moe::g_device_errors, &zero, sizeof(int32_t));
    if (e != cudaSuccess) return moe::cuda_fail(e);
  }
  int32_t epc = 0;
  if (int rc = moe::ep_combine_device_errors(&epc, clear)) return rc;
  *bits |= epc;
  return MOE_OK;
}

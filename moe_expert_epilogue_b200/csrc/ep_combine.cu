// ep_combine.cu -- EP combine: every rank's token-local unpermute and the
// rank-order reduce-scatter of its results, in one kernel over peer memory
// (core.inference.moe.batch_invariant: _unpermute_tokens_in_expert_order_kernel
// followed by ordered_reduce_scatter_v).
//
// On the pages each rank q first unpermutes its own experts' outputs into a
// block of partial sums for the tokens of all ranks (in symmetric memory),
// and every rank then sums its own tokens' rows of those blocks in rank order.
// Here rank `rank` computes, for each of its tokens t (global row
// g = rank_token_offset[rank] + t), straight from every rank's expert rows:
//   for q = 0, 1, ..., world-1:
//     part_q = partial_dt( +0 + sum over q's local experts e ascending with
//                          inverse_maps[q][g, e] >= 0 of f32(expert_outputs[q][row, :]) )
//     acc    = (q == 0) ? part_q : acc + part_q                         (fp32)
//   out[t, :] = out_dt(acc)
// -- the bits of the two-step form, with no partial blocks written or read:
// each partial lives in registers, and the peers' expert rows and
// inverse-map rows are read once, directly (1-D bulk copies into shared
// memory in the TMA-staged kernel, plain loads in the register-staged ones;
// never with multicast).  The kernel never waits on another rank: the caller
// orders the launch after every rank's expert outputs are complete.
//
// Up to 64 (rank, local expert) pairs and rows of a multiple of 8 elements
// take the TMA-staged kernel (ep_combine_tma, below); otherwise the
// register-staged ones:
//
// One warp per item = (token, 1/split of the row).  For a group of up to 8
// ranks the warp loads the token's inverse-map rows of all of them at once
// (the first group of the next item is prefetched) and compacts them into one
// rank-ordered list of row pointers in shared memory, each entry tagged with
// the number of rank partials to close before it; then, per 16-byte unit of
// the row, it keeps 4 expert rows' loads in flight (8 in the kernel for more
// than 8 ranks or odd widths) and closes each rank's partial in rank order
// (ranks without rows contribute +0, as their partial block row would).
#include <type_traits>

#include "common.cuh"
#include "launch.cuh"
#include "tma.cuh"

namespace moe {
namespace {

constexpr int kMaxWorld = 64;    // ranks (their table entries live in shared memory)
constexpr int kGroupRanks = 8;   // ranks whose inverse-map rows a warp stages at once
constexpr int kMaxE = 64;        // local experts per rank (two inverse entries per lane)
constexpr int kRowsGroup = 4;    // expert rows in flight per unit (one-group kernel)
constexpr int kRowsInFlight = 8; // expert rows in flight per unit (general kernel)

// A unit of a row: 8 elements (16-byte loads) or 1 element.
template <class D, bool VEC> struct Unit;
template <class D> struct Unit<D, true> {
  static constexpr int V = kVec;
  using Raw = Raw8<D>;
  template <bool ALIGNED>
  __device__ __forceinline__ static Raw load(const typename D::T* p) {
    if constexpr (ALIGNED) {
      return load8<D>(p);
    } else {
      Raw r;                                           // element loads, same bits
      typename D::T* dst = reinterpret_cast<typename D::T*>(&r);
#pragma unroll
      for (int i = 0; i < kVec; ++i) dst[i] = p[i];
      return r;
    }
  }
  __device__ __forceinline__ static void widen(const Raw& r, float (&v)[kVec]) { widen8<D>(r, v); }
};
template <class D> struct Unit<D, false> {
  static constexpr int V = 1;
  struct Raw { float v; };
  template <bool ALIGNED>
  __device__ __forceinline__ static Raw load(const typename D::T* p) { return {load1<D>(p)}; }
  __device__ __forceinline__ static void widen(const Raw& r, float (&v)[1]) { v[0] = r.v; }
};

template <class DP, int V>
__device__ __forceinline__ void round_partial(float (&p)[V]) {
  if constexpr (V == 1) {
    p[0] = round_to<DP>(p[0]);
  } else {
#pragma unroll
    for (int i = 0; i < V; i += 2) round2<DP>(p[i], p[i + 1]);
  }
}

// Appends rank k's live inverse entries (one per lane; two with TWO) to the
// warp's list as row pointers, in expert order.  The first appended entry
// carries `gap`: how many open partials must be closed before it is added
// (the ranks from the open one up to k).  Returns the number appended.
template <class T, bool TWO>
__device__ __forceinline__ int append_rank(int32_t r0, int32_t r1, int64_t max_rows,
                                           const T* base, int64_t hidden, int gap,
                                           const T** ptrs, uint8_t* gaps, int32_t* err,
                                           int lane) {
  if (r0 >= max_rows) { flag_error(err, MOE_DEVERR_INVERSE); r0 = -1; }
  if (TWO && r1 >= max_rows) { flag_error(err, MOE_DEVERR_INVERSE); r1 = -1; }
  const unsigned below = (1u << lane) - 1u;
  const unsigned m0 = __ballot_sync(0xffffffffu, r0 >= 0);
  const unsigned m1 = TWO ? __ballot_sync(0xffffffffu, r1 >= 0) : 0u;
  if (r0 >= 0) {
    const int pos = __popc(m0 & below);
    ptrs[pos] = base + (int64_t)r0 * hidden;
    gaps[pos] = pos == 0 ? (uint8_t)gap : (uint8_t)0;
  }
  if (TWO && r1 >= 0) {
    const int pos = __popc(m0) + __popc(m1 & below);
    ptrs[pos] = base + (int64_t)r1 * hidden;
    gaps[pos] = pos == 0 ? (uint8_t)gap : (uint8_t)0;
  }
  return __popc(m0) + __popc(m1);
}

// Rounds the open partial to DP and folds it into acc in rank order (rank 0's
// partial is the sum's first term); the next rank's partial starts at +0.
template <class DP, int V>
__device__ __forceinline__ void close_partial(float (&part)[V], float (&acc)[V], bool first) {
  round_partial<DP, V>(part);
#pragma unroll
  for (int i = 0; i < V; ++i) {
    acc[i] = first ? part[i] : acc[i] + part[i];
    part[i] = 0.0f;
  }
}

// One unit of the row: the list's rows (ROWS loads in flight), each
// rank's partial closed in rank order, `trailing` closes after the last row.
template <class DI, class DP, bool VEC, bool ALIGNED, int ROWS = kRowsInFlight>
__device__ __forceinline__ void fold_unit(const typename DI::T* const* ptrs, const uint8_t* gaps,
                                          int F, int trailing, int q0, int64_t u,
                                          float (&acc)[Unit<DI, VEC>::V]) {
  using U = Unit<DI, VEC>;
  constexpr int V = U::V;
  float part[V];
#pragma unroll
  for (int i = 0; i < V; ++i) part[i] = 0.0f;
  int q = q0;                                           // global rank of the open partial
  for (int f0 = 0; f0 < F; f0 += ROWS) {
    typename U::Raw raw[ROWS];
#pragma unroll
    for (int j = 0; j < ROWS; ++j)
      if (f0 + j < F) raw[j] = U::template load<ALIGNED>(ptrs[f0 + j] + u * V);
#pragma unroll
    for (int j = 0; j < ROWS; ++j) {
      if (f0 + j < F) {
        for (int c = gaps[f0 + j]; c > 0; --c, ++q) close_partial<DP, V>(part, acc, q == 0);
        float v[V];
        U::widen(raw[j], v);
#pragma unroll
        for (int i = 0; i < V; ++i) part[i] = part[i] + v[i];
      }
    }
  }
  for (int c = trailing; c > 0; --c, ++q) close_partial<DP, V>(part, acc, q == 0);
}

// The token-local inverse-map rows of ranks q0 .. q0+nq-1 for global row g:
// one entry per lane (TWO: two, for more than 32 local experts).
template <bool TWO>
__device__ __forceinline__ void load_group(const int32_t* const* inv, int q0, int nq, int64_t g,
                                           int E, int lane, int32_t (&p0)[kGroupRanks],
                                           int32_t (&p1)[kGroupRanks]) {
#pragma unroll
  for (int k = 0; k < kGroupRanks; ++k) {
    p0[k] = -1;
    if (TWO) p1[k] = -1;
    if (k < nq) {
      const int32_t* r = inv[q0 + k] + g * E;
      p0[k] = lane < E ? __ldg(r + lane) : -1;
      if (TWO) p1[k] = lane + 32 < E ? __ldg(r + lane + 32) : -1;
    }
  }
}

// The rank-ordered row list of ranks q0 .. q0+nq-1 from their staged
// inverse-map entries; returns its length and, in `trailing`, the partials
// still to close after its last row.
template <class T, bool TWO>
__device__ __forceinline__ int build_list(const int32_t (&p0)[kGroupRanks],
                                          const int32_t (&p1)[kGroupRanks], int q0, int nq,
                                          int64_t max_rows, const T* const* eo, int64_t hidden,
                                          const T** ptrs, uint8_t* gaps, int32_t* err, int lane,
                                          int& trailing) {
  int F = 0, open = 0;                                   // open: the rank whose partial is open
#pragma unroll
  for (int k = 0; k < kGroupRanks; ++k) {
    if (k < nq) {
      const int c = append_rank<T, TWO>(p0[k], p1[k], max_rows, eo[q0 + k], hidden, k - open,
                                        ptrs + F, gaps + F, err, lane);
      if (c > 0) open = k;
      F += c;
    }
  }
  trailing = nq - open;
  return F;
}

// The warp's items -- (token, slice of the row) pairs, strided over the grid
// with a division-free cursor -- for up to 8 ranks (one group): the row list
// is built once per item, then the item's 16-byte units are folded and
// stored one after another.
template <class DI, class DP, class DO, bool TWO, bool ALIGNED, int ROWS>
__device__ __forceinline__ void combine_one_group(
    const typename DI::T* const* eo, const int32_t* const* inv, const typename DI::T** ptrs,
    uint8_t* gaps, int world, int64_t first, int64_t t_lo, int64_t t_hi, int split,
    int64_t units, int64_t hidden, int64_t max_rows, int E, typename DO::T* __restrict__ out,
    int32_t* err, int lane, int64_t it0, int64_t nwarps) {
  using T = typename DI::T;
  const int64_t n_tok = t_hi - t_lo;
  const int64_t upi = (units + split - 1) / split;
  RowCursor cur(it0, nwarps, split);
  if (cur.r >= n_tok) return;                             // warp-uniform
  int32_t p0[kGroupRanks], p1[kGroupRanks];
  load_group<TWO>(inv, 0, world, first + t_lo + cur.r, E, lane, p0, p1);
  while (cur.r < n_tok) {
    const int64_t t = t_lo + cur.r;
    const int64_t u0 = cur.c * upi;
    const int64_t u1 = min(units, u0 + upi);
    RowCursor nxt = cur;
    nxt.advance();
    __syncwarp();                                        // the previous list is consumed
    int trailing;
    const int F = build_list<T, TWO>(p0, p1, 0, world, max_rows, eo, hidden, ptrs, gaps, err,
                                     lane, trailing);
    __syncwarp();
    if (nxt.r < n_tok)                                   // next item's entries, in flight
      load_group<TWO>(inv, 0, world, first + t_lo + nxt.r, E, lane, p0, p1);
    for (int64_t u = u0 + lane; u < u1; u += 32) {
      float acc[kVec];
#pragma unroll
      for (int i = 0; i < kVec; ++i) acc[i] = 0.0f;
      fold_unit<DI, DP, true, ALIGNED, ROWS>(ptrs, gaps, F, trailing, 0, u, acc);
      store8<DO>(out + t * hidden + u * kVec, acc);
    }
    cur = nxt;
  }
}

// Any number of ranks and any row width / alignment: one unit per lane per
// item, each unit's sum carried across the groups of 8 ranks, ROWS expert
// rows' loads in flight per unit.
template <class DI, class DP, class DO, bool VEC, bool ALIGNED, int ROWS = kRowsInFlight>
__device__ __forceinline__ void combine_groups(
    const typename DI::T* const* eo, const int32_t* const* inv, const typename DI::T** ptrs,
    uint8_t* gaps, int world, int64_t first, int64_t t_lo, int64_t t_hi, int split,
    int64_t units, int64_t hidden, int64_t max_rows, int E, typename DO::T* __restrict__ out,
    int32_t* err, int lane, int64_t it0, int64_t nwarps) {
  using T = typename DI::T;
  constexpr int V = Unit<DI, VEC>::V;
  const int64_t n_tok = t_hi - t_lo;
  const int64_t upi = (units + split - 1) / split;       // <= 32 units: one per lane
  const int nq0 = world < kGroupRanks ? world : kGroupRanks;
  RowCursor cur(it0, nwarps, split);
  if (cur.r >= n_tok) return;                             // warp-uniform
  int32_t p0[kGroupRanks], p1[kGroupRanks];
  load_group<true>(inv, 0, nq0, first + t_lo + cur.r, E, lane, p0, p1);
  while (cur.r < n_tok) {
    const int64_t t = t_lo + cur.r;
    const int64_t g = first + t;
    const int64_t u = cur.c * upi + lane;
    const bool mine = u < min(units, cur.c * upi + upi);
    RowCursor nxt = cur;
    nxt.advance();
    float acc[V];
#pragma unroll
    for (int i = 0; i < V; ++i) acc[i] = 0.0f;
    for (int q0 = 0; q0 < world; q0 += kGroupRanks) {
      const int nq = world - q0 < kGroupRanks ? world - q0 : kGroupRanks;
      if (q0 > 0) load_group<true>(inv, q0, nq, g, E, lane, p0, p1);   // later groups
      __syncwarp();
      int trailing;
      const int F = build_list<T, true>(p0, p1, q0, nq, max_rows, eo, hidden, ptrs, gaps, err,
                                        lane, trailing);
      __syncwarp();
      if (q0 + kGroupRanks >= world && nxt.r < n_tok)
        load_group<true>(inv, 0, nq0, first + t_lo + nxt.r, E, lane, p0, p1);
      if (mine) fold_unit<DI, DP, VEC, ALIGNED, ROWS>(ptrs, gaps, F, trailing, q0, u, acc);
    }
    if (mine) {
      if constexpr (VEC) store8<DO>(out + t * hidden + u * kVec, acc);
      else store1<DO>(out + t * hidden + u, acc[0]);
    }
    cur = nxt;
  }
}

// Shared set-up of both kernels: the valid rows of this rank (as the
// reduce-scatter) and the world's table entries in shared memory.
struct CombineSetup {
  int64_t first, t_lo, t_hi;
  bool aligned;
};

template <class T>
__device__ __forceinline__ CombineSetup combine_setup(
    const void* const* eo_tab, const void* const* inv_tab, int world, int rank,
    const int32_t* offs, const int32_t* ep_tokens, int64_t capacity, int64_t local,
    const T** s_eo, const int32_t** s_inv, int32_t* err) {
  CombineSetup c;
  c.first = __ldg(offs + rank);
  const int64_t ep = __ldg(ep_tokens);
  const int64_t avail = ep < 0 ? 0 : (ep > capacity ? capacity : ep);
  c.t_lo = c.first < 0 ? -c.first : 0;
  c.t_hi = avail - c.first < local ? avail - c.first : local;
  if (c.t_lo > local) c.t_lo = local;
  if (c.t_hi < c.t_lo) c.t_hi = c.t_lo;
  if ((ep < 0 || ep > capacity || c.t_lo > 0 || c.t_hi < local) && blockIdx.x == 0 &&
      threadIdx.x == 0)
    flag_error(err, MOE_DEVERR_COUNT);
  int misaligned = 0;
  for (int q = threadIdx.x; q < world; q += blockDim.x) {
    s_eo[q] = static_cast<const T*>(eo_tab[q]);
    s_inv[q] = static_cast<const int32_t*>(inv_tab[q]);
    misaligned |= (int)(reinterpret_cast<uintptr_t>(eo_tab[q]) & 15);
  }
  c.aligned = __syncthreads_or(misaligned) == 0;
  return c;
}

#define MOE_EPC_PARAMS                                                                        \
  const void* const* __restrict__ eo_tab, const void* const* __restrict__ inv_tab, int world, \
      int rank, const int32_t* __restrict__ offs, const int32_t* __restrict__ ep_tokens,      \
      int64_t capacity, int64_t max_rows, int E, typename DO::T* __restrict__ out,            \
      int64_t local, int64_t hidden, int split, int32_t* err

// Up to 8 ranks, 16-byte units (hidden % 8 == 0, out aligned); 4 expert rows
// in flight per unit keep it at 80 registers, 3 CTAs per SM (8 rows: 104
// registers, 2 CTAs, slower except on the shortest launches).
template <class DI, class DP, class DO, bool TWO>
__global__ void __launch_bounds__(kThreads)
ep_combine_group(MOE_EPC_PARAMS) {
  using TI = typename DI::T;
  __shared__ const TI* s_eo[kMaxWorld];
  __shared__ const int32_t* s_inv[kMaxWorld];
  __shared__ const TI* s_ptrs[kThreads / 32][kGroupRanks * kMaxE];
  __shared__ uint8_t s_gaps[kThreads / 32][kGroupRanks * kMaxE];
  pdl_prologue();
  const CombineSetup c = combine_setup<TI>(eo_tab, inv_tab, world, rank, offs, ep_tokens,
                                           capacity, local, s_eo, s_inv, err);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t it0 = (int64_t)blockIdx.x * (kThreads / 32) + warp;
  const int64_t nwarps = (int64_t)gridDim.x * (kThreads / 32);
  if (c.aligned)
    combine_one_group<DI, DP, DO, TWO, true, kRowsGroup>(
        s_eo, s_inv, s_ptrs[warp], s_gaps[warp], world, c.first, c.t_lo, c.t_hi, split,
        hidden / kVec, hidden, max_rows, E, out, err, lane, it0, nwarps);
  else                                                   // a buffer off 16-byte alignment
    combine_one_group<DI, DP, DO, TWO, false, kRowsGroup>(
        s_eo, s_inv, s_ptrs[warp], s_gaps[warp], world, c.first, c.t_lo, c.t_hi, split,
        hidden / kVec, hidden, max_rows, E, out, err, lane, it0, nwarps);
}

// Any number of ranks, any width and alignment.
template <class DI, class DP, class DO, bool VEC>
__global__ void __launch_bounds__(kThreads)
ep_combine_groups(MOE_EPC_PARAMS) {
  using TI = typename DI::T;
  constexpr int V = Unit<DI, VEC>::V;
  __shared__ const TI* s_eo[kMaxWorld];
  __shared__ const int32_t* s_inv[kMaxWorld];
  __shared__ const TI* s_ptrs[kThreads / 32][kGroupRanks * kMaxE];
  __shared__ uint8_t s_gaps[kThreads / 32][kGroupRanks * kMaxE];
  pdl_prologue();
  const CombineSetup c = combine_setup<TI>(eo_tab, inv_tab, world, rank, offs, ep_tokens,
                                           capacity, local, s_eo, s_inv, err);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t it0 = (int64_t)blockIdx.x * (kThreads / 32) + warp;
  const int64_t nwarps = (int64_t)gridDim.x * (kThreads / 32);
  if (!VEC || c.aligned)
    combine_groups<DI, DP, DO, VEC, true>(s_eo, s_inv, s_ptrs[warp], s_gaps[warp], world,
                                          c.first, c.t_lo, c.t_hi, split, hidden / V, hidden,
                                          max_rows, E, out, err, lane, it0, nwarps);
  else
    combine_groups<DI, DP, DO, VEC, false>(s_eo, s_inv, s_ptrs[warp], s_gaps[warp], world,
                                           c.first, c.t_lo, c.t_hi, split, hidden / V, hidden,
                                           max_rows, E, out, err, lane, it0, nwarps);
}
#undef MOE_EPC_PARAMS

// ------------------------------------------------------------------------
// TMA-staged EP combine (up to 32 * kTmaBatches (rank, local expert) pairs,
// hidden % 8 == 0): one CTA per SM, one producer warp and kTmaWarps consumer
// warps around a ring of shared-memory stages of up to R expert-row chunks.
//
// Work items are (token, chunk of up to kChunkUnits 8-element units of the
// row, at most kRowBytes); each CTA takes a contiguous range of them, so the
// chunks of one token follow each other and share its row list.  The producer
// loads the token's inverse-map entries of all ranks (the next token's are in
// flight while it works) and compacts them into the rank-ordered list of
// (rank, row) pairs with the partial-close counts; the item's rows go to
// ceil(F / R) consecutive stages, and producer lane j fills the item's j-th
// stage: waits for it to be free, writes its header (item, rows, closes before
// each row, first / last stage of the item) and issues one 1-D bulk copy
// (cp.async.bulk, no multicast) per row chunk.  Consumer thread u folds unit
// u of every row of a stage as it lands, in list order, closes each rank's
// partial in rank order (rounded to DP), and stores the item's unit after its
// last stage.  The expert rows are read once, by the copy engine, with up to
// a ring of row chunks (~190 KB) in flight per SM.
//
// Barriers: full[s] completes when the producer's arrival and the stage's
// bytes are in; empty[s] when the kTmaWarps consumer warps have read it.  Every
// wait is bounded: a timeout sets MOE_DEVERR_TIMEOUT and ends the warp; the
// producer drains every copy it issued before its CTA exits.  The producer
// ends the stream with a header marked `done`.
//
// If an expert-output base is not 16-byte aligned (no bulk copy can read it),
// every warp of the CTA runs the general register-staged combine instead,
// with 2 rows' loads in flight (it shares the kernel's register budget).

// Timeouts of the TMA-staged kernel for calls given no error word (per
// device; moe_device_errors() reads it with the forward SwiGLU's word).
__device__ int32_t g_epc_errors;

constexpr int kTmaWarps = 16;                       // consumer warps
constexpr int kTmaEpcThreads = 32 * (kTmaWarps + 1);
constexpr int kChunkUnits = 32 * kTmaWarps;         // at most one unit per consumer thread
constexpr int kRowBytes = 8192;                     // at most this much of a row per copy
constexpr int kMaxStages = 32;
constexpr int kTmaBatches = 2;                      // inverse entries per producer lane
#ifndef MOE_EPC_SMEM_KB
#define MOE_EPC_SMEM_KB 200
#endif
constexpr size_t kEpcSmemMax = (size_t)MOE_EPC_SMEM_KB * 1024;

enum : uint8_t { kFirst = 1, kLast = 2, kDone = 4 };

struct __align__(16) StageHeader {
  int64_t t;                    // token row of the output
  int64_t col;                  // first column of the chunk
  uint64_t gaps;                // byte j: partials to close before row j
  uint8_t rows;                 // rows in this stage
  uint8_t flags;                // kFirst / kLast (of the item) / kDone
  uint8_t trailing;             // partials to close after the item's last row (kLast)
  uint8_t pad[5];
};
static_assert(sizeof(StageHeader) == 32, "stage header layout");

// Dynamic shared memory of the kernel: the ring, the headers, the barriers
// and the producer's row list, in that order.
struct EpcSmem {
  size_t headers, bars, list_rows, list_q, list_gaps, total;
  __host__ __device__ EpcSmem(int stages, size_t stage_bytes) {
    headers = (size_t)stages * stage_bytes;
    bars = headers + (size_t)stages * sizeof(StageHeader);
    list_rows = bars + (size_t)2 * stages * sizeof(uint64_t);
    list_q = list_rows + (size_t)32 * kTmaBatches * sizeof(int32_t);
    list_gaps = list_q + (size_t)32 * kTmaBatches;
    total = list_gaps + (size_t)32 * kTmaBatches + 8;    // 8: the last 64-bit gap read
  }
};

// Compacts the token's entries (lane entry b is the flattened pair
// f = 32 b + lane, rank q[b]) into the list -- rank order, then expert order --
// with each row's partial-close count; returns the list length, and in
// `trailing` the partials left to close after its last row.
__device__ __forceinline__ int build_tma_list(const int32_t (&ent)[kTmaBatches],
                                              const int (&q)[kTmaBatches], int world,
                                              int64_t max_rows, int32_t* rows, uint8_t* qs,
                                              uint8_t* gaps, int32_t* err, int lane,
                                              int& trailing) {
  const unsigned below = (1u << lane) - 1u;
  int F = 0, carry_q = 0;                      // carry_q: rank of the last listed row
#pragma unroll
  for (int b = 0; b < kTmaBatches; ++b) {
    int32_t r = ent[b];
    if (r >= max_rows) { flag_error(err, MOE_DEVERR_INVERSE); r = -1; }
    const unsigned m = __ballot_sync(0xffffffffu, r >= 0);
    const unsigned pm = m & below;
    const int q_prev = __shfl_sync(0xffffffffu, q[b], pm ? 31 - __clz(pm) : 0);
    if (r >= 0) {
      const int pos = F + __popc(pm);
      rows[pos] = r;
      qs[pos] = (uint8_t)q[b];
      gaps[pos] = (uint8_t)(q[b] - (pm ? q_prev : carry_q));
    }
    if (m) carry_q = __shfl_sync(0xffffffffu, q[b], 31 - __clz(m));
    F += __popc(m);
  }
  trailing = world - carry_q;
  __syncwarp();
  return F;
}

// Row folds: fold_first, p = v + 0 (a partial's first row: +0 + v, which
// turns a -0 row into +0 as the definition's +0 start does); fold_add,
// p = p + v.
template <class D, bool FIRST>
__device__ __forceinline__ void fold_row(float (&p)[kVec], const Raw8<D>& r) {
  float v[kVec];
  widen8<D>(r, v);
#pragma unroll
  for (int i = 0; i < kVec; ++i) p[i] = FIRST ? v[i] + 0.0f : p[i] + v[i];
}

// Closes the open rank partial (n rows since it opened) into the rank-order
// sum: acc += round_DP(part).  acc starts at -0, the identity of fp32
// addition (-0 + x == x for every x, +0 and -0 included), so the first rank's
// close leaves exactly its partial, as the definition's first term.  A partial
// of fewer than two rows is +0 or +0 + v with v a value of the input dtype,
// which DP (the input dtype or fp32) represents exactly: it is not rounded.
// `empties` ranks without rows follow it: each adds +0, and since
// (acc + 0) + 0 == acc + 0 they collapse into one add.  The branches are
// uniform across the warp (every thread walks the same rows).
template <class DP>
__device__ __forceinline__ void close_rank(float (&part)[kVec], float (&acc)[kVec], int n,
                                           bool empties) {
  if (DP::kBytes == 2 && n >= 2) round_partial<DP, kVec>(part);
#pragma unroll
  for (int i = 0; i < kVec; ++i) acc[i] = acc[i] + part[i];
  if (empties) {
#pragma unroll
    for (int i = 0; i < kVec; ++i) acc[i] = acc[i] + 0.0f;
  }
}

template <class DI, class DP, class DO, int R>
__global__ void __launch_bounds__(kTmaEpcThreads, 1)
ep_combine_tma(const void* const* __restrict__ eo_tab, const void* const* __restrict__ inv_tab,
               int world, int rank, const int32_t* __restrict__ offs,
               const int32_t* __restrict__ ep_tokens, int64_t capacity, int64_t max_rows, int E,
               typename DO::T* __restrict__ out, int64_t local, int64_t hidden, int64_t chunk,
               int stages, int32_t* err) {
  static_assert(R >= 1 && R <= 8, "a stage header holds up to 8 closes");
  using TI = typename DI::T;
  __shared__ const TI* s_eo[kMaxWorld];
  __shared__ const int32_t* s_inv[kMaxWorld];
  extern __shared__ __align__(128) uint8_t smem[];
  pdl_prologue();
  const CombineSetup c = combine_setup<TI>(eo_tab, inv_tab, world, rank, offs, ep_tokens,
                                           capacity, local, s_eo, s_inv, err);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int32_t* const errw = err ? err : &g_epc_errors;
  if (!c.aligned) {                                     // no bulk copy can read a base
    const TI** ptrs = reinterpret_cast<const TI**>(smem) + (size_t)warp * kGroupRanks * kMaxE;
    uint8_t* gaps = smem + (size_t)(kTmaWarps + 1) * kGroupRanks * kMaxE * sizeof(void*) +
                    (size_t)warp * kGroupRanks * kMaxE;
    const int64_t units = hidden / kVec;
    const int64_t split = (units + 31) / 32;
    combine_groups<DI, DP, DO, true, false, 2>(
        s_eo, s_inv, ptrs, gaps, world, c.first, c.t_lo, c.t_hi, (int)split, units, hidden,
        max_rows, E, out, err, lane, (int64_t)blockIdx.x * (kTmaWarps + 1) + warp,
        (int64_t)gridDim.x * (kTmaWarps + 1));
    return;
  }
  const size_t row_bytes = (size_t)chunk * sizeof(TI);
  const size_t stage_bytes = (size_t)R * row_bytes;
  const EpcSmem lay(stages, stage_bytes);
  StageHeader* hdr = reinterpret_cast<StageHeader*>(smem + lay.headers);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + lay.bars);
  uint64_t* empty = full + stages;
  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      tma::mbar_init(&full[s], 1);
      tma::mbar_init(&empty[s], kTmaWarps);
    }
    tma::mbar_init_fence();
  }
  __syncthreads();
  const int64_t split = (hidden + chunk - 1) / chunk;
  const int64_t n_items = (c.t_hi - c.t_lo) * split;
  const int64_t lo = n_items * blockIdx.x / gridDim.x;
  const int64_t hi = n_items * (blockIdx.x + 1) / gridDim.x;

  if (warp == 0) {                                      // producer
    int32_t* l_rows = reinterpret_cast<int32_t*>(smem + lay.list_rows);
    uint8_t* l_q = smem + lay.list_q;
    uint8_t* l_gaps = smem + lay.list_gaps;
    // this lane's (rank, local expert) pairs, fixed for the whole launch
    int qb[kTmaBatches];
    const int32_t* pb[kTmaBatches];
#pragma unroll
    for (int b = 0; b < kTmaBatches; ++b) {
      const int f = 32 * b + lane;
      qb[b] = f < world * E ? f / E : world;
      pb[b] = f < world * E ? s_inv[qb[b]] + f % E : nullptr;
    }
    int32_t ent[kTmaBatches];
#pragma unroll
    for (int b = 0; b < kTmaBatches; ++b) {
      const int64_t g = c.first + c.t_lo + lo / split;
      ent[b] = pb[b] && lo < hi ? __ldg(pb[b] + g * E) : -1;
    }
    const int64_t last_t = c.t_lo + (hi - 1) / split;
    const int per_round = stages < 32 ? stages : 32;   // lanes filling distinct stages at once
    uint32_t k = 0;                                     // stages filled so far
    bool failed = false;
    int F = 0, trailing = 0;
    int64_t t = c.t_lo + lo / split, ci = lo % split;
    for (int64_t item = lo; item < hi && !failed; ++item) {
      if (item == lo || ci == 0) {                     // a new token: its row list
        F = build_tma_list(ent, qb, world, max_rows, l_rows, l_q, l_gaps, err, lane, trailing);
        if (t < last_t) {                              // the next token's entries, in flight
#pragma unroll
          for (int b = 0; b < kTmaBatches; ++b)
            ent[b] = pb[b] ? __ldg(pb[b] + (c.first + t + 1) * E) : -1;
        }
      }
      const int64_t col = ci * chunk;
      const uint32_t bytes = (uint32_t)((hidden - col < chunk ? hidden - col : chunk) *
                                        (int64_t)sizeof(TI));
      const int nst = F > 0 ? (F + R - 1) / R : 1;     // stages of this item
      for (int j0 = 0; j0 < nst && !failed; j0 += per_round) {
        const int cnt = nst - j0 < per_round ? nst - j0 : per_round;
        const int j = j0 + lane;                        // this lane's stage of the item
        const uint32_t kk = k + lane;
        const int s = (int)(kk % stages);
        bool ok = true;
        if (lane < cnt && kk >= (uint32_t)stages)       // wait until the stage is free
          ok = tma::mbar_wait(&empty[s], (kk / stages - 1) & 1);
        if (!__all_sync(0xffffffffu, ok)) {
          if (lane == 0) atomicOr(errw, MOE_DEVERR_TIMEOUT);
          failed = true;
          break;
        }
        if (lane < cnt) {
          const int r0 = j * R;
          const int nr = F - r0 < R ? F - r0 : R;       // <= 0 only for a row-less item
          StageHeader& h = hdr[s];
          uint64_t g8 = 0;
          for (int i = 0; i < nr; ++i) g8 |= (uint64_t)l_gaps[r0 + i] << (8 * i);
          h.t = t;
          h.col = col;
          h.gaps = g8;
          h.rows = (uint8_t)(nr > 0 ? nr : 0);
          h.flags = (uint8_t)((j == 0 ? kFirst : 0) | (j == nst - 1 ? kLast : 0));
          h.trailing = (uint8_t)trailing;
          if (nr > 0) {
            tma::mbar_arrive_expect_tx(&full[s], (uint32_t)nr * bytes);
            for (int i = 0; i < nr; ++i) {
              const TI* src = s_eo[l_q[r0 + i]] + (int64_t)l_rows[r0 + i] * hidden + col;
              tma::bulk_load(smem + (size_t)s * stage_bytes + (size_t)i * row_bytes, src, bytes,
                             &full[s]);
            }
          } else {
            tma::mbar_arrive(&full[s]);
          }
        }
        k += (uint32_t)cnt;
      }
      __syncwarp();                                    // the list is read before it changes
      if (++ci == split) { ci = 0; ++t; }
    }
    if (!failed) {                                     // end of stream
      const int s = (int)(k % stages);
      bool ok = true;
      if (lane == 0 && k >= (uint32_t)stages) ok = tma::mbar_wait(&empty[s], (k / stages - 1) & 1);
      if (lane == 0) {
        if (ok) {
          hdr[s].flags = kDone;
          tma::mbar_arrive(&full[s]);
          ++k;
        } else {
          atomicOr(errw, MOE_DEVERR_TIMEOUT);
        }
      }
      k = __shfl_sync(0xffffffffu, k, 0);
    }
    if (lane == 0) {                                   // drain: every issued fill has landed
      for (int s = 0; s < stages && (uint32_t)s < k; ++s) {
        const uint32_t last = s + ((k - 1 - s) / stages) * stages;
        if (!tma::mbar_wait(&full[s], (last / stages) & 1)) atomicOr(errw, MOE_DEVERR_TIMEOUT);
      }
    }
    return;
  }

  // consumers: thread u folds unit u of every row of a stage as it lands
  const int u = threadIdx.x - 32;
  const int64_t width0 = hidden < chunk ? hidden : chunk;
  const bool act_any = (int64_t)u * kVec < width0;
  float acc[kVec] = {}, part[kVec] = {};
  int n = 0;                                           // rows in the open partial
  int s = 0;
  uint32_t phase = 0;
  for (;;) {
    const bool ok = tma::mbar_wait(&full[s], phase);
    if (!__all_sync(0xffffffffu, ok)) {
      if (lane == 0) atomicOr(errw, MOE_DEVERR_TIMEOUT);
      return;
    }
    const StageHeader& h = hdr[s];
    const uint8_t flags = h.flags;
    if (flags & kDone) return;
    if (act_any) {
      const int64_t col = h.col;
      if (flags & kFirst) {                            // a new item: -0 sum, +0 partial
#pragma unroll
        for (int i = 0; i < kVec; ++i) {
          acc[i] = -0.0f;
          part[i] = 0.0f;
        }
        n = 0;
      }
      const bool mine = (int64_t)u * kVec < (hidden - col < chunk ? hidden - col : chunk);
      const int nr = h.rows;
      uint64_t gaps = h.gaps;
      const TI* st = reinterpret_cast<const TI*>(smem + (size_t)s * stage_bytes) +
                     (size_t)u * kVec;
      Raw8<DI> raw[R];
#pragma unroll
      for (int i = 0; i < R; ++i)
        if (i < nr && mine) raw[i] = tma::lds8<DI>(st + (size_t)i * chunk);
#pragma unroll
      for (int i = 0; i < R; ++i) {
        if (i < nr) {
          const int g = (int)(gaps & 0xffu);
          gaps >>= 8;
          if (g > 0) {                                 // the row opens a rank
            close_rank<DP>(part, acc, n, g > 1);
            fold_row<DI, true>(part, raw[i]);
            n = 1;
          } else {
            fold_row<DI, false>(part, raw[i]);
            ++n;
          }
        }
      }
      if (flags & kLast) {
        close_rank<DP>(part, acc, n, h.trailing > 1);  // the open rank, then empties
        if (mine) store8<DO>(out + h.t * hidden + col + (int64_t)u * kVec, acc);
      }
    }
    __syncwarp();                                      // the warp has read the stage
    if (lane == 0) tma::mbar_arrive(&empty[s]);
    if (++s == stages) {
      s = 0;
      phase ^= 1u;
    }
  }
}

#ifndef MOE_EPC_TMA
#define MOE_EPC_TMA 1
#endif

#ifndef MOE_EPC_STAGE_ROWS
#define MOE_EPC_STAGE_ROWS 4
#endif

template <class DI, class DP, class DO>
int launch_tma(const void* const* eos, const void* const* invs, int world, int rank,
               const int32_t* offs, const int32_t* ep_tokens, int64_t capacity, int64_t max_rows,
               int E, void* out, int64_t local, int64_t hidden, int32_t* err,
               cudaStream_t stream) {
  using TI = typename DI::T;
  constexpr int R = MOE_EPC_STAGE_ROWS;
  // row chunks of at most kRowBytes (and one unit per consumer thread)
  int64_t units = hidden / kVec;
  if (units > kChunkUnits) units = kChunkUnits;
  if (units * kVec * (int64_t)sizeof(TI) > kRowBytes) units = kRowBytes / (kVec * sizeof(TI));
  const int64_t chunk = units * kVec;
  const size_t stage_bytes = (size_t)R * chunk * sizeof(TI);
  int stages = kMaxStages;
  while (stages >= 3 && EpcSmem(stages, stage_bytes).total > kEpcSmemMax) --stages;
  if (stages < 3) return -1;
  // the misaligned-base path carves per-warp row lists out of the same memory
  const size_t lists = (size_t)(kTmaWarps + 1) * kGroupRanks * kMaxE * (sizeof(void*) + 1);
  size_t smem = EpcSmem(stages, stage_bytes).total;
  if (smem < lists) smem = lists;
  auto k = ep_combine_tma<DI, DP, DO, R>;
  if (int rc = ensure_smem_limit((const void*)k, kEpcSmemMax)) return rc;
  int sms = 0;
  if (int rc = device_sm_count(&sms)) return rc;
  const int64_t items = local * ((hidden + chunk - 1) / chunk);
  const int grid = (int)(items < sms ? items : sms);
  launch_kernel_block(k, grid, kTmaEpcThreads, smem, stream, eos, invs, world, rank, offs,
                      ep_tokens, capacity, max_rows, E, static_cast<typename DO::T*>(out), local,
                      hidden, chunk, stages, err);
  return check_launch();
}

template <class DI, class DP, class DO>
int launch(const void* const* eos, const void* const* invs, int world, int rank,
           const int32_t* offs, const int32_t* ep_tokens, int64_t capacity, int64_t max_rows,
           int E, void* out, int64_t local, int64_t hidden, int32_t* err, cudaStream_t stream) {
  using TO = typename DO::T;
  const bool vec = hidden % kVec == 0 && aligned16(out);
  if (MOE_EPC_TMA && vec && world * E <= 32 * kTmaBatches) {
    const int rc = launch_tma<DI, DP, DO>(eos, invs, world, rank, offs, ep_tokens, capacity,
                                          max_rows, E, out, local, hidden, err, stream);
    if (rc >= 0) return rc;
  }
  const bool one_group = vec && world <= kGroupRanks;
  const int64_t units = vec ? hidden / kVec : hidden;
  int sms = 0;
  if (int rc = device_sm_count(&sms)) return rc;
  // Units per item: one per lane across groups of ranks.  With one group, 4
  // per lane once there are at least two items per resident warp (3 CTAs of
  // 8 warps per SM), else 2, so that short launches still spread over the
  // GPU.  Measured on B200, 8 ranks x 8 experts, top-8, hidden 4096, 4 rows in
  // flight: 1024 tokens a rank 203.5 us (2 per lane) against 225.6 (4);
  // 4096 tokens a rank 598.8 (4) against 614.6 (2) and 763.3 for the earlier
  // 8 rows in flight x 8 per lane.
  int per_lane = 1;
  if (one_group) {
    const int64_t items4 = local * ((units + 32 * 4 - 1) / (32 * 4));
    per_lane = items4 >= 2 * (int64_t)sms * 24 ? 4 : 2;
  }
  const int64_t per_item = 32 * (int64_t)per_lane;
  const int64_t split64 = (units + per_item - 1) / per_item;
  const int split = (int)(split64 < 1 ? 1 : split64);
  const int64_t warps = local * split;
  const void* k;
  if (one_group)
    k = E > 32 ? (const void*)ep_combine_group<DI, DP, DO, true>
               : (const void*)ep_combine_group<DI, DP, DO, false>;
  else
    k = vec ? (const void*)ep_combine_groups<DI, DP, DO, true>
            : (const void*)ep_combine_groups<DI, DP, DO, false>;
  int grid;
  if (int rc = persistent_grid(k, 0, (warps + kThreads / 32 - 1) / (kThreads / 32), &grid))
    return rc;
#define MOE_EPC_LAUNCH(KERNEL)                                                                 \
  launch_kernel(KERNEL, grid, 0, stream, eos, invs, world, rank, offs, ep_tokens, capacity,    \
                max_rows, E, static_cast<TO*>(out), local, hidden, split, err)
  if (one_group) {
    if (E > 32) MOE_EPC_LAUNCH((ep_combine_group<DI, DP, DO, true>));
    else MOE_EPC_LAUNCH((ep_combine_group<DI, DP, DO, false>));
  } else if (vec) {
    MOE_EPC_LAUNCH((ep_combine_groups<DI, DP, DO, true>));
  } else {
    MOE_EPC_LAUNCH((ep_combine_groups<DI, DP, DO, false>));
  }
#undef MOE_EPC_LAUNCH
  return check_launch();
}

// partial_dt and out_dt are each either the expert outputs' dtype or fp32
template <class DI>
int dispatch(moe_dtype partial_dt, moe_dtype out_dt, const void* const* eos,
             const void* const* invs, int world, int rank, const int32_t* offs,
             const int32_t* ep_tokens, int64_t capacity, int64_t max_rows, int E, void* out,
             int64_t local, int64_t hidden, int32_t* err, cudaStream_t stream) {
  const bool p32 = partial_dt == MOE_FP32, o32 = out_dt == MOE_FP32;
#define MOE_EPC_ARGS eos, invs, world, rank, offs, ep_tokens, capacity, max_rows, E, out, local, \
                     hidden, err, stream
  if (p32 && o32) return launch<DI, F32, F32>(MOE_EPC_ARGS);
  if (p32) return launch<DI, F32, DI>(MOE_EPC_ARGS);
  if (o32) return launch<DI, DI, F32>(MOE_EPC_ARGS);
  return launch<DI, DI, DI>(MOE_EPC_ARGS);
#undef MOE_EPC_ARGS
}

}  // namespace

int max_ep_combine_world() { return kMaxWorld; }

int ep_combine_device_errors(int32_t* bits, int clear) {
  cudaError_t e = cudaMemcpyFromSymbol(bits, g_epc_errors, sizeof(int32_t));
  if (e != cudaSuccess) return cuda_fail(e);
  if (clear) {
    const int32_t zero = 0;
    e = cudaMemcpyToSymbol(g_epc_errors, &zero, sizeof(int32_t));
    if (e != cudaSuccess) return cuda_fail(e);
  }
  return MOE_OK;
}
int max_ep_combine_experts() { return kMaxE; }

int launch_unpermute_reduce_scatter(const void* const* expert_outputs, moe_dtype eo_dt,
                                    int64_t max_rows, const void* const* inverse_maps,
                                    int num_local_experts, int64_t capacity_rows,
                                    const int32_t* ep_tokens, int world, int rank,
                                    const int32_t* rank_token_offset, moe_dtype partial_dt,
                                    void* out, moe_dtype out_dt, int64_t local_tokens,
                                    int64_t hidden, int32_t* err, cudaStream_t stream) {
#define MOE_EPC_ARGS partial_dt, out_dt, expert_outputs, inverse_maps, world, rank, \
                     rank_token_offset, ep_tokens, capacity_rows, max_rows, num_local_experts, \
                     out, local_tokens, hidden, err, stream
  switch (eo_dt) {
    case MOE_BF16: return dispatch<BF16>(MOE_EPC_ARGS);
    case MOE_FP16: return dispatch<F16>(MOE_EPC_ARGS);
    default: return dispatch<F32>(MOE_EPC_ARGS);
  }
#undef MOE_EPC_ARGS
}

}  // namespace moe

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
// inverse-map rows are read once, directly (plain loads; no bulk copies, no
// multicast).  The kernel never waits on another rank: the caller orders the
// launch after every rank's expert outputs are complete.
//
// One warp per item = (token, 1/split of the row).  For a group of up to 8
// ranks the warp loads the token's inverse-map rows of all of them at once
// (the first group of the next item is prefetched) and compacts them into one
// rank-ordered list of row pointers in shared memory, each entry tagged with
// the number of rank partials to close before it; then, per 16-byte unit of
// the row, it keeps 4 expert rows' loads in flight (8 in the kernel for more
// than 8 ranks or odd widths) and closes each rank's partial in rank order
// (ranks without rows contribute +0, as their partial block row would).
#include "common.cuh"
#include "launch.cuh"

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
// item, each unit's sum carried across the groups of 8 ranks.
template <class DI, class DP, class DO, bool VEC, bool ALIGNED>
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
      if (mine) fold_unit<DI, DP, VEC, ALIGNED>(ptrs, gaps, F, trailing, q0, u, acc);
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

template <class DI, class DP, class DO>
int launch(const void* const* eos, const void* const* invs, int world, int rank,
           const int32_t* offs, const int32_t* ep_tokens, int64_t capacity, int64_t max_rows,
           int E, void* out, int64_t local, int64_t hidden, int32_t* err, cudaStream_t stream) {
  using TO = typename DO::T;
  const bool vec = hidden % kVec == 0 && aligned16(out);
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

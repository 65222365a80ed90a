// rowlist.cuh -- ordered compaction of an inverse-map row (token -> rows of
// its local experts), shared by the unpermute and the fused epilogue.
#pragma once

#include "common.cuh"
#include "moe_epilogue.h"

namespace moe {

// Compacts inverse_map row t (entries e = 0 .. E-1) into list[], keeping the
// increasing-expert order: each 32-entry slice is one ballot, and a live
// entry's position is the number of live entries before it.  Entries at or
// past max_rows are reported and dropped.  Warp-wide; returns the count.
__device__ __forceinline__ int compact_row(const int32_t* inv_row, int E, int64_t max_rows,
                                           int32_t* list, int32_t* err, int lane) {
  int count = 0;
  for (int e0 = 0; e0 < E; e0 += 32) {
    const int e = e0 + lane;
    int32_t row = e < E ? __ldg(inv_row + e) : -1;
    if (row >= max_rows) {
      flag_error(err, MOE_DEVERR_INVERSE);
      row = -1;
    }
    const unsigned live = __ballot_sync(0xffffffffu, row >= 0);
    if (row >= 0) list[count + __popc(live & ((1u << lane) - 1u))] = row;
    count += __popc(live);
  }
  return count;
}

// Same, for E <= 64, from two entries per lane already loaded into registers.
__device__ __forceinline__ int compact_pair(int32_t r0, int32_t r1, int64_t max_rows,
                                            int32_t* list, int32_t* err, int lane) {
  if (r0 >= max_rows) { flag_error(err, MOE_DEVERR_INVERSE); r0 = -1; }
  if (r1 >= max_rows) { flag_error(err, MOE_DEVERR_INVERSE); r1 = -1; }
  const unsigned m0 = __ballot_sync(0xffffffffu, r0 >= 0);
  const unsigned m1 = __ballot_sync(0xffffffffu, r1 >= 0);
  const unsigned below = (1u << lane) - 1u;
  if (r0 >= 0) list[__popc(m0 & below)] = r0;
  if (r1 >= 0) list[__popc(m0) + __popc(m1 & below)] = r1;
  return __popc(m0) + __popc(m1);
}

}  // namespace moe

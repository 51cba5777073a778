// Validity of one block_idx row entry, shared by the kernels that read the
// selections.  An entry is used when it is a fully visible block index and
// larger than every earlier in-range entry of its row (so the used entries
// are ascending and distinct); anything else is skipped.
#pragma once

#include <stdint.h>

namespace ssa {

// Warp-collective: lane j holds entry v of the row (-1 for lanes >= topk).
// Returns whether this lane's entry is used.
__device__ __forceinline__ bool selection_valid(int v, int nvis) {
  const int lane = threadIdx.x & 31;
  const bool inrange = v >= 0 && v < nvis;
  int run = inrange ? v : -1;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xFFFFFFFFu, run, o);
    if (lane >= o) run = max(run, y);
  }
  int prev = __shfl_up_sync(0xFFFFFFFFu, run, 1);
  if (lane == 0) prev = -1;
  return inrange && v > prev;
}

}  // namespace ssa

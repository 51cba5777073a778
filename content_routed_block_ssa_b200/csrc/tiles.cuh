// The key set of one (query row, kv-head) item as a list of 64-key tiles.
//
// The attended keys are the union of the selected blocks' keys and the
// causal window pos-W+1 .. pos ["Subquadratic Sparse Attention (SSA)",
// opening section, (i) and (ii)].  A selected block contributes all its
// keys (it is fully visible by construction); a 64-key tile of the window
// whose block is not selected contributes the keys inside the window.  Each
// key therefore appears exactly once.
//
// Computed cooperatively by one warp (ballots and shuffles); every lane
// ends with the same list description.
#pragma once

#include <stdint.h>

namespace ssa {

struct ItemTiles {
  int64_t pos;        // key position of the query
  int64_t lo;         // first window key
  uint32_t selmask;   // lanes holding a valid selected block
  int my_blk;         // this lane's block_idx entry
  int n_sel;          // valid selected blocks
  int spb;            // 64-key tiles per block
  int64_t win_t0;     // first window tile (units of 64 keys)
  uint64_t winmask;   // window tiles (relative to win_t0) not covered by a selected block
  int n_sub;          // tiles in the list
  int n_bad;          // block_idx entries skipped as invalid
};

// v: this lane's entry of the item's block_idx row (-1 for lanes >= topk).
__device__ __forceinline__ ItemTiles item_tiles_v(int v, int topk, int64_t pos, int nb, int block,
                                                  int window) {
  const int lane = threadIdx.x & 31;
  ItemTiles it;
  it.pos = pos;
  const int nvis = static_cast<int>(min(static_cast<int64_t>(nb), (pos + 1) / block));
  const bool inrange = v >= 0 && v < nvis;
  // strictly ascending among the in-range entries: compare with the running
  // maximum of the in-range entries on lower lanes
  int run = inrange ? v : -1;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xFFFFFFFFu, run, o);
    if (lane >= o) run = max(run, y);
  }
  int prev = __shfl_up_sync(0xFFFFFFFFu, run, 1);
  if (lane == 0) prev = -1;
  const bool valid = inrange && v > prev;
  it.selmask = __ballot_sync(0xFFFFFFFFu, valid);
  it.my_blk = valid ? v : -1;
  it.n_sel = __popc(it.selmask);
  it.n_bad = __popc(__ballot_sync(0xFFFFFFFFu, lane < topk && v != -1 && !valid));
  it.spb = block / 64;
  it.lo = pos - window + 1 > 0 ? pos - window + 1 : 0;
  it.win_t0 = it.lo / 64;
  const int ntw = static_cast<int>(pos / 64 - it.win_t0) + 1;     // window tiles, <= 64
  // window tiles covered by this lane's selected block, then OR over the warp
  uint32_t cov_lo = 0, cov_hi = 0;
  if (valid) {
    for (int q = 0; q < it.spb; ++q) {
      const int64_t r = static_cast<int64_t>(v) * it.spb + q - it.win_t0;
      if (r >= 0 && r < 32) cov_lo |= 1u << r;
      else if (r >= 32 && r < 64) cov_hi |= 1u << (r - 32);
    }
  }
  cov_lo = __reduce_or_sync(0xFFFFFFFFu, cov_lo);
  cov_hi = __reduce_or_sync(0xFFFFFFFFu, cov_hi);
  const uint64_t all = ntw >= 64 ? ~0ull : ((1ull << ntw) - 1ull);
  it.winmask = all & ~((static_cast<uint64_t>(cov_hi) << 32) | cov_lo);
  const uint64_t wm = it.winmask;
  it.n_sub = it.n_sel * it.spb + __popcll(wm);
  return it;
}

// sel: the item's block_idx row (topk entries).
__device__ __forceinline__ ItemTiles item_tiles(const int32_t* __restrict__ sel, int topk,
                                                int64_t pos, int nb, int block, int window) {
  const int lane = threadIdx.x & 31;
  const int v = lane < topk ? __ldg(sel + lane) : -1;
  return item_tiles_v(v, topk, pos, nb, block, window);
}

// n-th set bit (0-based) of a 32-bit mask.
__device__ __forceinline__ int nth_bit32(uint32_t m, int n) {
  for (int k = 0; k < n; ++k) m &= m - 1;
  return __ffs(static_cast<int>(m)) - 1;
}

// n-th set bit (0-based) of a 64-bit mask.
__device__ __forceinline__ int nth_bit64(uint64_t m, int n) {
  for (int k = 0; k < n; ++k) m &= m - 1;
  return __ffsll(static_cast<long long>(m)) - 1;
}

// First key of tile j, computed by each lane for its own j (any j per lane;
// every lane must call).  Tiles j < n_sel*spb are selected-block tiles.
__device__ __forceinline__ int64_t tile_key0_lane(const ItemTiles& it, int j, int block) {
  const int ns = it.n_sel * it.spb;
  const int which = (j < ns) ? j / it.spb : 0;
  int src = (j < ns) ? nth_bit32(it.selmask, which) : 0;
  src = src < 0 ? 0 : src;
  const int blk = __shfl_sync(0xFFFFFFFFu, it.my_blk, src);
  if (j < ns) return static_cast<int64_t>(blk) * block + (j % it.spb) * 64;
  const int wbit = nth_bit64(it.winmask, j - ns);
  return (it.win_t0 + (wbit < 0 ? 0 : wbit)) * 64;
}

// Tile j of the list: first key and whether it is a (masked) window tile.
// Warp-collective (all lanes must call with the same j).
__device__ __forceinline__ int64_t tile_key0(const ItemTiles& it, int j, int block, bool& window_tile) {
  const int ns = it.n_sel * it.spb;
  if (j < ns) {
    const int which = j / it.spb;
    const int lane_of = nth_bit32(it.selmask, which);
    const int blk = __shfl_sync(0xFFFFFFFFu, it.my_blk, lane_of);
    window_tile = false;
    return static_cast<int64_t>(blk) * block + (j % it.spb) * 64;
  }
  window_tile = true;
  return (it.win_t0 + nth_bit64(it.winmask, j - ns)) * 64;
}

}  // namespace ssa

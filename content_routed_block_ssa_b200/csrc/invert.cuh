// The attended key set of one (query, kv-head) item as a set of partial
// "slots", shared by the kernels of the block-major attention.
//
// The keys are the union of the selected blocks and the causal window
// pos-W+1 .. pos ["Subquadratic Sparse Attention (SSA)", opening section, (i)
// and (ii)].  Slot j < topk is the row's j-th block_idx entry when it is
// used: a fully visible block index larger than every earlier in-range entry
// (so the used entries are ascending and distinct; anything else is skipped
// and counted).  Slot topk + s is chunk s of the window: its keys
// pos-W+1 + C s .. min(pos, pos-W + C (s+1)) that lie in no used block, with
// C = win_chunk(G) keys per chunk.
// Every key of the set is thus in exactly one slot.  Selected slots are
// evaluated block by block (the block kernel), window chunks by a dense
// sliding-window kernel.
#pragma once

#include <stdint.h>

namespace ssa {

// Keys per window chunk (one slot each): 256, or 128 when a query has one
// head per kv-head (a sliding-window tile then spans 128 queries, and its
// keys must still fit six 64-key blocks).
__host__ __device__ constexpr int win_chunk(int G) { return G == 1 ? 128 : 256; }

// An inverted entry: the query row and the slot of that row.
__device__ __forceinline__ int32_t make_entry(int row, int slot) { return (row << 6) | slot; }
__device__ __forceinline__ int entry_row(int32_t e) { return e >> 6; }
__device__ __forceinline__ int entry_slot(int32_t e) { return e & 63; }

// Most key blocks a window of W keys overlaps (blocks lo/B .. pos/B).
__host__ __device__ constexpr int window_slots(int window, int block) {
  return (window - 1 + block - 1) / block + 1;
}

// Window chunks (slots) of a window of W keys.
__host__ __device__ constexpr int window_chunks(int window, int G) {
  return (window + win_chunk(G) - 1) / win_chunk(G);
}

struct SlotSet {
  uint64_t mask;   // bit j < topk: selected slot j holds keys
  int n_bad;       // block_idx entries skipped as invalid
  int v;           // this lane's block_idx entry (-1 past topk)
  int64_t lo;      // first window key
  int64_t b0;      // first window block
  uint32_t win;    // bit w: window block b0 + w is in no used entry
};

// Warp-collective: lane l < topk passes entry l of the row (any value past
// topk is ignored).  window_slots(window, block) <= 32.
__device__ __forceinline__ SlotSet row_slots(int v_in, int topk, int64_t pos, int nb, int block, int window) {
  const int lane = threadIdx.x & 31;
  const int v = lane < topk ? v_in : -1;
  // positions are below 2^31 and the block is a power of two (64 or 128):
  // 32-bit shifts instead of 64-bit divisions
  const int p32 = static_cast<int>(pos);
  const int lb = __ffs(block) - 1;
  const int nvis = min(nb, (p32 + 1) >> lb);
  const bool inrange = v >= 0 && v < nvis;
  int run = inrange ? v : -1;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xFFFFFFFFu, run, o);
    if (lane >= o) run = max(run, y);
  }
  int prev = __shfl_up_sync(0xFFFFFFFFu, run, 1);
  if (lane == 0) prev = -1;
  const bool valid = inrange && v > prev;
  SlotSet s;
  s.v = v;
  s.mask = __ballot_sync(0xFFFFFFFFu, valid);
  s.n_bad = __popc(__ballot_sync(0xFFFFFFFFu, v != -1 && !valid));
  const int lo32 = max(p32 - window + 1, 0);
  s.lo = lo32;
  s.b0 = lo32 >> lb;
  const int nwb = (p32 >> lb) - (lo32 >> lb) + 1;
  // window block w is uncovered unless some used entry selects it: each
  // lane marks the window block its own entry covers, OR over the warp
  const int64_t w = static_cast<int64_t>(v) - s.b0;
  const uint32_t cov = __reduce_or_sync(0xFFFFFFFFu, (valid && w >= 0 && w < 32) ? (1u << w) : 0u);
  const uint32_t all = nwb >= 32 ? 0xFFFFFFFFu : ((1u << nwb) - 1u);
  s.win = all & ~cov;
  return s;
}

// Paired slots (64-key blocks).  Each (batch, kv-head) has a hot set of at
// most kHotBlocks blocks, its most selected ones, numbered in block order.
// A row's used entries that select hot blocks are taken two at a time in
// ascending block order: each pair is one selected slot of 128 keys (the
// two blocks' keys), evaluated for all rows that chose the same two blocks
// together.  Every other used entry (a block outside the hot set, or the
// last hot one when their number is odd) is a single slot of its block's 64
// keys.  Slots are numbered pairs first, then singles, both in block order.
// Tiles are keyed per (batch, kv-head): single block c -> key c; pair of hot
// numbers h1 < h2 -> key nb + pair_index(h1, h2), the pairs numbered row by
// row of the upper triangle.
constexpr int kHotBlocks = 128;
constexpr int kPairKeys = kHotBlocks * (kHotBlocks - 1) / 2;

__host__ __device__ constexpr int pair_index(int h1, int h2) {
  return h1 * (2 * kHotBlocks - h1 - 1) / 2 + (h2 - h1 - 1);
}

// Inverse of pair_index: the pair of pair number t (0 <= t < kPairKeys).
__host__ __device__ inline void pair_of_index(int t, int& h1, int& h2) {
  int a = 0;
  while (pair_index(a + 1, a + 2) <= t) ++a;   // first pair of row a+1 is past t
  h1 = a;
  h2 = t - pair_index(a, a + 1) + a + 1;
}

struct PairSlot {
  bool emit;       // this lane's entry starts a slot
  int key;         // its tile key
  int slot;        // its slot number
  int nsel;        // selected slots of the row
};

// Warp-collective.  s from row_slots; hid = hot number of this lane's entry
// (-1 when it is not hot or not used).  Every lane gets nsel.
__device__ __forceinline__ PairSlot pair_slots(const SlotSet& s, int hid, int nb) {
  const int lane = threadIdx.x & 31;
  const uint32_t lt = (1u << lane) - 1u;
  const bool used = (s.mask >> lane) & 1;
  const uint32_t used_m = static_cast<uint32_t>(s.mask);
  const uint32_t hot_m = __ballot_sync(0xFFFFFFFFu, used && hid >= 0);
  const int nhot = __popc(hot_m), npair = nhot >> 1;
  const int r = __popc(hot_m & lt);                       // rank among hot entries
  const bool hot = (hot_m >> lane) & 1;
  const bool paired = hot && r < 2 * npair;
  const uint32_t paired_m = __ballot_sync(0xFFFFFFFFu, paired);
  const uint32_t single_m = used_m & ~paired_m;
  // the next hot lane above this one (the partner of a pair's first entry)
  const uint32_t above = hot_m & ~(lt | (1u << lane));
  const int partner = above ? __ffs(static_cast<int>(above)) - 1 : lane;
  const int hid2 = __shfl_sync(0xFFFFFFFFu, hid, partner);
  PairSlot o;
  o.nsel = __popc(used_m) - npair;
  if (paired) {
    o.emit = (r & 1) == 0;
    o.key = nb + pair_index(hid, hid2);
    o.slot = r >> 1;
  } else {
    o.emit = used;
    o.key = s.v;
    o.slot = npair + __popc(single_m & lt);
  }
  return o;
}

// Tile block field for a pair mode tile: first block in bits 0..14, second
// block + 1 above (0 for a single block).
__host__ __device__ constexpr int pair_tile_y(int c1, int c2) { return c1 | ((c2 + 1) << 15); }
__host__ __device__ constexpr int pair_tile_c1(int y) { return y & 0x7FFF; }
__host__ __device__ constexpr int pair_tile_c2(int y) { return (y >> 15) - 1; }

// Whether window chunk s (of `chunk` keys) of the row at pos holds keys:
// some block it overlaps is uncovered.  win as in SlotSet (blocks b0 + w).
__host__ __device__ inline bool chunk_has_keys(uint32_t win, int64_t pos, int window, int block, int s,
                                               int chunk) {
  const int64_t w0 = pos - window + 1;                 // unclamped window start
  int64_t klo = w0 + static_cast<int64_t>(s) * chunk;
  int64_t khi = w0 + static_cast<int64_t>(s + 1) * chunk - 1;
  if (khi > pos) khi = pos;
  if (klo < 0) klo = 0;
  if (khi < klo) return false;
  // non-negative keys below 2^31 and a power-of-two block: shifts
#ifdef __CUDA_ARCH__
  const int lb = __ffs(block) - 1;
#else
  const int lb = __builtin_ctz(static_cast<unsigned>(block));
#endif
  const int b0 = static_cast<int>(w0 > 0 ? w0 : 0) >> lb;
  const int f = (static_cast<int>(klo) >> lb) - b0, l = (static_cast<int>(khi) >> lb) - b0;
  const uint32_t span = (l - f + 1 >= 32) ? 0xFFFFFFFFu : ((1u << (l - f + 1)) - 1u);
  return ((win >> f) & span) != 0;
}

}  // namespace ssa

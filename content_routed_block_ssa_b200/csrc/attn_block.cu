// Block-major evaluation of the routed part of the attention (steps (ii) and
// (iii) of "Subquadratic Sparse Attention (SSA)", opening section): instead of
// every query gathering its selected key blocks, every selected block is
// read once and multiplied against the queries that selected it.
//
//  1. inversion: count the selections per key block, scan, scatter the
//     (query, slot) entries into per-block lists and cut each list into
//     tiles of 128 / G queries (128 tensor-core rows with the G query heads);
//  2. block tiles on tcgen05: the tile's Q rows are gathered with 16-byte
//     asynchronous copies into the 128-byte-swizzled operand layout, K_c and
//     V_c arrive by TMA, S = Q K_c^T and O = P V_c run on the tensor cores with TMEM
//     accumulators, the softmax over the block's keys runs in between, and
//     each (query, head, slot) gets a normalised partial output (float16
//     with a power-of-two row scale) and its log-sum-exp (base 2, of the
//     scaled logits);
//  3. the window keys and the merge of the partials into the final output
//     run in the gather kernel (attn.cu, merge mode), one query row at a time.
//
// Exact: the merge of normalised partials with their log-sum-exps is the
// same softmax over the union of the selected blocks and the window.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>

#include "common.cuh"
#include "invert.cuh"
#include "kernels.h"

namespace ssa {
namespace {

// ------------------------------------------------------------------ inversion
//
// The rows of one (batch, kv-head) are cut into chunks of kPlanRows.  A CTA
// per chunk counts its selected slots per key block in shared memory; a
// column scan over the chunks then gives every (chunk, block) its place in
// the block's entry list, so the scatter again needs only shared-memory
// atomics.  The counting pass also records each row's uncovered window
// blocks for the sliding-window kernel.

constexpr int kPlanThreads = 512;

// Hot number of this lane's entry (-1 when unused or not hot).
__device__ __forceinline__ int lane_hot_id(const BlockPlan& pl, const SlotSet& s, int bg) {
  const int lane = threadIdx.x & 31;
  return ((s.mask >> lane) & 1) ? __ldg(pl.hot_id + static_cast<int64_t>(bg) * pl.nb + s.v) : -1;
}

// Counting passes over the rows of one chunk.  MODE 0: counts per key block
// and each row's uncovered window blocks (the only pass without pairs).
// MODE 1 (pair mode, first pass): counts per key block over every
// kHotSample-th row only, added into per-block totals — they choose the hot
// set, and any hot set gives the same attention.  MODE 2 (pair mode):
// counts per tile key and the window blocks, every row.  chist columns:
// blocks (0) or keys (2).
constexpr int kHotSample = 8;

template <int MODE>
__global__ void __launch_bounds__(kPlanThreads) inv_hist_kernel(const BlockPlan pl, const int32_t* __restrict__ idx) {
  extern __shared__ int32_t hist[];
  const int ncol = MODE == 2 ? pl.nkey : pl.nb;
  const int step = MODE == 1 ? kHotSample : 1;
  const int k = blockIdx.x, bg = blockIdx.y;
  for (int c = threadIdx.x; c < ncol; c += blockDim.x) hist[c] = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int b = bg / pl.h_kv, g = bg % pl.h_kv;
  const int r1 = min((k + 1) * kPlanRows, pl.n_q);
  for (int i = k * kPlanRows + warp * step; i < r1; i += nw * step) {
    const int v = lane < pl.topk ? __ldg(idx + ((static_cast<int64_t>(b) * pl.n_q + i) * pl.h_kv + g) * pl.topk + lane) : -1;
    const SlotSet s = row_slots(v, pl.topk, pl.q_offset + i, pl.nb, pl.block, pl.window);
    uint32_t selmask = static_cast<uint32_t>(s.mask);
    if (MODE == 2) {
      const PairSlot ps = pair_slots(s, lane_hot_id(pl, s, bg), pl.nb);
      if (ps.emit) atomicAdd(&hist[ps.key], 1);
      selmask = ps.nsel >= 32 ? 0xFFFFFFFFu : ((1u << ps.nsel) - 1u);   // slots 0 .. nsel-1
    } else {
      if ((s.mask >> lane) & 1) atomicAdd(&hist[s.v], 1);
    }
    if (MODE != 1 && lane == 0) {
      const int64_t it = static_cast<int64_t>(bg) * pl.n_q + i;
      pl.win[it] = s.win;
      pl.rowinfo[it] = make_uint2(selmask, static_cast<uint32_t>(s.n_bad));
    }
  }
  __syncthreads();
  if (MODE == 1) {   // sampled block totals, summed over the chunks (pl.count zeroed)
    int32_t* tot = pl.count + static_cast<int64_t>(bg) * pl.nb;
    for (int c = threadIdx.x; c < ncol; c += blockDim.x)
      if (hist[c]) atomicAdd(&tot[c], hist[c]);
    return;
  }
  int32_t* out = pl.chist + (static_cast<int64_t>(bg) * pl.nchunk + k) * ncol;
  for (int c = threadIdx.x; c < ncol; c += blockDim.x) out[c] = hist[c];
}

// One CTA per (batch, kv-head), pair mode: from each block's sampled
// selections (totals of the first pass), the hot set is the largest set
// {c : count_c >= T} (T >= 2) of at most kHotBlocks blocks, numbered in
// block order.
__global__ void __launch_bounds__(1024) inv_hot_kernel(const BlockPlan pl) {
  extern __shared__ int32_t tot[];   // [nb]
  __shared__ int32_t red[32];
  __shared__ int32_t s_lo, s_hi;
  const int bg = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int32_t* cnt = pl.count + static_cast<int64_t>(bg) * pl.nb;
  for (int c = threadIdx.x; c < pl.nb; c += blockDim.x) tot[c] = cnt[c];
  // block-wide count of blocks with tot >= T
  auto count_ge = [&](int T) {
    int n = 0;
    for (int c = threadIdx.x; c < pl.nb; c += blockDim.x) n += tot[c] >= T ? 1 : 0;
#pragma unroll
    for (int o = 16; o; o >>= 1) n += __shfl_xor_sync(0xFFFFFFFFu, n, o);
    __syncthreads();   // red is free (also orders the tot writes before the first reads)
    if (lane == 0) red[warp] = n;
    __syncthreads();
    int t = 0;
    for (int w = 0; w < 32; ++w) t += red[w];
    return t;
  };
  // smallest T in [2, n_q + 1] with count_ge(T) <= kHotBlocks (count_ge(n_q + 1) = 0)
  if (threadIdx.x == 0) { s_lo = 2; s_hi = pl.n_q + 1; }
  __syncthreads();
  while (true) {
    const int lo = s_lo, hi = s_hi;   // uniform
    if (lo >= hi) break;
    const int mid = lo + ((hi - lo) >> 1);
    const int n = count_ge(mid);
    __syncthreads();
    if (threadIdx.x == 0) {
      if (n <= kHotBlocks) s_hi = mid; else s_lo = mid + 1;
    }
    __syncthreads();
  }
  const int T = s_lo;
  // hot numbers in block order: a block-wide exclusive scan of the flags
  const int per = (pl.nb + 1023) / 1024;
  const int c0 = threadIdx.x * per;
  int mine = 0;
  for (int c = c0; c < min(c0 + per, pl.nb); ++c) mine += tot[c] >= T ? 1 : 0;
  int inc = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xFFFFFFFFu, inc, o);
    if (lane >= o) inc += y;
  }
  __syncthreads();
  if (lane == 31) red[warp] = inc;
  __syncthreads();
  int base = inc - mine;
  for (int w = 0; w < warp; ++w) base += red[w];
  int32_t* hid = pl.hot_id + static_cast<int64_t>(bg) * pl.nb;
  int32_t* hb = pl.hot_blk + static_cast<int64_t>(bg) * kHotBlocks;
  for (int c = c0; c < min(c0 + per, pl.nb); ++c) {
    if (tot[c] >= T) {
      hid[c] = base;
      hb[base] = c;
      ++base;
    } else {
      hid[c] = -1;
    }
  }
}

// Thread per (batch, kv-head, key): exclusive scan of the chunk counts in
// place, and the key's total.
__global__ void __launch_bounds__(256) inv_colscan_kernel(const BlockPlan pl) {
  const int64_t x = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (x >= static_cast<int64_t>(pl.bgs) * pl.nkey) return;
  const int bg = static_cast<int>(x / pl.nkey), c = static_cast<int>(x % pl.nkey);
  int32_t* col = pl.chist + static_cast<int64_t>(bg) * pl.nchunk * pl.nkey + c;
  int run = 0;
  int k = 0;
  for (; k + 8 <= pl.nchunk; k += 8) {   // eight loads in flight per thread
    int v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = col[static_cast<int64_t>(k + u) * pl.nkey];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      col[static_cast<int64_t>(k + u) * pl.nkey] = run;
      run += v[u];
    }
  }
  for (; k < pl.nchunk; ++k) {
    const int v = col[static_cast<int64_t>(k) * pl.nkey];
    col[static_cast<int64_t>(k) * pl.nkey] = run;
    run += v;
  }
  pl.count[x] = run;
}

// One CTA per (batch, kv-head): exclusive scans of the per-key entry and
// tile counts.
__global__ void __launch_bounds__(1024) inv_scan_kernel(const BlockPlan pl) {
  __shared__ int32_t wsum_e[32], wsum_t[32];
  const int bg = blockIdx.x;
  const int32_t* cnt = pl.count + static_cast<int64_t>(bg) * pl.nkey;
  const int per = (pl.nkey + 1023) / 1024;
  const int c0 = threadIdx.x * per;
  int se = 0, st = 0;
  for (int c = c0; c < min(c0 + per, pl.nkey); ++c) {
    se += cnt[c];
    st += (cnt[c] + pl.qpt - 1) / pl.qpt;
  }
  // block-wide exclusive scan of (se, st)
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int ie = se, it = st;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int ye = __shfl_up_sync(0xFFFFFFFFu, ie, o), yt = __shfl_up_sync(0xFFFFFFFFu, it, o);
    if (lane >= o) { ie += ye; it += yt; }
  }
  if (lane == 31) { wsum_e[warp] = ie; wsum_t[warp] = it; }
  __syncthreads();
  if (warp == 0) {
    int ve = wsum_e[lane], vt = wsum_t[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int ye = __shfl_up_sync(0xFFFFFFFFu, ve, o), yt = __shfl_up_sync(0xFFFFFFFFu, vt, o);
      if (lane >= o) { ve += ye; vt += yt; }
    }
    wsum_e[lane] = ve;
    wsum_t[lane] = vt;
  }
  __syncthreads();
  int base_e = (warp ? wsum_e[warp - 1] : 0) + ie - se;
  int base_t = (warp ? wsum_t[warp - 1] : 0) + it - st;
  for (int c = c0; c < min(c0 + per, pl.nkey); ++c) {
    pl.blk_off[static_cast<int64_t>(bg) * pl.nkey + c] = base_e;
    pl.tile_off[static_cast<int64_t>(bg) * pl.nkey + c] = base_t;
    base_e += cnt[c];
    base_t += (cnt[c] + pl.qpt - 1) / pl.qpt;
  }
  if (threadIdx.x == 1023) {
    pl.bg_ents[bg] = base_e;
    pl.bg_tiles[bg] = base_t;
  }
}

// One thread: exclusive scans over (batch, kv-head); slot [bgs] holds the totals.
__global__ void __launch_bounds__(32) inv_scan_bg_kernel(const BlockPlan pl) {
  if (threadIdx.x != 0) return;
  int e = 0, t = 0;
  for (int bg = 0; bg < pl.bgs; ++bg) {
    pl.ent_base[bg] = e;
    pl.tile_base[bg] = t;
    e += pl.bg_ents[bg];
    t += pl.bg_tiles[bg];
  }
  pl.ent_base[pl.bgs] = e;
  pl.tile_base[pl.bgs] = t;
}

// Same rows as inv_hist_kernel: every selected slot becomes the entry
// make_entry(query row, slot) in its key's list.
__global__ void __launch_bounds__(kPlanThreads) inv_scatter_kernel(const BlockPlan pl, const int32_t* __restrict__ idx) {
  extern __shared__ int32_t cur[];
  const int k = blockIdx.x, bg = blockIdx.y;
  const int32_t* col = pl.chist + (static_cast<int64_t>(bg) * pl.nchunk + k) * pl.nkey;
  const int32_t* boff = pl.blk_off + static_cast<int64_t>(bg) * pl.nkey;
  const int ebase = pl.ent_base[bg];
  for (int c = threadIdx.x; c < pl.nkey; c += blockDim.x) cur[c] = ebase + boff[c] + col[c];
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int b = bg / pl.h_kv, g = bg % pl.h_kv;
  const int r1 = min((k + 1) * kPlanRows, pl.n_q);
  for (int i = k * kPlanRows + warp; i < r1; i += nw) {
    const int v = lane < pl.topk ? __ldg(idx + ((static_cast<int64_t>(b) * pl.n_q + i) * pl.h_kv + g) * pl.topk + lane) : -1;
    const SlotSet s = row_slots(v, pl.topk, pl.q_offset + i, pl.nb, pl.block, pl.window);
    if (pl.pair) {
      const PairSlot ps = pair_slots(s, lane_hot_id(pl, s, bg), pl.nb);
      if (ps.emit) pl.entries[atomicAdd(&cur[ps.key], 1)] = make_entry(i, ps.slot);
    } else {
      if ((s.mask >> lane) & 1) pl.entries[atomicAdd(&cur[s.v], 1)] = make_entry(i, lane);
    }
  }
}

// A warp per (batch, kv-head, key): its tiles written lane-strided (a
// block chosen by nearly every query has tens of thousands of tiles).  The
// tile's block field is the block, or in pair mode pair_tile_y(c1, c2).
__global__ void __launch_bounds__(256) inv_tiles_kernel(const BlockPlan pl) {
  const int64_t x = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  if (x >= static_cast<int64_t>(pl.bgs) * pl.nkey) return;   // warp-uniform
  const int lane = threadIdx.x & 31;
  const int bg = static_cast<int>(x / pl.nkey), c = static_cast<int>(x % pl.nkey);
  const int n = pl.count[x];
  if (n == 0) return;
  int y = c;
  if (pl.pair) {
    if (c < pl.nb) {
      y = pair_tile_y(c, -1);
    } else {
      int h1, h2;
      pair_of_index(c - pl.nb, h1, h2);
      const int32_t* hb = pl.hot_blk + static_cast<int64_t>(bg) * kHotBlocks;
      y = pair_tile_y(hb[h1], hb[h2]);
    }
  }
  const int e0 = pl.ent_base[bg] + pl.blk_off[x];
  const int t0 = pl.tile_base[bg] + pl.tile_off[x];
  const int nt = (n + pl.qpt - 1) / pl.qpt;
  for (int t = lane; t < nt; t += 32)
    pl.tiles[t0 + t] = make_int4(bg, y, e0 + t * pl.qpt, min(pl.qpt, n - t * pl.qpt));
}

// Work estimate of each tile for the split over CTAs (units of a quarter of
// a tile, from per-CTA cycle counts of the block kernel on B200): a tile
// costs 4, plus block_start_cost for the first tile of a block (loading
// K_c, V_c; with one K/V buffer the pipeline drains).  The per-256-tile
// sums go to csum.
__global__ void __launch_bounds__(256) inv_cost_kernel(const BlockPlan pl, int block_start_cost) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  const int T = pl.tile_base[pl.bgs];
  int cost = 0;
  if (t < T) {
    const int4 td = pl.tiles[t];
    cost = 4;
    if (t == 0) {
      cost += block_start_cost;
    } else {
      const int4 tp = pl.tiles[t - 1];
      if (tp.x != td.x || tp.y != td.y) cost += block_start_cost;
    }
    pl.tcost[t] = static_cast<uint8_t>(cost);
  }
  // block sum
  __shared__ int ws[8];
  int v = cost;
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  if ((threadIdx.x & 31) == 0) ws[threadIdx.x >> 5] = v;
  __syncthreads();
  if (threadIdx.x == 0) {
    int sum = 0;
    for (int w = 0; w < 8; ++w) sum += ws[w];
    pl.csum[blockIdx.x] = sum;
  }
}

// One CTA: exclusive scan of the 256-tile sums, then for every split point
// b * total / grid the first tile whose cost prefix reaches it.
__global__ void __launch_bounds__(1024) inv_split_kernel(const BlockPlan pl, int n_chunks) {
  __shared__ int wsum[32];
  __shared__ int total_s;
  const int per = (n_chunks + 1023) / 1024;
  const int c0 = threadIdx.x * per;
  int local = 0;
  for (int c = c0; c < min(c0 + per, n_chunks); ++c) local += pl.csum[c];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int inc = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xFFFFFFFFu, inc, o);
    if (lane >= o) inc += y;
  }
  if (lane == 31) wsum[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    int v = wsum[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xFFFFFFFFu, v, o);
      if (lane >= o) v += y;
    }
    wsum[lane] = v;
    if (lane == 31) total_s = v;
  }
  __syncthreads();
  int run = (warp ? wsum[warp - 1] : 0) + inc - local;
  for (int c = c0; c < min(c0 + per, n_chunks); ++c) {
    const int x = pl.csum[c];
    pl.csum[c] = run;   // exclusive prefix
    run += x;
  }
  __syncthreads();
  const int total = total_s;
  const int T = pl.tile_base[pl.bgs];
  for (int b = threadIdx.x; b <= pl.grid; b += blockDim.x) {
    int t;
    if (b == 0) {
      t = 0;
    } else if (b == pl.grid) {
      t = T;
    } else {
      const int target = static_cast<int>((static_cast<int64_t>(total) * b) / pl.grid);
      // last chunk whose prefix is <= target, then walk its tiles
      int lo = 0, hi = n_chunks - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (pl.csum[mid] <= target) lo = mid; else hi = mid - 1;
      }
      int acc = pl.csum[lo];
      t = lo * 256;
      const int tend = min(T, (lo + 1) * 256);
      while (t < tend && acc + pl.tcost[t] <= target) acc += pl.tcost[t++];
      t = min(t, T);
    }
    pl.t_start[b] = t;
  }
}

// ------------------------------------------------------------------ block tiles

// The second 128-key sub-tile of a 256-key tile keeps the softmax's running
// maximum while its own maximum exceeds it by at most this many powers of
// two (P <= 2^16 then).  Pairs of selected blocks differ in their largest
// logit by more than 8 powers of two in a few percent of rows, by more than
// 16 in about one in a thousand.
constexpr float kStaleMax = 16.f;

template <int G, int BLK>
struct BlkCfg {
  static_assert(BLK == 128 || BLK == 256, "tiles hold pairs of 64- or 128-key blocks");
  static constexpr int D = 128;
  static constexpr int ROW = 128;                       // bytes per 64-wide swizzled row
  static constexpr int A_HALF = 128 * ROW;              // 128 rows x 64 dims
  static constexpr int A_BYTES = 2 * A_HALF;            // Q tile
  // Q tile buffers: with G = 8 one warp fills them all by TMA; otherwise one
  // cp.async warp per buffer.  256-key tiles fit two beside their 128 KB of
  // K and V.
  static constexpr bool TMA_Q = (G == 8);
  static constexpr int NA = BLK == 256 ? 2 : 4;
  static constexpr int NGW = TMA_Q ? 1 : NA;            // gather warps
  static constexpr int KV_HALF = BLK * ROW;             // BLK keys x 64 dims
  static constexpr int KV_BYTES = 4 * KV_HALF;          // K lo, K hi, V lo, V hi
  static constexpr int NKV = 1;                         // K/V buffers
  static constexpr int STG_WARP = 32 * 64;              // epilogue staging per softmax warp: 32 rows x 32 dims
  // S sub-tiles: a 256-key tile runs as two 128-key sub-tiles that share its
  // Q rows and its O accumulator
  static constexpr int SK = 128;                        // keys per sub-tile
  static constexpr int SUB = BLK / SK;                  // sub-tiles per tile
  // barriers: a[NA] x 2, kv[NKV] x 2, s_full and p_full [2][SUB], s_empty,
  // o_full, o_empty, ml_empty, pa_done [2], mma_done
  static constexpr int NBAR = 2 * NA + 2 * NKV + 4 * SUB + 10 + 1;
  // (m, l, lr) of each row from the softmax to the epilogue, by tile parity
  static constexpr int ML_BYTES = 2 * 128 * 16;
  static constexpr int USED = NA * A_BYTES + NKV * KV_BYTES + 8 * STG_WARP + ML_BYTES + NBAR * 8 + 16;
  // room to align the base to 1024 bytes, up to the 227 KB limit (the
  // kernel checks that the aligned layout fits)
  static constexpr int SMEM = USED + 1024 < 232448 ? USED + 1024 : 232448;
  static constexpr int SW0 = 2 + NGW;                   // first softmax warp
  static constexpr int THREADS = 32 * (SW0 + 8);        // KV, MMA, gather, 2 x 4 softmax warps
  // registers per thread: a sub-partition (SMSP) holds ceil(warps / 4) warps
  // of its 16384 registers
  static constexpr int MAXREG = (16384 / (32 * ((SW0 + 8 + 3) / 4))) & ~7;
  // TMEM: S[2] by sub-tile parity (P over the first SK/2 columns of its S),
  // O[2] by tile parity
  static constexpr int NSB = 2;
  static constexpr int S_COL = 0;
  static constexpr int O_COL = NSB * SK;
  static_assert(O_COL + 2 * D <= 512, "tensor memory");
  static_assert(USED <= 232448, "shared memory");
};

struct BlkArgs {
  const __nv_bfloat16* Q;
  const int4* tiles;
  const int32_t* t_start;    // device: [grid + 1] first tile of each CTA
  const int32_t* entries;    // make_entry(query row, slot)
  int32_t n_q, n_kv, h_q, h_kv, topk, window, nsl;
  int64_t q_offset;
  float scale_log2;
  __half* partO;             // [items][nsl][G][D], o / 2^e per 64-dim half
  float2* partL;             // [items][nsl][G]: (log2-sum-exp, e0 | e1 << 16 as int16s)
  uint32_t* err;
};

__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ int64_t tile_key(const int4& t) { return static_cast<int64_t>(t.x) * 0x7FFFFFFF + t.y; }

// Shared-memory descriptor of an MN-major operand written by TMA with the
// 128-byte swizzle: rows of 64 MN-elements (128 B), 8-row groups `sbo` apart
// along K, 64-element MN groups `lbo` apart.
__device__ __forceinline__ uint64_t umma_desc_sw128_mn(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}

__device__ __forceinline__ float max8(const float (&v)[8]) {
  return fmaxf(fmaxf(fmaxf(v[0], v[1]), fmaxf(v[2], v[3])), fmaxf(fmaxf(v[4], v[5]), fmaxf(v[6], v[7])));
}

// 64 consecutive TMEM columns of this warp's 32 lanes into registers.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&r)[64]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) tmem_ld16(taddr + q * 16, *reinterpret_cast<uint32_t(*)[16]>(&r[q * 16]));
  tmem_wait_ld();
  tmem_regs_ready(r);
}

// One CTA per SM walks a contiguous range of tiles (ordered by key block, so
// a block's K_c, V_c are loaded once per CTA).  Warp roles:
//   0      K/V producer: TMA of each new block's K_c, V_c;
//   1      MMA issuer and TMEM owner: a non-blocking loop that issues
//          S = Q K_c^T for the next tile whose Q rows have landed and
//          O = P V_c for the oldest tile whose P is written, whichever is
//          ready first;
//   2 ..   Q gather into NA buffers: with G = 8 one warp issues two TMA
//          boxes per entry for every tile; otherwise warp 2 + q fills
//          buffer q with the rows of tiles q, q + NA, ... (16-byte
//          asynchronous copies to their 128-byte-swizzled positions);
//   SW0 .. softmax and epilogue in two groups of four warps that take
//          alternate tiles (S, P and O are double-buffered by tile parity),
//          one tensor-core row = one (query, head) pair per thread.
//
// PAIR (BLK = 2 x the block size: 128 for 64-key blocks, 256 for 128-key
// blocks): a tile's keys are the two blocks of a pair, pair_tile_c1/c2 of
// its block field, loaded into the two halves; a single-block tile loads its
// block into both halves and its softmax leaves the second half out (P = 0
// there).
template <int G, int BLK>
__global__ void __maxnreg__((BlkCfg<G, BLK>::MAXREG))
    attn_block_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                      const __grid_constant__ CUtensorMap tmQ, const BlkArgs a) {
  using C = BlkCfg<G, BLK>;
  constexpr int D = C::D;
  constexpr int QPT = 128 / G;
  constexpr int NA = C::NA;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  if (static_cast<int>(smem - smem_raw) + C::USED > C::SMEM) {   // never with a 1024-aligned base
    if (threadIdx.x == 0) atomicCAS(a.err, 0u, static_cast<uint32_t>(SITE_BLK_SMEM));
    return;
  }
  uint8_t* sA = smem;                                   // [NA][A_BYTES]
  uint8_t* sKV = sA + NA * C::A_BYTES;                  // [NKV][KV_BYTES]
  uint8_t* sStg = sKV + C::NKV * C::KV_BYTES;           // [8][STG_WARP] epilogue staging
  float4* sML = reinterpret_cast<float4*>(sStg + 8 * C::STG_WARP);   // [2][128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sStg + 8 * C::STG_WARP + C::ML_BYTES);
  uint64_t* a_full = bars;                  // [NA] gather warp arrives once its copies landed
  uint64_t* a_empty = a_full + NA;          // [NA]
  uint64_t* kv_full = a_empty + NA;         // [NKV]
  uint64_t* kv_empty = kv_full + C::NKV;    // [NKV]
  uint64_t* s_full = kv_empty + C::NKV;     // [2][SUB]
  uint64_t* p_full = s_full + 2 * C::SUB;   // [2][SUB]
  uint64_t* s_empty = p_full + 2 * C::SUB;  // [2] by S buffer
  uint64_t* o_full = s_empty + 2;           // [2]
  uint64_t* o_empty = o_full + 2;           // [2]
  uint64_t* ml_empty = o_empty + 2;         // [2]
  uint64_t* pa_done = ml_empty + 2;         // [2]
  uint64_t* mma_done = pa_done + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    for (int i = 0; i < NA; ++i) { mbar_init(&a_full[i], 1); mbar_init(&a_empty[i], 1); }
    for (int i = 0; i < C::NKV; ++i) { mbar_init(&kv_full[i], 1); mbar_init(&kv_empty[i], 1); }
    for (int i = 0; i < 2 * C::SUB; ++i) { mbar_init(&s_full[i], 1); mbar_init(&p_full[i], 4); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_empty[i], 1);
      mbar_init(&o_full[i], 1); mbar_init(&o_empty[i], 4);
      mbar_init(&ml_empty[i], 4);
      mbar_init(&pa_done[i], 1);
    }
    mbar_init(mma_done, 1);
    fence_barrier_init();
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    if (C::TMA_Q) tma_prefetch_desc(&tmQ);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int t0 = a.t_start[blockIdx.x], t1 = a.t_start[blockIdx.x + 1];
  const int T = t1 - t0;
  const int4 none = make_int4(-1, -1, 0, 0);

  if (warp == 0) {
    // ------------------------------------------------------------ K/V producer
    if (lane == 0) {
      bool ok = true;
      int kv_ord = -1;
      int64_t prev = -1;
      uint32_t kv_loads = 0;
      int4 nxt = T > 0 ? a.tiles[t0] : none;
      for (int t = t0; t < t1 && ok; ++t) {
        const int4 td = nxt;
        nxt = t + 1 < t1 ? a.tiles[t + 1] : none;
        const int64_t key = tile_key(td);
        if (key == prev) continue;
        ++kv_ord;
        prev = key;
        const int kb = kv_ord % C::NKV;
        ok = mbar_wait(&kv_empty[kb], ((kv_ord / C::NKV) & 1) ^ 1, a.err, SITE_BLK_KV_EMPTY);
        if (!ok) break;
        const int b = td.x / a.h_kv, g = td.x % a.h_kv;
        uint8_t* kv = sKV + kb * C::KV_BYTES;
        mbar_arrive_expect_tx(&kv_full[kb], C::KV_BYTES);
        // first key of each 64-key half of the tile
        int zs[BLK / 64];
        constexpr int KPB = BLK / 2;   // keys per block of the pair
        const int c1 = pair_tile_c1(td.y), c2 = pair_tile_c2(td.y);
#pragma unroll
        for (int sub = 0; sub < BLK / 64; ++sub) {
          const int src = sub * 64 < KPB ? c1 : (c2 >= 0 ? c2 : c1);
          zs[sub] = static_cast<int>(static_cast<int64_t>(b) * a.n_kv + static_cast<int64_t>(src) * KPB +
                                     (sub * 64) % KPB);
        }
#pragma unroll
        for (int sub = 0; sub < BLK / 64; ++sub) {
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            tma_load_3d(kv + hf * C::KV_HALF + sub * 64 * C::ROW, &tmK, &kv_full[kb], hf * 64, g, zs[sub]);
            tma_load_3d(kv + (2 + hf) * C::KV_HALF + sub * 64 * C::ROW, &tmV, &kv_full[kb], hf * 64, g, zs[sub]);
          }
        }
        ++kv_loads;
      }
      if (!ok) {   // let issued copies land before the CTA exits
        const uint64_t tq = global_timer_ns();
        for (uint32_t n = (kv_loads > C::NKV ? kv_loads - C::NKV : 0); n < kv_loads; ++n)
          while (!mbar_try_wait(&kv_full[n % C::NKV], (n / C::NKV) & 1) && global_timer_ns() - tq < kWaitLimitNs) {}
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr int SK = C::SK, SUB = C::SUB;
      constexpr uint32_t IDESC1 = umma_idesc_bf16(128, SK);
      constexpr uint32_t IDESC2 = umma_idesc_bf16(128, D) | (1u << 16);   // B (V) is MN-major
      const uint32_t sA_u = smem_u32(sA), sKV_u = smem_u32(sKV);
      // sub-tiles u = SUB tile + sub whose S = Q K^T / O += P V are issued
      int u1 = 0, u2 = 0;
      const int U = T * SUB;
      int kv_ord = -1;
      int64_t prev = -1;
      uint32_t ring_kb = 0, ring_last = 0;   // bit (n & 3) per tile in flight, read by its P V
      int4 cur = T > 0 ? a.tiles[t0] : none;
      int4 nxt = T > 1 ? a.tiles[t0 + 1] : none;
      int4 nxt2 = T > 2 ? a.tiles[t0 + 2] : none;
      bool fresh = tile_key(cur) != prev;
      int kb = (kv_ord + (fresh ? 1 : 0)) % C::NKV;
      uint64_t last_progress = global_timer_ns();
      uint32_t spins = 0;
      bool ok = true;
      while (u2 < U) {
        bool progressed = false;
        const int n1 = u1 / SUB, s1 = u1 % SUB;
        if (u1 < U && n1 - u2 / SUB < 4) {
          const int ab = n1 % NA;
          const int ord = kv_ord + (fresh ? 1 : 0);
          // a tile's first sub-tile waits for its K, V and Q rows; S(u1)
          // reuses the S columns of sub-tile u1 - NSB once its P V has read
          // them (each barrier waited on in order)
          if ((s1 > 0 || ((!fresh || mbar_test_wait(&kv_full[kb], (ord / C::NKV) & 1)) &&
                          mbar_test_wait(&a_full[ab], (n1 / NA) & 1))) &&
              (u1 < C::NSB ||
               mbar_test_wait(&s_empty[(u1 - C::NSB) & 1], ((u1 - C::NSB) >> 1) & 1))) {
            tc_fence_after();
            const uint32_t s_tmem = tmem_base + C::S_COL + (u1 & 1) * SK;
            const uint32_t kbase = sKV_u + kb * C::KV_BYTES + s1 * SK * C::ROW;
#pragma unroll
            for (int ks = 0; ks < D / 16; ++ks) {
              const uint64_t ad = umma_desc_sw128(sA_u + ab * C::A_BYTES + (ks >> 2) * C::A_HALF + (ks & 3) * 32);
              const uint64_t bd = umma_desc_sw128(kbase + (ks >> 2) * C::KV_HALF + (ks & 3) * 32);
              umma_bf16(s_tmem, ad, bd, IDESC1, ks != 0 ? 1u : 0u);
            }
            umma_commit(&s_full[(n1 & 1) * SUB + s1]);
            if (s1 == 0) {   // the tile's K/V buffer, and whether it is the buffer's last tile
              const uint32_t bit = 1u << (n1 & 3);
              ring_kb = kb ? (ring_kb | bit) : (ring_kb & ~bit);
              ring_last = (n1 + 1 == T || tile_key(nxt) != tile_key(cur)) ? (ring_last | bit) : (ring_last & ~bit);
            }
            if (s1 == SUB - 1) {   // the tile's Q rows are read
              umma_commit(&a_empty[ab]);
              if (fresh) { kv_ord = ord; prev = tile_key(cur); }
              cur = nxt;
              nxt = nxt2;
              nxt2 = n1 + 3 < T ? a.tiles[t0 + n1 + 3] : none;
              fresh = tile_key(cur) != prev;
              kb = (kv_ord + (fresh ? 1 : 0)) % C::NKV;
            }
            ++u1;
            progressed = true;
          }
        }
        if (u2 < u1) {
          const int n2 = u2 / SUB, s2 = u2 % SUB;
          const int ob = n2 & 1;
          if (mbar_test_wait(&p_full[ob * SUB + s2], (n2 >> 1) & 1) &&
              (s2 > 0 || mbar_test_wait(&o_empty[ob], ((n2 >> 1) & 1) ^ 1))) {
            tc_fence_after();
            const int kb2 = (ring_kb >> (n2 & 3)) & 1;
            const uint32_t d_tmem = tmem_base + C::O_COL + ob * D;
            // P (bf16, two per column) sits over the first SK/2 columns of
            // this sub-tile's S; 16 keys = 8 columns per step
            const uint32_t p_tmem = tmem_base + C::S_COL + (u2 & 1) * SK;
            const uint32_t vbase = sKV_u + kb2 * C::KV_BYTES + 2 * C::KV_HALF + s2 * SK * C::ROW;
#pragma unroll
            for (int kk = 0; kk < SK / 16; ++kk) {
              const uint64_t bd = umma_desc_sw128_mn(vbase + kk * 16 * C::ROW, C::KV_HALF, 1024);
              umma_bf16_tmem_a(d_tmem, p_tmem + kk * 8, bd, IDESC2, (s2 != 0 || kk != 0) ? 1u : 0u);
            }
            umma_commit(&s_empty[u2 & 1]);   // P read: the S / P columns may take sub-tile u2 + NSB
            if (s2 == SUB - 1) {
              umma_commit(&o_full[ob]);
              if ((ring_last >> (n2 & 3)) & 1) umma_commit(&kv_empty[kb2]);
            } else {
              umma_commit(&pa_done[ob]);
            }
            ++u2;
            progressed = true;
          }
        }
        if (progressed) {
          spins = 0;
        } else if ((++spins & 255u) == 0) {
          const uint64_t now = global_timer_ns();
          if (spins == 256u) last_progress = now;
          if (*reinterpret_cast<volatile uint32_t*>(a.err) != 0) { ok = false; break; }
          if (now - last_progress > kWaitLimitNs) {
            atomicCAS(a.err, 0u, static_cast<uint32_t>(SITE_BLK_MMA_STALL));
            ok = false;
            break;
          }
        }
      }
      (void)ok;
      umma_commit(mma_done);
      const uint64_t tq = global_timer_ns();
      while (!mbar_try_wait(mma_done, 0) && global_timer_ns() - tq < kWaitLimitNs) {}
    }
  } else if (warp >= C::SW0) {
    // ------------------------------------------------------------ softmax + epilogue
    // Group g runs the softmax of tiles g, g + 2, ... and, after each, the
    // epilogue of the other group's previous tile, whose O is complete by
    // then: neither group waits on its own tile's P V.  A tile's S columns
    // take its P, and are free for the next tile of the same parity as soon
    // as P V has read them.
    const int grp = (warp - C::SW0) >> 2;
    const int eq = warp & 3;
    const int row = eq * 32 + lane;
    const int e = row / G, h = row % G;
    const uint32_t lane_base = static_cast<uint32_t>(eq * 32) << 16;
    // this warp's 32 staging rows (32 dims of each)
    uint8_t* stage = sStg + (grp * 4 + eq) * C::STG_WARP;
    auto tile_at = [&](int x) { return (x >= 0 && x < T) ? a.tiles[t0 + x] : none; };
    auto entry_of = [&](const int4& td) { return e < td.w ? __ldg(a.entries + td.z + e) : 0; };
    // the epilogue's tile descriptors two tiles ahead and this thread's entry
    // one tile ahead (epilogue tiles grp - 1 + 2k; the softmax needs neither:
    // every entry is a selected block, all of whose keys the row attends)
    int4 e_td = tile_at(grp - 1), e_td2 = tile_at(grp + 1);
    int e_ent = entry_of(e_td);
    bool ok = true;
    for (int ts = grp; ok; ts += 2) {
      const int te = ts - 1;
      if (ts >= T && te >= T) break;
      const int4 etd = e_td;
      const int eent = e_ent;
      e_td = e_td2; e_td2 = tile_at(te + 4);
      e_ent = entry_of(e_td);
      if (ts < T) {
        // ---------------- softmax of tile ts: P = 2^(x - m) in bf16 of the
        // scaled scores x over the S columns, one 128-key sub-tile after the
        // other.  A sub-tile's maximum over its two 64-key halves comes
        // first (one pass over S), then the powers and the row sums (a
        // second).  Barriers and the (m, l) slot go by tile parity (each
        // group waits on its own barriers, in order), S columns by sub-tile
        // parity.  A second sub-tile keeps the first one's maximum m unless
        // its own exceeds m by more than kStaleMax: then that row's m moves
        // up, and its O (complete for the first sub-tile) and l are rescaled.
        const int sb = ts & 1, use = ts >> 1;
        const bool single = pair_tile_c2(tile_at(ts).y) < 0;   // keys in the first BLK / 2 only
        // l sums P in float32 (the tile's log-sum-exp).  lr, the normaliser
        // of O, adds to it the bf16 rounding of each sub-tile's largest P:
        // P V multiplies the rounded P, so a key that dominates the row
        // divides out exactly (its P is 1 unless a kept maximum leaves it
        // anywhere in (1, 2^kStaleMax]); the other keys' roundings stay
        // below 2^-9 of their weights either way.
        float m = -INFINITY, l = 0.f, lr = 0.f;
        for (int s = 0; s < C::SUB; ++s) {
          ok = __all_sync(0xFFFFFFFFu, mbar_wait(&s_full[sb * C::SUB + s], use & 1, a.err, SITE_BLK_S_FULL));
          if (!ok) break;
          tc_fence_after();
          const uint32_t scol = tmem_base + lane_base + C::S_COL + ((ts * C::SUB + s) & 1) * C::SK;
          const int nhalf = !single ? 2 : (C::SUB == 2 ? (s == 0 ? 2 : 0) : 1);   // halves holding keys
          // maxima and sums in independent chains
          float mx[8] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY, -INFINITY, -INFINITY, -INFINITY, -INFINITY};
          float ls[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            if (hf >= nhalf) break;
            uint32_t r[64];
            tmem_ld64(scol + hf * 64, r);
#pragma unroll
            for (int u = 0; u < 64; ++u) mx[u & 7] = fmaxf(mx[u & 7], __uint_as_float(r[u]));
          }
          const float raw_max = max8(mx);
          const float mt = raw_max * a.scale_log2;
          if (s == 0) {
            m = mt;
          } else {
            const bool up = mt > m + kStaleMax;
            if (__any_sync(0xFFFFFFFFu, up)) {   // warp-uniform: the TMEM accesses are collective
              const float alpha = up ? fast_exp2(m - mt) : 1.f;
              if (up) m = mt;
              l *= alpha;
              lr *= alpha;
              ok = __all_sync(0xFFFFFFFFu, mbar_wait(&pa_done[sb], use & 1, a.err, SITE_BLK_O_FULL));
              if (!ok) break;
              tc_fence_after();
              const uint32_t ocol = tmem_base + lane_base + C::O_COL + sb * D;
#pragma unroll
              for (int hf = 0; hf < D / 64; ++hf) {
                uint32_t r[64];
                tmem_ld64(ocol + hf * 64, r);
#pragma unroll
                for (int u = 0; u < 64; ++u) r[u] = __float_as_uint(__uint_as_float(r[u]) * alpha);
#pragma unroll
                for (int q = 0; q < 4; ++q)
                  tmem_st16(ocol + hf * 64 + q * 16, *reinterpret_cast<const uint32_t(*)[16]>(&r[q * 16]));
              }
            }
          }
          // P of half hf goes to columns hf*32 .. hf*32+31: the S columns it
          // covers are already in registers (half 0) or consumed (half 1)
#pragma unroll
          for (int hf = 0; hf < 2; ++hf) {
            if (hf >= nhalf) {   // no keys: P = 0 over this half's 32 columns
              uint32_t pw[16];
#pragma unroll
              for (int u = 0; u < 16; ++u) pw[u] = 0u;
              tmem_st16(scol + hf * 32, pw);
              tmem_st16(scol + hf * 32 + 16, pw);
              continue;
            }
            uint32_t r[64];
            tmem_ld64(scol + hf * 64, r);
#pragma unroll
            for (int qq = 0; qq < 2; ++qq) {   // 32 keys = 16 columns of P per store
              uint32_t pw[16];
#pragma unroll
              for (int u = 0; u < 16; ++u) {
                const int c = qq * 32 + 2 * u;
                const float p0 = fast_exp2(fmaf(__uint_as_float(r[c]), a.scale_log2, -m));
                const float p1 = fast_exp2(fmaf(__uint_as_float(r[c + 1]), a.scale_log2, -m));
                ls[c & 7] += p0;
                ls[(c + 1) & 7] += p1;
                pw[u] = pack_bf16(p0, p1);
              }
              tmem_st16(scol + hf * 32 + qq * 16, pw);
            }
          }
          const float ps = ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
          // the sub-tile's largest P, computed as its element's own was
          const float pmax = nhalf > 0 ? fast_exp2(fmaf(raw_max, a.scale_log2, -m)) : 0.f;
          l += ps;
          lr += ps + (__bfloat162float(__float2bfloat16_rn(pmax)) - pmax);
          if (s == C::SUB - 1) {
            // (m, l) into this parity's slot once the epilogue two tiles back read it
            ok = __all_sync(0xFFFFFFFFu, mbar_wait(&ml_empty[sb], (use & 1) ^ 1, a.err, SITE_BLK_ML_EMPTY));
            if (!ok) break;
            tc_fence_after();
            sML[sb * 128 + row] = make_float4(m, l, lr, 0.f);
          }
          tmem_wait_st();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&p_full[sb * C::SUB + s]);
        }
        if (!ok) break;
      }
      if (te >= 0 && te < T) {
        // ---------------- epilogue of tile te: o = O / l as scaled float16
        const int ob = te & 1, use = te >> 1;
        const int bg = etd.x, ne = etd.w;
        const int i = entry_row(eent), j = entry_slot(eent);
        const bool valid = e < ne && static_cast<unsigned>(i) < static_cast<unsigned>(a.n_q) && j < a.topk;
        // the softmax's (m, l) are published with P (p_full); O follows P V
        ok = __all_sync(0xFFFFFFFFu, mbar_wait(&p_full[ob * C::SUB + C::SUB - 1], use & 1, a.err, SITE_BLK_O_FULL) &&
                                         mbar_wait(&o_full[ob], use & 1, a.err, SITE_BLK_O_FULL));
        if (!ok) break;
        tc_fence_after();
        const float4 ml = sML[ob * 128 + row];
        const float m = ml.x, l = ml.y, lr = ml.z;
        // (m, l) read: its slot may take the next tile of this parity
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ml_empty[ob]);
        // One pass over the row in halves of 64 dims: the normalised
        // o = O / lr of each half stored as float16 times 2^-e, the power of
        // two 2^e chosen per half so its largest entry lands in
        // [2^14, 2^15): 11 significant bits whatever the scale of V.  Every
        // lane runs the (warp-collective) TMEM loads; only valid rows store.
        const uint32_t ocol = tmem_base + lane_base + C::O_COL + ob * D;
        const float inv_l = 1.f / lr;
        const int64_t slot = ((static_cast<int64_t>(bg) * a.n_q + i) * a.nsl + j) * G + h;
        // Coalesced stores: the warp's 32 rows pass through its staging rows
        // 32 dims at a time (16-byte chunk c of row r at r * 64 +
        // 16 (c ^ ((r >> 1) & 3)), free of bank conflicts), then eight rows of
        // 64 bytes go out per instruction.  Lane l stores rows 8 k + l / 4.
        const int srow = lane >> 2, sch = lane & 3;
        int64_t rslot[4];
        bool rvalid[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          rslot[k] = __shfl_sync(0xFFFFFFFFu, slot, k * 8 + srow);
          rvalid[k] = __shfl_sync(0xFFFFFFFFu, valid ? 1 : 0, k * 8 + srow) != 0;
        }
        uint32_t exs = 0;   // the two halves' exponents, 16 bits each
#pragma unroll
        for (int hf = 0; hf < D / 64; ++hf) {
          uint32_t r[64];
          tmem_ld64(ocol + hf * 64, r);
          if (hf == D / 64 - 1) {   // all of O is in registers: free the buffer
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&o_empty[ob]);
          }
          float am[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int x = 0; x < 64; ++x) am[x & 7] = fmaxf(am[x & 7], fabsf(__uint_as_float(r[x])));
          const float xm = max8(am) * inv_l;
          int ex = xm > 0.f ? static_cast<int>((__float_as_uint(xm) >> 23) & 0xFFu) - 127 - 14 : 0;
          ex = min(max(ex, -100), 100);
          exs |= (static_cast<uint32_t>(ex) & 0xFFFFu) << (16 * hf);
          const float mul = inv_l * __uint_as_float(static_cast<uint32_t>(127 - ex) << 23);
#pragma unroll
          for (int qh = 0; qh < 2; ++qh) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {   // 8 dims = 16 bytes
              uint32_t w[4];
#pragma unroll
              for (int u = 0; u < 4; ++u) {
                const int c = qh * 32 + q * 8 + 2 * u;
                const __half2 hv = __floats2half2_rn(__uint_as_float(r[c]) * mul, __uint_as_float(r[c + 1]) * mul);
                w[u] = *reinterpret_cast<const uint32_t*>(&hv);
              }
              *reinterpret_cast<uint4*>(stage + lane * 64 + ((q ^ ((lane >> 1) & 3)) << 4)) =
                  make_uint4(w[0], w[1], w[2], w[3]);
            }
            __syncwarp();
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int rr = k * 8 + srow;
              const uint4 v = *reinterpret_cast<const uint4*>(stage + rr * 64 + ((sch ^ ((rr >> 1) & 3)) << 4));
              if (rvalid[k]) reinterpret_cast<uint4*>(a.partO + rslot[k] * D + hf * 64 + qh * 32)[sch] = v;
            }
            __syncwarp();
          }
        }
        if (valid) a.partL[slot] = make_float2(m + log2f(l), __uint_as_float(exs));
      }
    }
  } else {
    // ------------------------------------------------------------ Q gather
    const int q = warp - 2;   // tiles q, q + NGW, ... into buffers lt % NA
    bool ok = true;
    int4 nxt = q < T ? a.tiles[t0 + q] : none;
    int4 nxt2 = q + C::NGW < T ? a.tiles[t0 + q + C::NGW] : none;   // two ahead (TMA path)
    // the next tile's entries, entry j in register j / 32 of lane j % 32
    constexpr int NEN = (QPT + 31) / 32;
    int nen[NEN];
    auto load_entries = [&](const int4& td) {
#pragma unroll
      for (int k = 0; k < NEN; ++k) nen[k] = lane + 32 * k < td.w ? __ldg(a.entries + td.z + 32 * k + lane) : 0;
    };
    load_entries(nxt);
    int last_lt = -1;
    for (int lt = q; lt < T && ok; lt += C::NGW) {
      const int ab = lt % NA;
      const uint32_t use = static_cast<uint32_t>(lt / NA);
      const int4 td = nxt;
      int en[NEN];
#pragma unroll
      for (int k = 0; k < NEN; ++k) en[k] = nen[k];
      const int b = td.x / a.h_kv, g = td.x % a.h_kv, ne = td.w;
      if (lane == 0) ok = mbar_wait(&a_empty[ab], (use & 1) ^ 1, a.err, SITE_BLK_A_EMPTY);
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (!ok) break;
      last_lt = lt;
      uint8_t* abuf = sA + ab * C::A_BYTES;
      if (C::TMA_Q) {
        // an entry's 8 query heads are 8 tensor-core rows = one 1024-byte
        // swizzle atom per 64-dim half: lane e issues entry e's two TMA boxes
        if (lane == 0) mbar_arrive_expect_tx(&a_full[ab], static_cast<uint32_t>(ne) * G * D * 2);
        __syncwarp();
        if (lane < ne) {
          const int i = entry_row(en[0]);
          if (static_cast<unsigned>(i) < static_cast<unsigned>(a.n_q)) {
            const int z = static_cast<int>(static_cast<int64_t>(b) * a.n_q + i);
#pragma unroll
            for (int hf = 0; hf < 2; ++hf)
              tma_load_3d(abuf + hf * C::A_HALF + lane * (G * C::ROW), &tmQ, &a_full[ab], hf * 64, g * G, z);
          } else {   // never for a consistent plan; the tile's wait then times out
            atomicCAS(a.err, 0u, static_cast<uint32_t>(SITE_BLK_BAD_ENTRY));
          }
        }
        nxt = nxt2;
        nxt2 = lt + 2 * C::NGW < T ? a.tiles[t0 + lt + 2 * C::NGW] : none;
        load_entries(nxt);
      } else {
        const uint32_t abase = smem_u32(abuf);
        // an entry is G rows of 16 chunks of 8 dims; a warp instruction
        // copies 32 chunks: one entry's (G >= 2) or two entries' (G = 1)
        constexpr int CPE = G * 16;
        constexpr int EPI = CPE >= 32 ? 1 : 32 / CPE;
        for (int ee0 = 0; ee0 < ne; ee0 += EPI) {
          const int ee = ee0 + (EPI > 1 ? lane / CPE : 0);   // ee0 and ee share a register: ee0 is even
          int reg = en[0];
#pragma unroll
          for (int k = 1; k < NEN; ++k) reg = (ee0 >> 5) == k ? en[k] : reg;
          const int ent = __shfl_sync(0xFFFFFFFFu, reg, ee & 31);
          const int i = entry_row(ent);
          const bool live = ee < ne;
          const bool row_ok = static_cast<unsigned>(i) < static_cast<unsigned>(a.n_q);
          if (live && !row_ok) atomicCAS(a.err, 0u, static_cast<uint32_t>(SITE_BLK_BAD_ENTRY));   // never for a consistent plan
          if (!live || !row_ok) continue;
          const __nv_bfloat16* qrow = a.Q + ((static_cast<int64_t>(b) * a.n_q + i) * a.h_q +
                                             static_cast<int64_t>(g) * G) * D;
#pragma unroll
          for (int x = (EPI > 1 ? lane % CPE : lane); x < CPE; x += (EPI > 1 ? CPE : 32)) {
            const int hh = x >> 4, ch = x & 15;
            const int r = ee * G + hh;
            const uint32_t dst = abase + (ch >> 3) * C::A_HALF + r * C::ROW + (((ch & 7) ^ (r & 7)) << 4);
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(qrow + hh * D + ch * 8)
                         : "memory");
          }
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
        // this warp's next tile: descriptor and entries load while the copies fly
        nxt = lt + C::NGW < T ? a.tiles[t0 + lt + C::NGW] : none;
        load_entries(nxt);
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        fence_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&a_full[ab]);
      }
    }
    if (C::TMA_Q) {
      // after a failure, let the TMA boxes of the buffers in flight land before
      // the CTA exits
      if (!ok && lane == 0) {
        const uint64_t tq = global_timer_ns();
        for (int lt = (last_lt - NA + 1 > 0 ? last_lt - NA + 1 : 0); lt <= last_lt; ++lt)
          while (!mbar_try_wait(&a_full[lt % NA], (lt / NA) & 1) && global_timer_ns() - tq < kWaitLimitNs) {}
      }
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// ------------------------------------------------------------------ merge
//
// One warp per (query, kv-head) item: the item's slots are recomputed from
// its block_idx row (same rule as the inversion), and the normalised slot
// partials o_j with base-2 log-sum-exps L_j combine into the softmax over
// the union of their keys: o = sum_j 2^(L_j - M) o_j / sum_j 2^(L_j - M),
// lse = (M + log2 sum_j 2^(L_j - M)) ln 2, with M the largest L_j.

struct MergeArgs {
  const uint32_t* win;       // [items] uncovered window blocks (from the plan)
  const uint2* rowinfo;      // [items] {selected-slot mask, skipped block_idx entries}
  const __half* partO;
  const float2* partL;
  __nv_bfloat16* O;
  float* lse;
  int32_t* bad;
  int32_t n_q, h_q, h_kv, nb, block, topk, window, nsl;
  int64_t q_offset, n_items;
};

// Latency bound on its partial loads: the register cap keeps at least
// 16 (G = 8) / 24 / 32 warps per SM resident.
template <int G>
__global__ void __launch_bounds__(256, (G == 8 ? 2 : (G == 4 ? 3 : 4))) attn_merge_kernel(const MergeArgs a) {
  constexpr int D = 128;
  const int lane = threadIdx.x & 31;
  const int64_t item = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (item >= a.n_items) return;   // warp-uniform
  const int it32 = static_cast<int>(item);   // items (b * h_kv * n_q) fit 31 bits
  const int i = it32 % a.n_q;
  const int bg = it32 / a.n_q;
  const int b = bg / a.h_kv, g = bg % a.h_kv;
  // the row's slots as the plan recorded them: selected slots (bit j) and,
  // from its uncovered window blocks, the window chunks (slots topk + c)
  // that hold keys, one lane each
  const uint2 ri = __ldg(a.rowinfo + item);
  const uint32_t win = __ldg(a.win + item);
  if (lane == 0 && a.bad && ri.y) atomicAdd(a.bad, static_cast<int>(ri.y));
  const uint32_t wch = __ballot_sync(0xFFFFFFFFu, lane < a.nsl - a.topk &&
                                                      chunk_has_keys(win, a.q_offset + i, a.window, a.block, lane,
                                                                     win_chunk(G)));
  struct { uint64_t mask; } s;
  s.mask = static_cast<uint64_t>(ri.x) | (static_cast<uint64_t>(wch) << a.topk);
  const float2* pl = a.partL + item * a.nsl * G;
  const __half* po = a.partO + item * a.nsl * G * D;
  // Per head, the slots' weights 2^(L - M) 2^e, e the slot's exponent for
  // the 64-dim half this lane accumulates (lanes 0-15: dims 0-63, lanes
  // 16-31: dims 64-127): lane i of each 16-lane half holds slots i, i + 16,
  // i + 32, i + 48, so one 16-wide shuffle hands every lane the weight of
  // its own half.
  const int li = lane & 15, eshift = (lane >> 4) * 16;
  float w[4][G], inv_den[G], lse2[G];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    float2 lv[4];
    bool hv[4];
    float M = -INFINITY;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int j = li + 16 * k;
      hv[k] = (s.mask >> j) & 1;
      lv[k] = hv[k] ? pl[j * G + h] : make_float2(-INFINITY, 0.f);
      M = fmaxf(M, lv[k].x);
    }
#pragma unroll
    for (int o = 8; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xFFFFFFFFu, M, o));
    float den = 0.f;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float f = hv[k] ? fast_exp2(lv[k].x - M) : 0.f;
      den += f;
      const int e = static_cast<int16_t>((__float_as_uint(lv[k].y) >> eshift) & 0xFFFFu);   // |e| <= 100
      w[k][h] = f * __uint_as_float(static_cast<uint32_t>(127 + e) << 23);
    }
#pragma unroll
    for (int o = 8; o; o >>= 1) den += __shfl_xor_sync(0xFFFFFFFFu, den, o);
    inv_den[h] = 1.f / den;
    lse2[h] = M + log2f(den);
  }
  // every lane accumulates dims 4 lane .. 4 lane + 3 of every head, SU
  // slots at a time (loads of SU x G rows in flight)
  constexpr int SU = G == 8 ? 2 : (G == 4 ? 3 : 4);
  float acc[G][4];
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int u = 0; u < 4; ++u) acc[h][u] = 0.f;
  uint64_t m = s.mask;
  while (m) {
    int js[SU];
#pragma unroll
    for (int q = 0; q < SU; ++q) {
      js[q] = m ? __ffsll(static_cast<long long>(m)) - 1 : -1;
      m &= m - 1;
    }
    uint2 raw[SU][G];
#pragma unroll
    for (int q = 0; q < SU; ++q)
#pragma unroll
      for (int h = 0; h < G; ++h)
        raw[q][h] = js[q] >= 0 ? __ldg(reinterpret_cast<const uint2*>(po + (js[q] * G + h) * D) + lane)
                               : make_uint2(0u, 0u);
#pragma unroll
    for (int q = 0; q < SU; ++q) {
      if (js[q] < 0) break;   // warp-uniform
      const int src = js[q] & 15, grp16 = js[q] >> 4;   // warp-uniform
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float wg = w[0][h];
#pragma unroll
        for (int k = 1; k < 4; ++k) wg = grp16 == k ? w[k][h] : wg;
        const float wj = __shfl_sync(0xFFFFFFFFu, wg, src, 16);
        const float2 o01 = __half22float2(*reinterpret_cast<const __half2*>(&raw[q][h].x));
        const float2 o23 = __half22float2(*reinterpret_cast<const __half2*>(&raw[q][h].y));
        acc[h][0] += wj * o01.x;
        acc[h][1] += wj * o01.y;
        acc[h][2] += wj * o23.x;
        acc[h][3] += wj * o23.y;
      }
    }
  }
  const int64_t qrow = (static_cast<int64_t>(b) * a.n_q + i) * a.h_q + static_cast<int64_t>(g) * G;
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const uint32_t lo = pack_bf16(acc[h][0] * inv_den[h], acc[h][1] * inv_den[h]);
    const uint32_t hi = pack_bf16(acc[h][2] * inv_den[h], acc[h][3] * inv_den[h]);
    reinterpret_cast<uint2*>(a.O + (qrow + h) * D)[lane] = make_uint2(lo, hi);
  }
  if (a.lse && lane < G) {
    float x = lse2[0];
#pragma unroll
    for (int h = 1; h < G; ++h) x = lane == h ? lse2[h] : x;
    a.lse[qrow + lane] = x * 0.69314718055994531f;
  }
}

template <int G, int BLK>
cudaError_t run_block(const CUtensorMap& tmK, const CUtensorMap& tmV, const CUtensorMap& tmQ, const BlkArgs& a,
                      const LaunchCtx& c) {
  using C = BlkCfg<G, BLK>;
  cudaError_t e = cudaFuncSetAttribute(attn_block_kernel<G, BLK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::SMEM);
  if (e != cudaSuccess) return e;
  attn_block_kernel<G, BLK><<<c.sm_count, C::THREADS, C::SMEM, c.stream>>>(tmK, tmV, tmQ, a);
  note_launch();
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_merge(const ssa_params& p, const uint32_t* win, const uint2* rowinfo,
                              const void* partO, const void* partL, void* O, float* lse, int32_t* bad,
                              const LaunchCtx& c) {
  MergeArgs a;
  a.win = win;
  a.rowinfo = rowinfo;
  a.partO = static_cast<const __half*>(partO);
  a.partL = static_cast<const float2*>(partL);
  a.O = static_cast<__nv_bfloat16*>(O);
  a.lse = lse;
  a.bad = bad;
  a.n_q = p.n_q; a.h_q = p.h_q; a.h_kv = p.h_kv; a.nb = p.n_kv / p.block; a.block = p.block; a.topk = p.topk;
  a.window = p.window;
  a.nsl = p.topk + window_chunks(p.window, p.h_q / p.h_kv);
  a.q_offset = p.q_offset;
  a.n_items = static_cast<int64_t>(p.batch) * p.h_kv * p.n_q;
  if (p.d != 128) return cudaErrorInvalidValue;
  const unsigned grid = static_cast<unsigned>((a.n_items + 7) / 8);
  switch (p.h_q / p.h_kv) {
    case 1: attn_merge_kernel<1><<<grid, 256, 0, c.stream>>>(a); break;
    case 2: attn_merge_kernel<2><<<grid, 256, 0, c.stream>>>(a); break;
    case 4: attn_merge_kernel<4><<<grid, 256, 0, c.stream>>>(a); break;
    case 8: attn_merge_kernel<8><<<grid, 256, 0, c.stream>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  note_launch();
  return cudaGetLastError();
}


cudaError_t launch_block_plan(const ssa_params& p, const int32_t* block_idx, const BlockPlan& pl,
                              const LaunchCtx& c) {
  const int blk_smem = pl.nb * static_cast<int>(sizeof(int32_t));
  const int key_smem = pl.nkey * static_cast<int>(sizeof(int32_t));
  cudaError_t e = cudaFuncSetAttribute(inv_hist_kernel<0>, cudaFuncAttributeMaxDynamicSharedMemorySize, blk_smem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(inv_hist_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, blk_smem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(inv_hist_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, key_smem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(inv_hot_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, blk_smem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(inv_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, key_smem);
  if (e != cudaSuccess) return e;
  const dim3 rows(static_cast<unsigned>(pl.nchunk), static_cast<unsigned>(pl.bgs));
  const unsigned cols = static_cast<unsigned>((static_cast<int64_t>(pl.bgs) * pl.nkey + 255) / 256);
  // per-block counts and window blocks; in pair mode sampled per-block
  // counts, the hot sets, then the counts per tile key and window blocks
  if (pl.pair) {
    e = cudaMemsetAsync(pl.count, 0, static_cast<size_t>(pl.bgs) * pl.nb * sizeof(int32_t), c.stream);
    if (e != cudaSuccess) return e;
    inv_hist_kernel<1><<<rows, kPlanThreads, blk_smem, c.stream>>>(pl, block_idx);
    note_launch();
    inv_hot_kernel<<<pl.bgs, 1024, blk_smem, c.stream>>>(pl);
    note_launch();
    inv_hist_kernel<2><<<rows, kPlanThreads, key_smem, c.stream>>>(pl, block_idx);
    note_launch();
  } else {
    inv_hist_kernel<0><<<rows, kPlanThreads, blk_smem, c.stream>>>(pl, block_idx);
    note_launch();
  }
  inv_colscan_kernel<<<cols, 256, 0, c.stream>>>(pl);
  note_launch();
  inv_scan_kernel<<<pl.bgs, 1024, 0, c.stream>>>(pl);
  note_launch();
  inv_scan_bg_kernel<<<1, 32, 0, c.stream>>>(pl);
  note_launch();
  inv_scatter_kernel<<<rows, kPlanThreads, key_smem, c.stream>>>(pl, block_idx);
  note_launch();
  inv_tiles_kernel<<<static_cast<unsigned>((static_cast<int64_t>(pl.bgs) * pl.nkey * 32 + 255) / 256), 256, 0,
                     c.stream>>>(pl);
  note_launch();
  if (pl.grid < 1 || pl.grid > kMaxBlockGrid) return cudaErrorInvalidValue;
  const int n_chunks = (pl.max_tiles + 255) / 256;
  // one K/V buffer: a new tile key costs two tiles
  inv_cost_kernel<<<n_chunks, 256, 0, c.stream>>>(pl, 8);
  note_launch();
  inv_split_kernel<<<1, 1024, 0, c.stream>>>(pl, n_chunks);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_attn_block(const ssa_params& p, const BlockPlan& pl, const void* Q,
                              const CUtensorMap& tmK, const CUtensorMap& tmV, const CUtensorMap& tmQ,
                              void* partO, void* partL, const LaunchCtx& c) {
  BlkArgs a;
  a.Q = static_cast<const __nv_bfloat16*>(Q);
  a.tiles = pl.tiles;
  a.t_start = pl.t_start;
  a.entries = pl.entries;
  a.n_q = p.n_q; a.n_kv = p.n_kv; a.h_q = p.h_q; a.h_kv = p.h_kv; a.topk = p.topk; a.window = p.window;
  a.nsl = p.topk + window_chunks(p.window, p.h_q / p.h_kv);
  a.q_offset = p.q_offset;
  a.scale_log2 = p.scale * 1.4426950408889634f;
  a.partO = static_cast<__half*>(partO);
  a.partL = static_cast<float2*>(partL);
  a.err = c.err;
  const int G = p.h_q / p.h_kv;
  if (p.d != 128) return cudaErrorInvalidValue;
  // tiles hold pairs of blocks: 128 keys for 64-key blocks, 256 for 128-key blocks
  if (!pl.pair) return cudaErrorInvalidValue;
  if (p.block == 64) {
    if (G == 1) return run_block<1, 128>(tmK, tmV, tmQ, a, c);
    if (G == 2) return run_block<2, 128>(tmK, tmV, tmQ, a, c);
    if (G == 4) return run_block<4, 128>(tmK, tmV, tmQ, a, c);
    if (G == 8) return run_block<8, 128>(tmK, tmV, tmQ, a, c);
  } else if (p.block == 128) {
    if (G == 1) return run_block<1, 256>(tmK, tmV, tmQ, a, c);
    if (G == 2) return run_block<2, 256>(tmK, tmV, tmQ, a, c);
    if (G == 4) return run_block<4, 256>(tmK, tmV, tmQ, a, c);
    if (G == 8) return run_block<8, 256>(tmK, tmV, tmQ, a, c);
  }
  return cudaErrorInvalidValue;
}

}  // namespace ssa

// Block-major attention, the causal window: step (ii) of the layer, "a
// local window" of the W keys pos-W+1 .. pos ["Subquadratic Sparse Attention
// (SSA)", opening section], evaluated densely for runs of consecutive
// queries.
//
// A tile is the 128 tensor-core rows of 128/G consecutive queries x the G
// query heads of one kv-head, for one window chunk s (keys pos-W+1 + C s ..
// min(pos, pos-W + C (s+1)) of each row, C = 256 keys, 128 when G = 1).  The
// chunks of the tile's rows together span at most C + 128/G - 1 keys, six
// 64-key blocks: S = Q K^T
// over the whole span fits 384 TMEM columns next to the 128 of O, so the
// softmax needs no rescaling.  Each row masks the keys outside its own chunk
// and the keys of blocks it already attends through its selected slots (the
// row's uncovered window blocks come from the plan), and the tile writes one
// normalised partial per (row, chunk) in the block kernel's format (slot
// topk + s), for the merge.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <math.h>

#include "common.cuh"
#include "invert.cuh"
#include "kernels.h"

namespace ssa {
namespace {

template <int G>
struct WinCfg {
  static constexpr int D = 128;
  static constexpr int QT = 128 / G;                 // queries per tile
  static constexpr int ROW = 128;                    // bytes per 64-wide swizzled row
  static constexpr int Q_HALF = 128 * ROW;           // 128 rows x 64 dims
  static constexpr int KB = 6;                       // 64-key blocks per tile, at most
  static constexpr int K_BLK = 64 * ROW;             // one 64-key block, one 64-dim half
  static constexpr int K_HALF = KB * K_BLK;          // half h of all K blocks, block kb at kb * K_BLK
  static constexpr int V_SLOT = 2 * K_BLK;           // one V block, both halves (LBO = K_BLK)
  static constexpr int NBAR = 14;
  static constexpr int XCH = 2 * 2 * 128 * 4;         // two buffers of one float per (group, row)
  // bytes used from the 1024-byte-aligned base; the allocation adds what
  // alignment may cost, up to the per-block limit (checked in the kernel)
  static constexpr int USED = 2 * Q_HALF + 2 * K_HALF + KB * V_SLOT + XCH + NBAR * 8 + 16;
  static constexpr int SMEM = USED + 1024 < 232448 ? USED + 1024 : 232448;
  static constexpr int THREADS = 448;                // producer, MMA, 2 x 4 softmax, 4 epilogue warps
  static constexpr int S_COL = 0;                    // TMEM: S (KB * 64 columns), then O
  static constexpr int O_COL = KB * 64;
  static constexpr int ML_COL = S_COL + 32;          // (m, l): in the first block's S, past its P
  static_assert(O_COL + D <= 512, "tensor memory");
  static_assert(USED <= 232448, "shared memory");
};

struct WinArgs {
  const uint32_t* win;       // [bgs * n_q] uncovered window blocks of each row
  int32_t n_q, n_kv, h_q, h_kv, block, topk, window, nsl, nwc, n_qt;
  int64_t q_offset;
  int32_t n_tiles;           // bgs * n_qt * nwc
  float scale_log2;
  __half* partO;             // [items][nsl][G][D], o / 2^e per 64-dim half
  float2* partL;             // [items][nsl][G]: (log2-sum-exp, e0 | e1 << 16 as int16s)
  uint32_t* err;
};

// A tile's place and key span; kb0 < 0 when no row of it has keys in the
// chunk (every role skips such tiles alike).
struct WinTile {
  int bg, q0, s, kb0, nkb;
};

template <int G>
__device__ __forceinline__ WinTile win_tile(const WinArgs& a, int t) {
  constexpr int QT = WinCfg<G>::QT;
  WinTile w;
  const int per_bg = a.n_qt * a.nwc;
  w.bg = t / per_bg;
  const int r = t % per_bg;
  w.q0 = (r / a.nwc) * QT;
  w.s = r % a.nwc;
  const int64_t p0 = a.q_offset + w.q0;
  const int64_t pl = a.q_offset + min(w.q0 + QT, a.n_q) - 1;
  constexpr int CH = win_chunk(G);
  int64_t lo = p0 - a.window + 1 + static_cast<int64_t>(w.s) * CH;
  int64_t hi = pl - a.window + static_cast<int64_t>(w.s + 1) * CH;
  if (lo < 0) lo = 0;
  if (hi > pl) hi = pl;
  if (hi < lo) {
    w.kb0 = -1;
    w.nkb = 0;
  } else {
    w.kb0 = static_cast<int>(lo / 64);
    w.nkb = static_cast<int>(hi / 64) - w.kb0 + 1;
  }
  return w;
}

__device__ __forceinline__ uint64_t win_desc_mn(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}

__device__ __forceinline__ void win_ld32(uint32_t taddr, uint32_t (&r)[32]) {
#pragma unroll
  for (int q = 0; q < 2; ++q) tmem_ld16(taddr + q * 16, *reinterpret_cast<uint32_t(*)[16]>(&r[q * 16]));
  tmem_wait_ld();
  tmem_regs_ready(r);
}

__device__ __forceinline__ void win_ld64(uint32_t taddr, uint32_t (&r)[64]) {
#pragma unroll
  for (int q = 0; q < 4; ++q) tmem_ld16(taddr + q * 16, *reinterpret_cast<uint32_t(*)[16]>(&r[q * 16]));
  tmem_wait_ld();
  tmem_regs_ready(r);
}

// Warp roles: 0 TMA producer (Q, then K, then V of each tile), 1 MMA issuer
// and TMEM owner, 2..9 softmax in two groups of four warps (one tensor-core
// row = one (query, head) pair per thread of each group; group g takes half
// of the tile's 64-key blocks, and the groups swap each row's maximum and
// sum through shared memory), 10..13 epilogue.  The epilogue of a tile runs
// while the softmax works on the next: the next tile's Q and K load during
// this tile's softmax, its S runs once this tile's P V has read P (which
// lies over S); the epilogue stages its stores through the first V slot, so
// the next tile's V loads after it.
template <int G>
__global__ void __launch_bounds__(WinCfg<G>::THREADS, 1)
    attn_window_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                       const __grid_constant__ CUtensorMap tmV, const WinArgs a) {
  using C = WinCfg<G>;
  constexpr int D = C::D;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  if (static_cast<int>(smem - smem_raw) + C::USED > C::SMEM) {   // never with a 1024-aligned base
    if (threadIdx.x == 0) atomicCAS(a.err, 0u, static_cast<uint32_t>(SITE_WIN_SMEM));
    return;
  }
  uint8_t* sQ = smem;                                  // [2 halves][128 rows][128 B]
  uint8_t* sK = sQ + 2 * C::Q_HALF;                    // [2 halves][KB blocks][64 keys][128 B]
  uint8_t* sV = sK + 2 * C::K_HALF;                    // [KB blocks][2 halves][64 keys][128 B]
  float* xch = reinterpret_cast<float*>(sV + C::KB * C::V_SLOT);   // [2 buffers][2 groups][128 rows]
  uint64_t* bars = reinterpret_cast<uint64_t*>(xch + 2 * 2 * 128);
  uint64_t* q_full = bars + 0;
  uint64_t* q_empty = bars + 1;     // S done: Q and K free
  uint64_t* k_full = bars + 2;
  uint64_t* v_full = bars + 3;
  uint64_t* s_full = bars + 4;
  uint64_t* p_full = bars + 5;
  uint64_t* o_full = bars + 6;      // P V done
  uint64_t* o_empty = bars + 7;     // the epilogue has read O
  uint64_t* stg_done = bars + 8;    // the epilogue's staging rows are written out (V slot 0 free)
  uint64_t* xbar = bars + 9;        // [2] both softmax groups' row partials of a tile written
  uint64_t* ml_full = bars + 11;    // (m, l) of the tile written to TMEM
  uint64_t* ml_read = bars + 12;    // ... and read by the epilogue (its columns may take S)
  uint64_t* mma_done = bars + 13;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 14);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1); mbar_init(q_empty, 1); mbar_init(k_full, 1); mbar_init(v_full, 1);
    mbar_init(s_full, 1); mbar_init(p_full, 8); mbar_init(o_full, 1); mbar_init(o_empty, 4);
    mbar_init(stg_done, 4);
    mbar_init(&xbar[0], 8); mbar_init(&xbar[1], 8);
    mbar_init(ml_full, 4); mbar_init(ml_read, 4);
    mbar_init(mma_done, 1);
    fence_barrier_init();
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t u = 0, uqk = 0, uv = 0;   // tiles started; with Q, K issued; with V issued
      bool ok = true;
      for (int t = blockIdx.x; t < a.n_tiles && ok; t += gridDim.x) {
        const WinTile w = win_tile<G>(a, t);
        if (w.kb0 < 0) continue;
        const int b = w.bg / a.h_kv, g = w.bg % a.h_kv;
        const uint32_t par = (u & 1) ^ 1;
        // Q and K of this tile once the previous tile's S has read them
        if (!mbar_wait(q_empty, par, a.err, SITE_WIN_PRODUCER)) { ok = false; break; }
        mbar_arrive_expect_tx(q_full, 2 * C::Q_HALF);
        const int qz = b * a.n_q + w.q0;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) tma_load_3d(sQ + hf * C::Q_HALF, &tmQ, q_full, hf * 64, g * G, qz);
        mbar_arrive_expect_tx(k_full, static_cast<uint32_t>(w.nkb) * 2 * C::K_BLK);
        const int kz = b * a.n_kv + w.kb0 * 64;
        for (int kb = 0; kb < w.nkb; ++kb)
#pragma unroll
          for (int hf = 0; hf < 2; ++hf)
            tma_load_3d(sK + hf * C::K_HALF + kb * C::K_BLK, &tmK, k_full, hf * 64, g, kz + kb * 64);
        ++uqk;
        // V once the previous tile's epilogue has left the staging rows
        if (!mbar_wait(stg_done, par, a.err, SITE_WIN_PRODUCER)) { ok = false; break; }
        mbar_arrive_expect_tx(v_full, static_cast<uint32_t>(w.nkb) * C::V_SLOT);
        for (int kb = 0; kb < w.nkb; ++kb)
#pragma unroll
          for (int hf = 0; hf < 2; ++hf)
            tma_load_3d(sV + kb * C::V_SLOT + hf * C::K_BLK, &tmV, v_full, hf * 64, g, kz + kb * 64);
        ++uv;
        ++u;
      }
      if (!ok) {   // let issued copies land before the CTA exits
        const uint64_t tq = global_timer_ns();
        if (uqk > 0) {
          while (!mbar_try_wait(q_full, (uqk - 1) & 1) && global_timer_ns() - tq < kWaitLimitNs) {}
          while (!mbar_try_wait(k_full, (uqk - 1) & 1) && global_timer_ns() - tq < kWaitLimitNs) {}
        }
        if (uv > 0)
          while (!mbar_try_wait(v_full, (uv - 1) & 1) && global_timer_ns() - tq < kWaitLimitNs) {}
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t IDESC_PV = umma_idesc_bf16(128, D) | (1u << 16);   // V is MN-major
      const uint32_t sQ_u = smem_u32(sQ), sK_u = smem_u32(sK), sV_u = smem_u32(sV);
      uint32_t u = 0;
      for (int t = blockIdx.x; t < a.n_tiles; t += gridDim.x) {
        const WinTile w = win_tile<G>(a, t);
        if (w.kb0 < 0) continue;
        const uint32_t par = u & 1;
        // S over the span: the previous tile's P V has read its P and the
        // epilogue its (m, l), both over S
        if (!mbar_wait(o_full, par ^ 1, a.err, SITE_WIN_MMA) || !mbar_wait(ml_read, par ^ 1, a.err, SITE_WIN_MMA) ||
            !mbar_wait(q_full, par, a.err, SITE_WIN_MMA) || !mbar_wait(k_full, par, a.err, SITE_WIN_MMA))
          break;
        tc_fence_after();
        // the span's first four blocks (N = 256) and the rest (N = 64 or
        // 128) go to separate accumulators: their K-steps alternate, so one
        // product runs while the other waits for its previous step
        const uint32_t idesc_hi = umma_idesc_bf16(128, 64 * max(w.nkb - 4, 1));
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint64_t ad = umma_desc_sw128(sQ_u + (ks >> 2) * C::Q_HALF + (ks & 3) * 32);
#pragma unroll
          for (int n0 = 0; n0 < C::KB; n0 += 4) {
            if (n0 >= w.nkb) break;
            const uint32_t idesc = n0 == 0 ? umma_idesc_bf16(128, 64 * min(4, w.nkb)) : idesc_hi;
            const uint64_t bd = umma_desc_sw128(sK_u + (ks >> 2) * C::K_HALF + n0 * C::K_BLK + (ks & 3) * 32);
            umma_bf16(tmem_base + C::S_COL + n0 * 64, ad, bd, idesc, ks != 0 ? 1u : 0u);
          }
        }
        umma_commit(s_full);
        umma_commit(q_empty);
        // O = P V: P (bf16, two per column) over the first 32 columns of each
        // block's 64 S columns; the previous tile's epilogue has read O
        if (!mbar_wait(p_full, par, a.err, SITE_WIN_MMA) || !mbar_wait(o_empty, par ^ 1, a.err, SITE_WIN_MMA) ||
            !mbar_wait(v_full, par, a.err, SITE_WIN_MMA))
          break;
        tc_fence_after();
        for (int kb = 0; kb < w.nkb; ++kb) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t bd = win_desc_mn(sV_u + kb * C::V_SLOT + kk * 16 * C::ROW, C::K_BLK, 1024);
            umma_bf16_tmem_a(tmem_base + C::O_COL, tmem_base + C::S_COL + kb * 64 + kk * 8, bd, IDESC_PV,
                             (kb | kk) != 0 ? 1u : 0u);
          }
        }
        umma_commit(o_full);
        ++u;
      }
      umma_commit(mma_done);   // all issued MMAs complete before TMEM is freed
      const uint64_t tq = global_timer_ns();
      while (!mbar_try_wait(mma_done, 0) && global_timer_ns() - tq < kWaitLimitNs) {}
    }
  } else if (warp < 10) {
    // ------------------------------------------------------------ softmax
    const int gs = (warp - 2) >> 2;   // this group's half of the tile's blocks
    const int eq = warp & 3;
    const int row = eq * 32 + lane;
    const int e = row / G;
    const uint32_t lane_base = static_cast<uint32_t>(eq * 32) << 16;
    const uint32_t scol = tmem_base + lane_base + C::S_COL;
    // publish this thread's row partial, then read the other group's once
    // both groups have published (bounded waits; the phase is the tile
    // count).  Exchanges alternate between two buffers: a buffer is written
    // again only after every warp has passed the exchange in between, so
    // after every warp has read it.
    uint32_t nx = 0;
    auto swap = [&](int k, float v, uint32_t par, bool& ok) {
      float* buf = xch + (nx++ & 1) * 256;
      buf[gs * 128 + row] = v;
      __syncwarp();
      if (lane == 0) mbar_arrive(&xbar[k]);
      ok = __all_sync(0xFFFFFFFFu, mbar_wait(&xbar[k], par, a.err, SITE_WIN_SOFTMAX));
      return buf[(gs ^ 1) * 128 + row];
    };
    uint32_t u = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < a.n_tiles && ok; t += gridDim.x) {
      const WinTile w = win_tile<G>(a, t);
      if (w.kb0 < 0) continue;
      const uint32_t par = u & 1;
      const int kbh = (w.nkb + 1) >> 1;
      const int kb_lo = gs ? kbh : 0, kb_hi = gs ? w.nkb : kbh;
      const int i = w.q0 + e;
      const bool valid = i < a.n_q;
      // this row's keys: its chunk of the window, minus the blocks it
      // selected, as offsets from the span's first key (key positions are
      // below 2^31: every key index fits the 32-bit TMA coordinates)
      const int pos = static_cast<int>(a.q_offset) + i;
      const int w0 = pos - a.window + 1;
      const int span0 = w.kb0 * 64;
      constexpr int CH = win_chunk(G);
      int klo = max(w0 + w.s * CH, 0), khi = min(w0 + (w.s + 1) * CH - 1, pos);
      if (!valid) { klo = 1; khi = 0; }
      klo -= span0;
      khi -= span0;
      const int lbk = __ffs(a.block) - 1;   // the block is a power of two (64 or 128)
      const int b0 = max(w0, 0) >> lbk;
      const uint32_t win = valid ? __ldg(a.win + static_cast<int64_t>(w.bg) * a.n_q + i) : 0u;
      // columns [c_lo, c_hi] of span block kb hold this row's keys (empty
      // when c_lo > c_hi); a selected block contributes none
      auto cols = [&](int kb, int& c_lo, int& c_hi) {
        const int wb = ((span0 + kb * 64) >> lbk) - b0;
        const bool open = wb >= 0 && wb < 32 && ((win >> wb) & 1u);
        c_lo = max(klo - kb * 64, 0);
        c_hi = min(khi - kb * 64, 63);
        if (!open) { c_lo = 1; c_hi = 0; }
      };
      ok = __all_sync(0xFFFFFFFFu, mbar_wait(s_full, par, a.err, SITE_WIN_SOFTMAX));
      if (!ok) break;
      tc_fence_after();
      // the row maximum over its keys (this group's blocks, then both);
      // blocks whole for every row of the warp skip the masking
      float mx[8] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY, -INFINITY, -INFINITY, -INFINITY, -INFINITY};
      for (int kb = kb_lo; kb < kb_hi; ++kb) {
        int c_lo, c_hi;
        cols(kb, c_lo, c_hi);
        if (!__any_sync(0xFFFFFFFFu, c_lo <= c_hi)) continue;   // warp-uniform
        const bool whole = __all_sync(0xFFFFFFFFu, c_lo == 0 && c_hi == 63);
#pragma unroll 1
        for (int qq = 0; qq < 2; ++qq) {
          uint32_t r[32];
          win_ld32(scol + kb * 64 + qq * 32, r);
          if (whole) {
#pragma unroll
            for (int u2 = 0; u2 < 32; ++u2) mx[u2 & 7] = fmaxf(mx[u2 & 7], __uint_as_float(r[u2]));
          } else {
            const int lo = c_lo - qq * 32, hi = c_hi - qq * 32;
#pragma unroll
            for (int u2 = 0; u2 < 32; ++u2)
              if (u2 >= lo && u2 <= hi) mx[u2 & 7] = fmaxf(mx[u2 & 7], __uint_as_float(r[u2]));
          }
        }
      }
      float m = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])), fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
      m = fmaxf(m, swap(0, m, par, ok));
      if (!ok) break;
      m = m == -INFINITY ? 0.f : m * a.scale_log2;
      // P = 2^(s - m) in bf16 over the first 32 columns of each block's S
      // (zero outside the row's keys), and the row sum
      float ls[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      for (int kb = kb_lo; kb < kb_hi; ++kb) {
        int c_lo, c_hi;
        cols(kb, c_lo, c_hi);
        const bool any = __any_sync(0xFFFFFFFFu, c_lo <= c_hi);
        const bool whole = __all_sync(0xFFFFFFFFu, c_lo == 0 && c_hi == 63);
        // 32 keys at a time: their S columns in, 16 columns of P out
#pragma unroll 1
        for (int qq = 0; qq < 2; ++qq) {
          uint32_t r[32], pw[16];
          if (any) win_ld32(scol + kb * 64 + qq * 32, r);
          if (whole) {
#pragma unroll
            for (int u2 = 0; u2 < 16; ++u2) {
              const float p0 = fast_exp2(fmaf(__uint_as_float(r[2 * u2]), a.scale_log2, -m));
              const float p1 = fast_exp2(fmaf(__uint_as_float(r[2 * u2 + 1]), a.scale_log2, -m));
              ls[(2 * u2) & 7] += p0;
              ls[(2 * u2 + 1) & 7] += p1;
              pw[u2] = pack_bf16(p0, p1);
            }
          } else {
            const int lo = c_lo - qq * 32, hi = c_hi - qq * 32;
#pragma unroll
            for (int u2 = 0; u2 < 16; ++u2) {
              float p0 = 0.f, p1 = 0.f;
              if (any) {
                p0 = (2 * u2 >= lo && 2 * u2 <= hi) ? fast_exp2(fmaf(__uint_as_float(r[2 * u2]), a.scale_log2, -m))
                                                      : 0.f;
                p1 = (2 * u2 + 1 >= lo && 2 * u2 + 1 <= hi)
                         ? fast_exp2(fmaf(__uint_as_float(r[2 * u2 + 1]), a.scale_log2, -m))
                         : 0.f;
              }
              ls[(2 * u2) & 7] += p0;
              ls[(2 * u2 + 1) & 7] += p1;
              pw[u2] = pack_bf16(p0, p1);
            }
          }
          tmem_st16(scol + kb * 64 + qq * 16, pw);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
      float l = ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
      // both groups' sums, in group order (the same l in both)
      {
        const float other = swap(1, l, par, ok);
        l = gs ? other + l : l + other;
      }
      if (!ok) break;
      // (m, l) to the epilogue through TMEM columns past the first block's P
      // (both groups are past their S loads here); the next tile's S waits
      // until the epilogue has read them
      if (gs == 0) {
        const uint32_t mlv[2] = {__float_as_uint(m), __float_as_uint(l)};
        tmem_st2(scol + (C::ML_COL - C::S_COL), mlv);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(ml_full);
      }
      ++u;
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int eq = warp & 3;
    const int row = eq * 32 + lane;
    const int e = row / G, h = row % G;
    const uint32_t ocol = tmem_base + (static_cast<uint32_t>(eq * 32) << 16) + C::O_COL;
    uint8_t* stage = sV + eq * 32 * C::ROW;   // this warp's 32 staging rows (first V slot)
    uint32_t u = 0;
    for (int t = blockIdx.x; t < a.n_tiles; t += gridDim.x) {
      const WinTile w = win_tile<G>(a, t);
      if (w.kb0 < 0) continue;
      const uint32_t par = u & 1;
      const int i = w.q0 + e;
      const bool valid = i < a.n_q;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait(ml_full, par, a.err, SITE_WIN_SOFTMAX) &&
                                       mbar_wait(o_full, par, a.err, SITE_WIN_SOFTMAX)))
        break;
      tc_fence_after();
      uint32_t mlv[2];
      tmem_ld2(tmem_base + (static_cast<uint32_t>(eq * 32) << 16) + C::ML_COL, mlv);
      tmem_wait_ld();
      tmem_regs_ready(mlv);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(ml_read);
      const float m = __uint_as_float(mlv[0]), l = __uint_as_float(mlv[1]);
      // one pass over O in halves of 64 dims: o = O / l of each half as
      // float16 times 2^-e, e chosen per half so its largest entry lands in
      // [2^14, 2^15); a row with no keys in this chunk (never read by the
      // merge) stores zeros
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      const int64_t slot = ((static_cast<int64_t>(w.bg) * a.n_q + i) * a.nsl + a.topk + w.s) * G + h;
      const int srow = lane >> 3, sch = lane & 7;
      uint32_t exs = 0;   // the two halves' exponents, 16 bits each
      // the staging rows are free once the previous tile's stores have read them
#pragma unroll
      for (int hf = 0; hf < D / 64; ++hf) {
        uint32_t r[64];
        win_ld64(ocol + hf * 64, r);
        if (hf == D / 64 - 1) {   // all of O is in registers: free the accumulator
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(o_empty);
        }
        float am[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int u2 = 0; u2 < 64; ++u2) am[u2 & 7] = fmaxf(am[u2 & 7], fabsf(__uint_as_float(r[u2])));
        const float x = fmaxf(fmaxf(fmaxf(am[0], am[1]), fmaxf(am[2], am[3])),
                              fmaxf(fmaxf(am[4], am[5]), fmaxf(am[6], am[7]))) * inv_l;
        int ex = x > 0.f ? static_cast<int>((__float_as_uint(x) >> 23) & 0xFFu) - 127 - 14 : 0;
        ex = min(max(ex, -100), 100);
        exs |= (static_cast<uint32_t>(ex) & 0xFFFFu) << (16 * hf);
        const float mul = inv_l * __uint_as_float(static_cast<uint32_t>(127 - ex) << 23);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          uint32_t wv[4];
#pragma unroll
          for (int u2 = 0; u2 < 4; ++u2) {
            const __half2 hv = __floats2half2_rn(__uint_as_float(r[q * 8 + 2 * u2]) * mul,
                                                 __uint_as_float(r[q * 8 + 2 * u2 + 1]) * mul);
            wv[u2] = *reinterpret_cast<const uint32_t*>(&hv);
          }
          *reinterpret_cast<uint4*>(stage + lane * C::ROW + ((q ^ (lane & 7)) << 4)) =
              make_uint4(wv[0], wv[1], wv[2], wv[3]);
        }
        __syncwarp();
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int rr = k * 4 + srow;
          const int64_t rslot = __shfl_sync(0xFFFFFFFFu, slot, rr);
          const bool rvalid = __shfl_sync(0xFFFFFFFFu, valid ? 1 : 0, rr) != 0;
          const uint4 v = *reinterpret_cast<const uint4*>(stage + rr * C::ROW + ((sch ^ (rr & 7)) << 4));
          if (rvalid) reinterpret_cast<uint4*>(a.partO + rslot * D + hf * 64)[sch] = v;
        }
        __syncwarp();
      }
      if (valid) a.partL[slot] = make_float2(l > 0.f ? m + log2f(l) : -INFINITY, __uint_as_float(exs));
      if (lane == 0) mbar_arrive(stg_done);
      ++u;
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

template <int G>
cudaError_t run_window(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV, const WinArgs& a,
                       const LaunchCtx& c) {
  using C = WinCfg<G>;
  cudaError_t e = cudaFuncSetAttribute(attn_window_kernel<G>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const int grid = a.n_tiles < c.sm_count ? a.n_tiles : c.sm_count;
  if (grid <= 0) return cudaSuccess;
  attn_window_kernel<G><<<grid, C::THREADS, C::SMEM, c.stream>>>(tmQ, tmK, tmV, a);
  note_launch();
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_window(const ssa_params& p, const BlockPlan& pl, const CUtensorMap& tmQ,
                               const CUtensorMap& tmK, const CUtensorMap& tmV, void* partO, void* partL,
                               const LaunchCtx& c) {
  const int G = p.h_q / p.h_kv;
  if (p.d != 128 || (G != 1 && G != 2 && G != 4 && G != 8)) return cudaErrorInvalidValue;
  WinArgs a;
  a.win = pl.win;
  a.n_q = p.n_q; a.n_kv = p.n_kv; a.h_q = p.h_q; a.h_kv = p.h_kv; a.block = p.block; a.topk = p.topk;
  a.window = p.window;
  a.nwc = window_chunks(p.window, G);
  a.nsl = p.topk + a.nwc;
  const int qt = 128 / G;
  a.n_qt = (p.n_q + qt - 1) / qt;
  a.q_offset = p.q_offset;
  const int64_t nt = static_cast<int64_t>(p.batch) * p.h_kv * a.n_qt * a.nwc;
  if (nt > 2147483647) return cudaErrorInvalidValue;
  a.n_tiles = static_cast<int32_t>(nt);
  a.scale_log2 = p.scale * 1.4426950408889634f;
  a.partO = static_cast<__half*>(partO);
  a.partL = static_cast<float2*>(partL);
  a.err = c.err;
  if (G == 1) return run_window<1>(tmQ, tmK, tmV, a, c);
  if (G == 2) return run_window<2>(tmQ, tmK, tmV, a, c);
  if (G == 4) return run_window<4>(tmQ, tmK, tmV, a, c);
  return run_window<8>(tmQ, tmK, tmV, a, c);
}

}  // namespace ssa

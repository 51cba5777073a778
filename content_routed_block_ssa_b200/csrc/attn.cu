// Steps (ii)+(iii) of the layer: exact softmax attention over the union of
// the routed blocks and the causal local window ["Subquadratic Sparse
// Attention (SSA)", opening section], per (query row, kv-head) item with the
// G query heads of the kv-head processed together.
//
// bf16 kernel.  A persistent CTA walks its items in (batch, kv-head,
// position) order so that concurrently running CTAs touch one kv-head's keys
// at a time.  A producer warp gathers every 64-key tile of the key set with
// TMA (K and V, 128-byte swizzled) into a ring of shared-memory stages; four
// consumer warps take the tiles of an item round-robin, each keeping its own
// online-softmax state (running max and sum), and merge the four partial
// results at the end of the item.  The G query heads are far too few rows for
// a tensor-core tile, so the keys are put on the M side instead:
//   S^T = K Q^T  (m16 = keys, n8 = heads, k16 = dims)
//   O^T += V^T P^T (m16 = dims, n8 = heads, k16 = keys)
// with warp-level bf16 MMAs; P^T is re-laid as the second operand with an
// 8x8 register transpose.  The kernel is bound by the bytes it gathers.
//
// float32 kernel: one CTA per item, SIMT, same tile list.
#include <cuda_bf16.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "tiles.cuh"

namespace ssa {
namespace {

struct AttnArgs {
  const void* Q;
  const void* K;     // float32 kernel only (the bf16 kernel reads K/V by TMA)
  const void* V;
  const int32_t* idx;
  void* O;
  float* lse;
  int32_t* bad;
  int32_t n_q, n_kv, h_q, h_kv, nb, block, topk, window;
  int64_t q_offset;
  int64_t n_items;
  float scale_log2;   // scale * log2(e)
  float scale;
  uint32_t* err;
};

template <int D>
struct AttnCfg {
  static constexpr int HALF = 64 * 64 * 2;            // 64 keys x 64 dims bf16 (8 KB)
  static constexpr int KBYTES = (D / 64) * HALF;
  static constexpr int STAGE = 2 * KBYTES;            // K then V of one 64-key tile
  static constexpr int NS = (D == 128) ? 6 : 12;      // tile ring
  static constexpr int MAXT = 32 * 2 + 66;            // selected tiles (k <= 32, <= 2 per block) + window tiles
  // item slot: Q tile (<= 8 heads, as D/64 boxes of G x 64), tile list, meta
  static constexpr int QBYTES = 8 * D * 2;
  static constexpr int SLOT = 4096;
  static constexpr int MERGE = 4 * 8 * D * 4 + 4 * 8 * 2 * 4;
  static constexpr int NSLOT = 3;
  static constexpr int NBAR = 2 * NS + 2 * NSLOT;
  static constexpr int SMEM = 1024 + NS * STAGE + NSLOT * SLOT + MERGE + NBAR * 8 + 32;
  static_assert(QBYTES + MAXT * 4 + 64 <= SLOT, "item slot too small");
};

struct ItemMeta {
  int64_t pos, lo, qrow;
  int32_t n_sub, ns;
};

__device__ __forceinline__ void named_bar_consumers() {
  asm volatile("bar.sync 1, 256;" ::: "memory");
}

// Warp roles: warp 8 = producer (item setup one item ahead: block list,
// tile list and Q into an item slot; then TMA gathers of the item's tiles
// into the ring), warps 0-7 = consumers in two groups of four; group 0 takes
// the even tiles of an item, group 1 the odd ones.  Within a group every
// 64-key tile is shared by the four warps, 16 keys each, so a ring stage is
// released after a quarter of the tile's work and the rest of the ring stays
// in flight; two groups give each SM sub-partition two warps to overlap.
template <int D, int G>
__global__ void __launch_bounds__(288, 1)
    attn_bf16_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const __grid_constant__ CUtensorMap tmQ, const AttnArgs a) {
  using C = AttnCfg<D>;
  constexpr int KS = D / 16;    // k-steps over dims
  constexpr int MT = D / 16;    // dim m-tiles of O^T
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = smem;
  uint8_t* slots = stages + C::NS * C::STAGE;                        // item slots
  float* mO = reinterpret_cast<float*>(slots + C::NSLOT * C::SLOT);   // [4][8][D]
  float* mM = mO + 4 * 8 * D;                                         // [4][8]
  float* mL = mM + 4 * 8;                                             // [4][8]
  uint64_t* full = reinterpret_cast<uint64_t*>(mL + 4 * 8);
  uint64_t* empty = full + C::NS;
  uint64_t* item_full = empty + C::NS;
  uint64_t* item_empty = item_full + C::NSLOT;
  int* abort_flag = reinterpret_cast<int*>(item_empty + C::NSLOT);   // [8]

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NS; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 4); }
    for (int s = 0; s < C::NSLOT; ++s) { mbar_init(&item_full[s], 1); mbar_init(&item_empty[s], 8); }
    fence_barrier_init();
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
    tma_prefetch_desc(&tmQ);
  }
  __syncthreads();

  __nv_bfloat16* Out = static_cast<__nv_bfloat16*>(a.O);
  auto slot_q = [&](int sl) { return slots + sl * C::SLOT; };
  auto slot_tiles = [&](int sl) { return reinterpret_cast<int32_t*>(slots + sl * C::SLOT + C::QBYTES); };
  auto slot_meta = [&](int sl) {
    return reinterpret_cast<ItemMeta*>(slots + sl * C::SLOT + C::QBYTES + C::MAXT * 4);
  };

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    // Item setup (tile list + Q) runs one item ahead of the tile gathers, so
    // the consumers find the next item ready when they finish the current one.
    uint32_t cnt = 0;
    bool ok = true;
    auto sel_ptr = [&](int64_t u) {
      const int i = static_cast<int>(u % a.n_q);
      const int64_t bg = u / a.n_q;
      const int g = static_cast<int>(bg % a.h_kv);
      const int64_t b = bg / a.h_kv;
      return a.idx + ((b * a.n_q + i) * a.h_kv + g) * a.topk;
    };
    // set up item number `local` (u = blockIdx.x + local * gridDim.x) in slot local % NSLOT
    auto setup = [&](int local, int v) -> bool {
      const int64_t u = blockIdx.x + static_cast<int64_t>(local) * gridDim.x;
      const int i = static_cast<int>(u % a.n_q);
      const int64_t bg = u / a.n_q;
      const int g = static_cast<int>(bg % a.h_kv);
      const int64_t b = bg / a.h_kv;
      const ItemTiles it = item_tiles_v(v, a.topk, a.q_offset + i, a.nb, a.block, a.window);
      const int sl = local % C::NSLOT;
      bool w_ok = true;
      if (lane == 0) w_ok = mbar_wait(&item_empty[sl], ((local / C::NSLOT) & 1) ^ 1, a.err, SITE_ATTN_PRODUCER);
      w_ok = __shfl_sync(0xFFFFFFFFu, w_ok, 0);
      if (!w_ok) return false;
      int32_t* tl = slot_tiles(sl);
      for (int j0 = 0; j0 < it.n_sub; j0 += 32) {
        const int j = j0 + lane;
        const int64_t k0 = tile_key0_lane(it, j, a.block);
        if (j < it.n_sub) tl[j] = static_cast<int32_t>(k0);
      }
      if (lane == 0) {
        ItemMeta* m = slot_meta(sl);
        m->pos = it.pos;
        m->lo = it.lo;
        m->qrow = (b * a.n_q + i) * a.h_q + static_cast<int64_t>(g) * G;
        m->n_sub = it.n_sub;
        m->ns = it.n_sel * it.spb;
        if (a.bad && it.n_bad) atomicAdd(a.bad, it.n_bad);
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive_expect_tx(&item_full[sl], G * D * 2);
        const int qrow = static_cast<int>((b * a.n_q + i) * a.h_q + static_cast<int64_t>(g) * G);
#pragma unroll
        for (int hf = 0; hf < D / 64; ++hf) tma_load_2d(slot_q(sl) + hf * G * 128, &tmQ, &item_full[sl], hf * 64, qrow);
      }
      return true;
    };
    const int n_local = static_cast<int>((a.n_items - blockIdx.x + gridDim.x - 1) / gridDim.x);
    int vnext = (n_local > 1 && lane < a.topk) ? __ldg(sel_ptr(blockIdx.x + gridDim.x) + lane) : -1;
    if (n_local > 0) {
      const int v0 = lane < a.topk ? __ldg(sel_ptr(blockIdx.x) + lane) : -1;
      ok = setup(0, v0);
    }
    for (int local = 0; local < n_local && ok; ++local) {
      if (local + 1 < n_local) {
        const int v = vnext;
        vnext = (local + 2 < n_local && lane < a.topk)
                    ? __ldg(sel_ptr(blockIdx.x + static_cast<int64_t>(local + 2) * gridDim.x) + lane) : -1;
        ok = setup(local + 1, v);
        if (!ok) break;
      }
      const int64_t u = blockIdx.x + static_cast<int64_t>(local) * gridDim.x;
      const int64_t bg = u / a.n_q;
      const int g = static_cast<int>(bg % a.h_kv);
      const int64_t b = bg / a.h_kv;
      const int sl = local % C::NSLOT;
      const int32_t* tl = slot_tiles(sl);
      const int n_sub = slot_meta(sl)->n_sub;
      if (lane == 0) {
        for (int j = 0; j < n_sub; ++j) {
          const int s = cnt % C::NS;
          if (!mbar_wait(&empty[s], ((cnt / C::NS) & 1) ^ 1, a.err, SITE_ATTN_PRODUCER)) { ok = false; break; }
          uint8_t* st = stages + s * C::STAGE;
          mbar_arrive_expect_tx(&full[s], C::STAGE);
          const int z = static_cast<int>(b * a.n_kv + tl[j]);
#pragma unroll
          for (int hf = 0; hf < D / 64; ++hf) {
            tma_load_3d(st + hf * C::HALF, &tmK, &full[s], hf * 64, g, z);
            tma_load_3d(st + C::KBYTES + hf * C::HALF, &tmV, &full[s], hf * 64, g, z);
          }
          ++cnt;
        }
      }
      cnt = __shfl_sync(0xFFFFFFFFu, cnt, 0);
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
    }
    if (!ok && lane == 0) {   // let copies already issued land before the CTA exits
      for (uint32_t n = (cnt > C::NS ? cnt - C::NS : 0); n < cnt; ++n) {
        const uint64_t t0 = global_timer_ns();
        while (!mbar_try_wait(&full[n % C::NS], (n / C::NS) & 1))
          if (global_timer_ns() - t0 > kWaitLimitNs) break;
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    const int gq = lane >> 2, tq = lane & 3;   // fragment row group / column pair
    uint32_t cnt = 0;
    int local = 0;
    const int wq = warp & 3, grp = warp >> 2;
    const int krow = wq * 16;                  // this warp's 16 keys of each of its tiles
    for (int64_t u = blockIdx.x; u < a.n_items; u += gridDim.x, ++local) {
      const int sl = local % C::NSLOT;
      bool ok = __all_sync(0xFFFFFFFFu, mbar_wait(&item_full[sl], (local / C::NSLOT) & 1, a.err, SITE_ATTN_CONSUMER));
      float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
      float oacc[MT][4];
#pragma unroll
      for (int mm = 0; mm < MT; ++mm)
#pragma unroll
        for (int r = 0; r < 4; ++r) oacc[mm][r] = 0.f;
      ItemMeta meta{};
      if (ok) {
        meta = *slot_meta(sl);
        const int32_t* tl = slot_tiles(sl);
        // Q^T as the n8 operand: (dims 2t..2t+1 (+8), head gq), zero for gq >= G
        uint32_t qf[KS][2];
        const uint8_t* qs = slot_q(sl);
#pragma unroll
        for (int ks = 0; ks < KS; ++ks) {
          if (gq < G) {
            const uint32_t* qp = reinterpret_cast<const uint32_t*>(
                qs + (ks >> 2) * G * 128 + gq * 128 + ((ks & 3) * 16 + 2 * tq) * 2);
            qf[ks][0] = qp[0];
            qf[ks][1] = qp[4];
          } else {
            qf[ks][0] = 0u;
            qf[ks][1] = 0u;
          }
        }
        for (int j = grp; j < meta.n_sub; j += 2) {
          const uint32_t n = cnt + j;
          const int s = n % C::NS;
          ok = __all_sync(0xFFFFFFFFu, mbar_wait(&full[s], (n / C::NS) & 1, a.err, SITE_ATTN_CONSUMER));
          if (!ok) break;
          const int key0 = tl[j];
          const bool wt = j >= meta.ns;
          const uint32_t kb = smem_u32(stages + s * C::STAGE);
          const uint32_t vb = kb + C::KBYTES;
          // copy this warp's 16-key slice of K and V into registers and give
          // the stage back at once, so the ring refills while we compute
          uint32_t kf[KS][4], vf[MT][4];
          {
            const int row = krow + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) {
              const int chunk = (ks & 3) * 2 + (lane >> 4);
              ldmatrix_x4(kf[ks], kb + (ks >> 2) * C::HALF + row * 128 + ((chunk ^ (row & 7)) << 4));
            }
            const int mi = lane >> 3;
            const int vrow = krow + (lane & 7) + (mi >> 1) * 8;
#pragma unroll
            for (int mm = 0; mm < MT; ++mm) {
              const int dchunk = mm * 2 + (mi & 1);
              ldmatrix_x4_trans(vf[mm], vb + (dchunk >> 3) * C::HALF + vrow * 128 + (((dchunk & 7) ^ (vrow & 7)) << 4));
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&empty[s]);

          // S^T = K Q^T for this warp's 16 keys (two independent accumulators)
          float sacc[4];
          {
            float part[4][4];
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
              for (int r = 0; r < 4; ++r) part[c][r] = 0.f;
#pragma unroll
            for (int ks = 0; ks < KS; ++ks) mma_16816(part[ks & 3], kf[ks], qf[ks][0], qf[ks][1]);
#pragma unroll
            for (int r = 0; r < 4; ++r) sacc[r] = (part[0][r] + part[1][r]) + (part[2][r] + part[3][r]);
          }
          // scale, mask (window tiles only), running max per head (heads 2tq, 2tq+1)
          float mx[2] = {-INFINITY, -INFINITY};
          if (wt) {
            const int klo = static_cast<int>(meta.lo) - key0 - krow - gq;
            const int khi = static_cast<int>(meta.pos) - key0 - krow - gq;
#pragma unroll
            for (int r = 0; r < 4; ++r) {
              const int kk = (r >= 2 ? 8 : 0);
              sacc[r] = (kk >= klo && kk <= khi) ? sacc[r] * a.scale_log2 : -INFINITY;
            }
          } else {
#pragma unroll
            for (int r = 0; r < 4; ++r) sacc[r] *= a.scale_log2;
          }
#pragma unroll
          for (int r = 0; r < 4; ++r) mx[r & 1] = fmaxf(mx[r & 1], sacc[r]);
          bool grow = false;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xFFFFFFFFu, mx[h], 4));
            mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xFFFFFFFFu, mx[h], 8));
            mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xFFFFFFFFu, mx[h], 16));
            grow |= mx[h] > m_run[h];
          }
          // rescale only when some head's running max rose (exact either way)
          if (__any_sync(0xFFFFFFFFu, grow)) {
            float alpha[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const float mnew = fmaxf(m_run[h], mx[h]);
              alpha[h] = (m_run[h] == -INFINITY) ? 0.f : fast_exp2(m_run[h] - mnew);
              m_run[h] = mnew;
              l_run[h] *= alpha[h];
            }
#pragma unroll
            for (int mm = 0; mm < MT; ++mm) {
              oacc[mm][0] *= alpha[0];
              oacc[mm][1] *= alpha[1];
              oacc[mm][2] *= alpha[0];
              oacc[mm][3] *= alpha[1];
            }
          }
          float p[4];
#pragma unroll
          for (int r = 0; r < 4; ++r) p[r] = (sacc[r] == -INFINITY) ? 0.f : fast_exp2(sacc[r] - m_run[r & 1]);
          l_run[0] += p[0] + p[2];
          l_run[1] += p[1] + p[3];
          const uint32_t pb0 = movmatrix_trans(pack_bf16(p[0], p[1]));
          const uint32_t pb1 = movmatrix_trans(pack_bf16(p[2], p[3]));
          // O^T += V^T P^T over this warp's 16 keys
#pragma unroll
          for (int mm = 0; mm < MT; ++mm) mma_16816(oacc[mm], vf[mm], pb0, pb1);
        }
        cnt += meta.n_sub;
      }

      // per-warp partials; all eight consumer warps meet here every item
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        l_run[h] += __shfl_xor_sync(0xFFFFFFFFu, l_run[h], 4);
        l_run[h] += __shfl_xor_sync(0xFFFFFFFFu, l_run[h], 8);
        l_run[h] += __shfl_xor_sync(0xFFFFFFFFu, l_run[h], 16);
      }
      if (lane == 0) abort_flag[warp] = ok ? 0 : 1;
      float* myO = mO + wq * 8 * D;
      // group 1 hands its partials to the group-0 warp with the same key slice
      if (grp == 1) {
#pragma unroll
        for (int mm = 0; mm < MT; ++mm) {
          const int d0 = mm * 16 + gq;
          myO[(2 * tq) * D + d0] = oacc[mm][0];
          myO[(2 * tq + 1) * D + d0] = oacc[mm][1];
          myO[(2 * tq) * D + d0 + 8] = oacc[mm][2];
          myO[(2 * tq + 1) * D + d0 + 8] = oacc[mm][3];
        }
        if (gq == 0) {
          mM[wq * 8 + 2 * tq] = m_run[0];
          mM[wq * 8 + 2 * tq + 1] = m_run[1];
          mL[wq * 8 + 2 * tq] = l_run[0];
          mL[wq * 8 + 2 * tq + 1] = l_run[1];
        }
      }
      named_bar_consumers();
      if (grp == 0) {
        float f0[2], f1[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const float mo = mM[wq * 8 + 2 * tq + h], lo_ = mL[wq * 8 + 2 * tq + h];
          const float M = fmaxf(m_run[h], mo);
          f0[h] = (m_run[h] == -INFINITY) ? 0.f : fast_exp2(m_run[h] - M);
          f1[h] = (mo == -INFINITY) ? 0.f : fast_exp2(mo - M);
          l_run[h] = f0[h] * l_run[h] + f1[h] * lo_;
          m_run[h] = M;
        }
#pragma unroll
        for (int mm = 0; mm < MT; ++mm) {
          const int d0 = mm * 16 + gq;
          float* o0 = &myO[(2 * tq) * D + d0];
          float* o1 = &myO[(2 * tq + 1) * D + d0];
          o0[0] = f0[0] * oacc[mm][0] + f1[0] * o0[0];
          o1[0] = f0[1] * oacc[mm][1] + f1[1] * o1[0];
          o0[8] = f0[0] * oacc[mm][2] + f1[0] * o0[8];
          o1[8] = f0[1] * oacc[mm][3] + f1[1] * o1[8];
        }
        __syncwarp();
        if (gq == 0) {
          mM[wq * 8 + 2 * tq] = m_run[0];
          mM[wq * 8 + 2 * tq + 1] = m_run[1];
          mL[wq * 8 + 2 * tq] = l_run[0];
          mL[wq * 8 + 2 * tq + 1] = l_run[1];
        }
      }
      named_bar_consumers();
      // a failed wait in any warp stops all eight together
      int ab = 0;
#pragma unroll
      for (int w = 0; w < 8; ++w) ab |= abort_flag[w];
      const bool any_abort = ab != 0;
      for (int e = threadIdx.x; e < G * D && !any_abort; e += 256) {
        const int h = e / D, dd = e % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < 4; ++w) M = fmaxf(M, mM[w * 8 + h]);
        float num = 0.f, den = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          const float mw = mM[w * 8 + h];
          const float f = (mw == -INFINITY) ? 0.f : fast_exp2(mw - M);
          num += f * mO[(w * 8 + h) * D + dd];
          den += f * mL[w * 8 + h];
        }
        Out[(meta.qrow + h) * D + dd] = __float2bfloat16_rn(num / den);
        if (dd == 0 && a.lse) a.lse[meta.qrow + h] = (M + log2f(den)) * 0.69314718055994531f;
      }
      named_bar_consumers();
      if (lane == 0) mbar_arrive(&item_empty[sl]);
      if (any_abort) break;
    }
  }
  __syncthreads();
}

// ------------------------------------------------------------------ float32

// One CTA per item.  Per 64-key tile: logits into shared memory, running
// max / sum per head, then every thread updates its (head, dim) outputs.
template <int D, int G>
__global__ void __launch_bounds__(128) attn_f32_kernel(const AttnArgs a) {
  extern __shared__ float fsm[];
  float* Ks = fsm;                   // [64][D+1] (padded: conflict-free row reads)
  float* Vs = Ks + 64 * (D + 1);     // [64][D]
  float* qsm = Vs + 64 * D;          // [G][D]
  float* ps = qsm + G * D;           // [G][64]
  float* st_m = ps + G * 64;         // [G]
  float* st_l = st_m + G;            // [G]
  float* st_a = st_l + G;            // [G]
  constexpr int PER = (G * D + 127) / 128;

  const int64_t u = blockIdx.x;
  const int i = static_cast<int>(u % a.n_q);
  const int64_t bg = u / a.n_q;
  const int g = static_cast<int>(bg % a.h_kv);
  const int64_t b = bg / a.h_kv;
  const float* Q = static_cast<const float*>(a.Q);
  const float* K = static_cast<const float*>(a.K);
  const float* V = static_cast<const float*>(a.V);
  float* Out = static_cast<float*>(a.O);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t qrow = (b * a.n_q + i) * a.h_q + static_cast<int64_t>(g) * G;
  for (int e = threadIdx.x; e < G * D; e += 128) qsm[e] = Q[qrow * D + e];
  if (threadIdx.x < G) { st_m[threadIdx.x] = -INFINITY; st_l[threadIdx.x] = 0.f; }

  const int32_t* sel = a.idx + ((b * a.n_q + i) * a.h_kv + g) * a.topk;
  const ItemTiles it = item_tiles(sel, a.topk, a.q_offset + i, a.nb, a.block, a.window);
  if (threadIdx.x == 0 && a.bad && it.n_bad) atomicAdd(a.bad, it.n_bad);

  float acc[PER];
#pragma unroll
  for (int k = 0; k < PER; ++k) acc[k] = 0.f;

  for (int j = 0; j < it.n_sub; ++j) {
    bool wt;
    const int64_t key0 = tile_key0(it, j, a.block, wt);
    __syncthreads();
    for (int e = threadIdx.x; e < 64 * (D / 4); e += 128) {
      const int r = e / (D / 4), c4 = e % (D / 4);
      const int64_t off = ((b * a.n_kv + key0 + r) * a.h_kv + g) * D + 4 * c4;
      const float4 kv = __ldg(reinterpret_cast<const float4*>(K + off));
      const float4 vv = __ldg(reinterpret_cast<const float4*>(V + off));
      float* kr = Ks + r * (D + 1) + 4 * c4;
      kr[0] = kv.x; kr[1] = kv.y; kr[2] = kv.z; kr[3] = kv.w;
      *reinterpret_cast<float4*>(Vs + r * D + 4 * c4) = vv;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < G * 64; e += 128) {
      const int h = e / 64, r = e % 64;
      const int64_t key = key0 + r;
      const bool in = !wt || (key >= it.lo && key <= it.pos);
      float dot = 0.f;
      if (in) {
#pragma unroll 8
        for (int t = 0; t < D; ++t) dot = fmaf(qsm[h * D + t], Ks[r * (D + 1) + t], dot);
      }
      ps[h * 64 + r] = in ? dot * a.scale : -INFINITY;
    }
    __syncthreads();
    for (int h = warp; h < G; h += 4) {
      float v0 = ps[h * 64 + lane], v1 = ps[h * 64 + lane + 32];
      float mx = fmaxf(v0, v1);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, o));
      const float mold = st_m[h];
      const float mnew = fmaxf(mold, mx);
      const float alpha = (mnew == -INFINITY) ? 1.f : expf(mold - mnew);
      const float p0 = (v0 == -INFINITY) ? 0.f : expf(v0 - mnew);
      const float p1 = (v1 == -INFINITY) ? 0.f : expf(v1 - mnew);
      ps[h * 64 + lane] = p0;
      ps[h * 64 + lane + 32] = p1;
      float sum = p0 + p1;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
      __syncwarp();
      if (lane == 0) {
        st_l[h] = st_l[h] * alpha + sum;
        st_m[h] = mnew;
        st_a[h] = alpha;
      }
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < PER; ++k) {
      const int e = threadIdx.x + 128 * k;
      if (e < G * D) {
        const int h = e / D, dd = e % D;
        float x = acc[k] * st_a[h];
#pragma unroll 8
        for (int r = 0; r < 64; ++r) x = fmaf(ps[h * 64 + r], Vs[r * D + dd], x);
        acc[k] = x;
      }
    }
  }
  __syncthreads();
#pragma unroll
  for (int k = 0; k < PER; ++k) {
    const int e = threadIdx.x + 128 * k;
    if (e < G * D) {
      const int h = e / D, dd = e % D;
      Out[(qrow + h) * D + dd] = acc[k] / st_l[h];
      if (dd == 0 && a.lse) a.lse[qrow + h] = st_m[h] + logf(st_l[h]);
    }
  }
}

AttnArgs attn_args(const ssa_params& p, const void* Q, const void* K, const void* V,
                   const int32_t* idx, void* O, float* lse, int32_t* bad, uint32_t* err) {
  AttnArgs a;
  a.Q = Q; a.K = K; a.V = V; a.idx = idx; a.O = O; a.lse = lse; a.bad = bad;
  a.n_q = p.n_q; a.n_kv = p.n_kv; a.h_q = p.h_q; a.h_kv = p.h_kv; a.nb = p.n_kv / p.block;
  a.block = p.block; a.topk = p.topk; a.window = p.window;
  a.q_offset = p.q_offset;
  a.n_items = static_cast<int64_t>(p.batch) * p.h_kv * p.n_q;
  a.scale = p.scale;
  a.scale_log2 = p.scale * 1.4426950408889634f;
  a.err = err;
  return a;
}

template <int D, int G>
cudaError_t run_bf16(const ssa_params& p, const CUtensorMap& tmK, const CUtensorMap& tmV,
                     const CUtensorMap& tmQ, const AttnArgs& a, const LaunchCtx& c) {
  using C = AttnCfg<D>;
  cudaError_t e = cudaFuncSetAttribute(attn_bf16_kernel<D, G>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  int per_sm = 1;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, attn_bf16_kernel<D, G>, 288, C::SMEM);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  int64_t grid = static_cast<int64_t>(per_sm) * c.sm_count;
  if (grid > a.n_items) grid = a.n_items;
  attn_bf16_kernel<D, G><<<static_cast<unsigned>(grid), 288, C::SMEM, c.stream>>>(tmK, tmV, tmQ, a);
  note_launch();
  return cudaGetLastError();
}

template <int D>
cudaError_t bf16_g(const ssa_params& p, const CUtensorMap& tmK, const CUtensorMap& tmV,
                   const CUtensorMap& tmQ, const AttnArgs& a, const LaunchCtx& c) {
  switch (p.h_q / p.h_kv) {
    case 1: return run_bf16<D, 1>(p, tmK, tmV, tmQ, a, c);
    case 2: return run_bf16<D, 2>(p, tmK, tmV, tmQ, a, c);
    case 4: return run_bf16<D, 4>(p, tmK, tmV, tmQ, a, c);
    case 8: return run_bf16<D, 8>(p, tmK, tmV, tmQ, a, c);
  }
  return cudaErrorInvalidValue;
}

template <int D, int G>
cudaError_t run_f32(const AttnArgs& a, const LaunchCtx& c) {
  const int smem = static_cast<int>(sizeof(float)) * (64 * (D + 1) + 64 * D + G * D + G * 64 + 3 * G);
  cudaError_t e = cudaFuncSetAttribute(attn_f32_kernel<D, G>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  attn_f32_kernel<D, G><<<static_cast<unsigned>(a.n_items), 128, smem, c.stream>>>(a);
  note_launch();
  return cudaGetLastError();
}

template <int D>
cudaError_t f32_g(const ssa_params& p, const AttnArgs& a, const LaunchCtx& c) {
  switch (p.h_q / p.h_kv) {
    case 1: return run_f32<D, 1>(a, c);
    case 2: return run_f32<D, 2>(a, c);
    case 4: return run_f32<D, 4>(a, c);
    case 8: return run_f32<D, 8>(a, c);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

int attn_bf16_smem_bytes(int d) { return d == 128 ? AttnCfg<128>::SMEM : AttnCfg<64>::SMEM; }

cudaError_t launch_attn_bf16(const ssa_params& p, const CUtensorMap& tmK, const CUtensorMap& tmV,
                             const CUtensorMap& tmQ, const void* Q, const int32_t* block_idx, void* O,
                             float* lse, int32_t* bad, const LaunchCtx& c) {
  const AttnArgs a = attn_args(p, Q, nullptr, nullptr, block_idx, O, lse, bad, c.err);
  if (p.d == 128) return bf16_g<128>(p, tmK, tmV, tmQ, a, c);
  if (p.d == 64) return bf16_g<64>(p, tmK, tmV, tmQ, a, c);
  return cudaErrorInvalidValue;
}

cudaError_t launch_attn_f32(const ssa_params& p, const void* Q, const void* K, const void* V,
                            const int32_t* block_idx, void* O, float* lse, int32_t* bad,
                            const LaunchCtx& c) {
  const AttnArgs a = attn_args(p, Q, K, V, block_idx, O, lse, bad, c.err);
  if (p.d == 128) return f32_g<128>(p, a, c);
  if (p.d == 64) return f32_g<64>(p, a, c);
  return cudaErrorInvalidValue;
}

}  // namespace ssa

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
  static constexpr int STAGE = 2 * KBYTES;            // K then V
  static constexpr int NS = (D == 128) ? 6 : 10;
  static constexpr int MERGE = 4 * 8 * D * 4 + 4 * 8 * 2 * 4;
  static constexpr int SMEM = 1024 + NS * STAGE + MERGE + 2 * NS * 8 + 16;
};

__device__ __forceinline__ void named_bar_consumers() {
  asm volatile("bar.sync 1, 128;" ::: "memory");
}

template <int D, int G>
__global__ void __launch_bounds__(160, 1)
    attn_bf16_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                     const AttnArgs a) {
  using C = AttnCfg<D>;
  constexpr int KS = D / 16;    // k-steps over dims
  constexpr int MT = D / 16;    // dim m-tiles of O^T
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* stages = smem;
  float* mO = reinterpret_cast<float*>(stages + C::NS * C::STAGE);   // [4][8][D]
  float* mM = mO + 4 * 8 * D;                                         // [4][8]
  float* mL = mM + 4 * 8;                                             // [4][8]
  uint64_t* full = reinterpret_cast<uint64_t*>(mL + 4 * 8);
  uint64_t* empty = full + C::NS;
  int* abort_flag = reinterpret_cast<int*>(empty + C::NS);   // [4]

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NS; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    fence_barrier_init();
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  __syncthreads();

  const __nv_bfloat16* Q = static_cast<const __nv_bfloat16*>(a.Q);
  __nv_bfloat16* Out = static_cast<__nv_bfloat16*>(a.O);

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    uint32_t cnt = 0;
    bool ok = true;
    for (int64_t u = blockIdx.x; u < a.n_items && ok; u += gridDim.x) {
      const int i = static_cast<int>(u % a.n_q);
      const int64_t bg = u / a.n_q;
      const int g = static_cast<int>(bg % a.h_kv);
      const int64_t b = bg / a.h_kv;
      const int32_t* sel = a.idx + ((b * a.n_q + i) * a.h_kv + g) * a.topk;
      const ItemTiles it = item_tiles(sel, a.topk, a.q_offset + i, a.nb, a.block, a.window);
      if (lane == 0 && a.bad && it.n_bad) atomicAdd(a.bad, it.n_bad);
      for (int j = 0; j < it.n_sub; ++j) {
        bool wt;
        const int64_t key0 = tile_key0(it, j, a.block, wt);
        if (lane == 0) {
          const int s = cnt % C::NS;
          ok = mbar_wait(&empty[s], ((cnt / C::NS) & 1) ^ 1, a.err, SITE_ATTN_PRODUCER);
          if (ok) {
            uint8_t* st = stages + s * C::STAGE;
            mbar_arrive_expect_tx(&full[s], C::STAGE);
            const int z = static_cast<int>(b * a.n_kv + key0);
#pragma unroll
            for (int hf = 0; hf < D / 64; ++hf) {
              tma_load_3d(st + hf * C::HALF, &tmK, &full[s], hf * 64, g, z);
              tma_load_3d(st + C::KBYTES + hf * C::HALF, &tmV, &full[s], hf * 64, g, z);
            }
          }
        }
        ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
        if (!ok) break;
        ++cnt;
      }
    }
    if (!ok && lane == 0) {
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
    bool ok = true;
    for (int64_t u = blockIdx.x; u < a.n_items && ok; u += gridDim.x) {
      const int i = static_cast<int>(u % a.n_q);
      const int64_t bg = u / a.n_q;
      const int g = static_cast<int>(bg % a.h_kv);
      const int64_t b = bg / a.h_kv;
      const int32_t* sel = a.idx + ((b * a.n_q + i) * a.h_kv + g) * a.topk;
      const ItemTiles it = item_tiles(sel, a.topk, a.q_offset + i, a.nb, a.block, a.window);
      const int64_t qrow = (b * a.n_q + i) * a.h_q + static_cast<int64_t>(g) * G;

      // Q^T as the n8 operand: (dims 2t..2t+1 (+8), head gq), zero for gq >= G
      uint32_t qf[KS][2];
#pragma unroll
      for (int ks = 0; ks < KS; ++ks) {
        if (gq < G) {
          const uint32_t* qp = reinterpret_cast<const uint32_t*>(Q + (qrow + gq) * D + ks * 16 + 2 * tq);
          qf[ks][0] = __ldg(qp);
          qf[ks][1] = __ldg(qp + 4);
        } else {
          qf[ks][0] = 0u;
          qf[ks][1] = 0u;
        }
      }
      float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
      float oacc[MT][4];
#pragma unroll
      for (int mm = 0; mm < MT; ++mm)
#pragma unroll
        for (int r = 0; r < 4; ++r) oacc[mm][r] = 0.f;

      for (int j = warp; j < it.n_sub; j += 4) {
        bool wt;
        const int64_t key0 = tile_key0(it, j, a.block, wt);
        const uint32_t n = cnt + j;
        const int s = n % C::NS;
        ok = __all_sync(0xFFFFFFFFu, mbar_wait(&full[s], (n / C::NS) & 1, a.err, SITE_ATTN_CONSUMER));
        if (!ok) break;
        const uint32_t kb = smem_u32(stages + s * C::STAGE);
        const uint32_t vb = kb + C::KBYTES;

        // S^T = K Q^T for 4 tiles of 16 keys
        float sacc[4][4];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
#pragma unroll
          for (int r = 0; r < 4; ++r) sacc[m][r] = 0.f;
          const int row = m * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
          for (int ks = 0; ks < KS; ++ks) {
            const int chunk = (ks & 3) * 2 + (lane >> 4);
            const uint32_t addr = kb + (ks >> 2) * C::HALF + row * 128 + ((chunk ^ (row & 7)) << 4);
            uint32_t af[4];
            ldmatrix_x4(af, addr);
            mma_16816(sacc[m], af, qf[ks][0], qf[ks][1]);
          }
        }
        // scale, mask, running max per head (heads 2tq, 2tq+1)
        float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
        for (int m = 0; m < 4; ++m) {
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const int64_t key = key0 + m * 16 + gq + (r >= 2 ? 8 : 0);
            const bool in = !wt || (key >= it.lo && key <= it.pos);
            const float sv = in ? sacc[m][r] * a.scale_log2 : -INFINITY;
            sacc[m][r] = sv;
            mx[r & 1] = fmaxf(mx[r & 1], sv);
          }
        }
        float alpha[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xFFFFFFFFu, mx[h], 4));
          mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xFFFFFFFFu, mx[h], 8));
          mx[h] = fmaxf(mx[h], __shfl_xor_sync(0xFFFFFFFFu, mx[h], 16));
          const float mnew = fmaxf(m_run[h], mx[h]);
          alpha[h] = (mnew == -INFINITY) ? 1.f : fast_exp2(m_run[h] - mnew);
          m_run[h] = mnew;
        }
        uint32_t pb[4][2];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          float p[4];
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const float mr = m_run[r & 1];
            p[r] = (mr == -INFINITY) ? 0.f : fast_exp2(sacc[m][r] - mr);
          }
          l_run[0] = l_run[0] * (m == 0 ? alpha[0] : 1.f) + p[0] + p[2];
          l_run[1] = l_run[1] * (m == 0 ? alpha[1] : 1.f) + p[1] + p[3];
          pb[m][0] = movmatrix_trans(pack_bf16(p[0], p[1]));
          pb[m][1] = movmatrix_trans(pack_bf16(p[2], p[3]));
        }
#pragma unroll
        for (int mm = 0; mm < MT; ++mm) {
          oacc[mm][0] *= alpha[0];
          oacc[mm][1] *= alpha[1];
          oacc[mm][2] *= alpha[0];
          oacc[mm][3] *= alpha[1];
        }
        // O^T += V^T P^T
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const int mi = lane >> 3;
          const int row = m * 16 + (lane & 7) + (mi >> 1) * 8;
#pragma unroll
          for (int mm = 0; mm < MT; ++mm) {
            const int dchunk = mm * 2 + (mi & 1);
            const uint32_t addr = vb + (dchunk >> 3) * C::HALF + row * 128 + (((dchunk & 7) ^ (row & 7)) << 4);
            uint32_t af[4];
            ldmatrix_x4_trans(af, addr);
            mma_16816(oacc[mm], af, pb[m][0], pb[m][1]);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
      }
      cnt += it.n_sub;

      // per-warp partials -> shared memory
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        l_run[h] += __shfl_xor_sync(0xFFFFFFFFu, l_run[h], 4);
        l_run[h] += __shfl_xor_sync(0xFFFFFFFFu, l_run[h], 8);
        l_run[h] += __shfl_xor_sync(0xFFFFFFFFu, l_run[h], 16);
      }
      float* myO = mO + warp * 8 * D;
#pragma unroll
      for (int mm = 0; mm < MT; ++mm) {
        const int d0 = mm * 16 + gq;
        myO[(2 * tq) * D + d0] = oacc[mm][0];
        myO[(2 * tq + 1) * D + d0] = oacc[mm][1];
        myO[(2 * tq) * D + d0 + 8] = oacc[mm][2];
        myO[(2 * tq + 1) * D + d0 + 8] = oacc[mm][3];
      }
      if (lane == 0) abort_flag[warp] = ok ? 0 : 1;
      if (gq == 0) {
        mM[warp * 8 + 2 * tq] = m_run[0];
        mM[warp * 8 + 2 * tq + 1] = m_run[1];
        mL[warp * 8 + 2 * tq] = l_run[0];
        mL[warp * 8 + 2 * tq + 1] = l_run[1];
      }
      named_bar_consumers();
      // every consumer warp reaches both barriers of an item, so a failed
      // wait in one warp stops all four together after the first
      const bool any_abort = (abort_flag[0] | abort_flag[1] | abort_flag[2] | abort_flag[3]) != 0;
      for (int e = threadIdx.x; e < G * D && !any_abort; e += 128) {
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
        Out[(qrow + h) * D + dd] = __float2bfloat16_rn(num / den);
        if (dd == 0 && a.lse) a.lse[qrow + h] = (M + log2f(den)) * 0.69314718055994531f;
      }
      named_bar_consumers();
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
                     const AttnArgs& a, const LaunchCtx& c) {
  using C = AttnCfg<D>;
  cudaError_t e = cudaFuncSetAttribute(attn_bf16_kernel<D, G>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  int per_sm = 1;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, attn_bf16_kernel<D, G>, 160, C::SMEM);
  if (e != cudaSuccess) return e;
  if (per_sm < 1) per_sm = 1;
  int64_t grid = static_cast<int64_t>(per_sm) * c.sm_count;
  if (grid > a.n_items) grid = a.n_items;
  attn_bf16_kernel<D, G><<<static_cast<unsigned>(grid), 160, C::SMEM, c.stream>>>(tmK, tmV, a);
  note_launch();
  return cudaGetLastError();
}

template <int D>
cudaError_t bf16_g(const ssa_params& p, const CUtensorMap& tmK, const CUtensorMap& tmV,
                   const AttnArgs& a, const LaunchCtx& c) {
  switch (p.h_q / p.h_kv) {
    case 1: return run_bf16<D, 1>(p, tmK, tmV, a, c);
    case 2: return run_bf16<D, 2>(p, tmK, tmV, a, c);
    case 4: return run_bf16<D, 4>(p, tmK, tmV, a, c);
    case 8: return run_bf16<D, 8>(p, tmK, tmV, a, c);
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
                             const void* Q, const int32_t* block_idx, void* O, float* lse,
                             int32_t* bad, const LaunchCtx& c) {
  const AttnArgs a = attn_args(p, Q, nullptr, nullptr, block_idx, O, lse, bad, c.err);
  if (p.d == 128) return bf16_g<128>(p, tmK, tmV, a, c);
  if (p.d == 64) return bf16_g<64>(p, tmK, tmV, a, c);
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

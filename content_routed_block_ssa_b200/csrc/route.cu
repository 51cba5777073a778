// Step (i) of the layer: route every query row to its top-k key blocks.
//
// Score of fully visible block c for the query heads h of kv-head g:
//   s_c = sum_h r_c(q_h),  r_c(q) = <q, mu_c> + (beta/2) q^T Sigma_c q
// ["Subquadratic Sparse Attention (SSA)", "The idea in one screen",
// routing-score equation], with a fixed budget of k blocks per row
// ["fixed budget kappa << n", opening section].  Ties go to the lower block
// index.
//
// For bf16 problems with a diagonal Sigma the score is the dot product of
// the feature row f = [sum_h q_h ; (beta/2) sum_h q_h*q_h] with the table
// row [mu_c ; sigma_c^2], so routing a tile of query rows is a dense
// contraction (rows x 2d) . (2d x blocks).  The tiled router runs it on the
// tcgen05 tensor cores with TMEM accumulators and selects the top-k in the
// epilogue while the next chunk is being multiplied: scores never leave the
// SM.
#include <cuda_bf16.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace ssa {
namespace {

// ------------------------------------------------------------------ features

// F[b, g, i, :] = [bf16(qs), bf16(hb * qq)], qs / qq accumulated in float32
// in head order.  Thread = (row, 8 consecutive dimensions).
template <int D, int G>
__global__ void __launch_bounds__(256) features_kernel(const __nv_bfloat16* __restrict__ Q,
                                                       __nv_bfloat16* __restrict__ F,
                                                       int64_t rows, int n_q, int h_kv,
                                                       float half_beta) {
  constexpr int CG = D / 8;
  constexpr int RPC = 256 / CG;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * RPC + threadIdx.x / CG;
  const int cg = threadIdx.x % CG;
  if (row >= rows) return;
  const int i = static_cast<int>(row % n_q);
  const int64_t bg = row / n_q;
  const int g = static_cast<int>(bg % h_kv);
  const int64_t b = bg / h_kv;
  const int h_q = h_kv * G;
  const __nv_bfloat16* q = Q + ((b * n_q + i) * h_q + static_cast<int64_t>(g) * G) * D + cg * 8;
  float qs[8], qq[8];
#pragma unroll
  for (int v = 0; v < 8; ++v) { qs[v] = 0.f; qq[v] = 0.f; }
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const uint4 raw = __ldg(reinterpret_cast<const uint4*>(q + h * D));
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float lo = __uint_as_float(w[j] << 16), hi = __uint_as_float(w[j] & 0xFFFF0000u);
      qs[2 * j] = __fadd_rn(qs[2 * j], lo);
      qs[2 * j + 1] = __fadd_rn(qs[2 * j + 1], hi);
      qq[2 * j] = __fmaf_rn(lo, lo, qq[2 * j]);         // lo*lo is exact in float32
      qq[2 * j + 1] = __fmaf_rn(hi, hi, qq[2 * j + 1]);
    }
  }
  uint4 o1, o2;
  uint32_t* p1 = reinterpret_cast<uint32_t*>(&o1);
  uint32_t* p2 = reinterpret_cast<uint32_t*>(&o2);
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    p1[j] = pack_bf16(qs[2 * j], qs[2 * j + 1]);
    p2[j] = pack_bf16(__fmul_rn(half_beta, qq[2 * j]), __fmul_rn(half_beta, qq[2 * j + 1]));
  }
  __nv_bfloat16* f = F + row * (2 * D) + cg * 8;
  *reinterpret_cast<uint4*>(f) = o1;
  *reinterpret_cast<uint4*>(f + D) = o2;
}

// ------------------------------------------------------------------ tiled router

struct RouteTiledArgs {
  int32_t batch, n_q, h_kv, nb, block, topk;
  int32_t S;                 // table rows (sub-blocks) per block

  int32_t n_tiles, n_units;
  int64_t q_offset;
  int32_t* block_idx;
  float* top_scores;
  uint32_t* err;
  // optional [batch * h_kv * n_tiles] flags: units whose flag is 0 are
  // skipped (every role reads the same flag; no output is written for them)
  const int32_t* unit_need;
  // seeds (0 snapshots: none): a unit whose first row sees snapshot s first
  // scores that snapshot's kSeedRows seed rows, at row (bg * n_snap + s) * kSeedRows
  int32_t n_snap;
};

constexpr int kSeedRows = 128;   // seed rows per snapshot: one chunk of columns

// The unit's seed snapshot, or -1: the last snapshot whose 32 (s + 1)
// blocks are all visible to the unit's first row (and so to all its rows).
__device__ __forceinline__ int unit_snap(const RouteTiledArgs& a, int row0) {
  if (a.n_snap == 0) return -1;
  const int64_t nv0 = min(static_cast<int64_t>(a.nb), (a.q_offset + row0 + 1) / a.block);
  return static_cast<int>(nv0 / 32) - 1;
}

__device__ __forceinline__ bool unit_skipped(const RouteTiledArgs& a, int bg, int row0) {
  return a.unit_need && a.unit_need[bg * a.n_tiles + row0 / 256] == 0;
}

template <int KF>
struct TiledCfg {
  static constexpr int RT = 2;                            // 128-row feature tiles per unit
  static constexpr int A_BOXES = KF / 64;                 // 64-wide K slices
  static constexpr int BOX_BYTES = 128 * 128;             // 128 rows x 64 bf16
  static constexpr int A_TILE = A_BOXES * BOX_BYTES;      // one 128-row feature tile
  static constexpr int A_BYTES = RT * A_TILE;             // a unit's feature rows
  static constexpr int NAB = (KF == 256) ? 1 : 2;         // unit buffers
  static constexpr int NS = 2;                            // table-slice ring
  // candidates per row (per epilogue group); a row's buffered candidates are
  // merged once some lane holds more than CAP - 16, so a deeper buffer merges
  // larger batches (the warp runs as many insertions as its fullest lane)
  static constexpr int CAP = 32;
  static constexpr int NACC = 4;                          // TMEM accumulators: 2 chunks x RT tiles
  static constexpr int NBAR = 2 * NAB + 2 * NS + 2 * NACC + 1;
  static constexpr int SMEM = 1024 + NAB * A_BYTES + NS * BOX_BYTES + RT * CAP * 128 * 8 + NBAR * 8 + 16;
  static constexpr int THREADS = 64 + RT * 128;           // TMA, MMA, RT epilogue groups
  static_assert(SMEM <= 232448, "shared memory");
};

// A unit is 256 query rows (two 128-row tensor-core tiles) of one (batch,
// kv-head): every table slice is loaded once for both tiles.
__device__ __forceinline__ void route_unit(const RouteTiledArgs& a, int r, int& bg, int& row0,
                                           int& nch) {
  const int BG = a.batch * a.h_kv;
  bg = r % BG;
  const int unit = a.n_tiles - 1 - r / BG;   // heaviest units first
  row0 = unit * 256;
  const int rows = min(256, a.n_q - row0);
  const int64_t pos = a.q_offset + row0 + rows - 1;
  const int nv = static_cast<int>(min(static_cast<int64_t>(a.nb), (pos + 1) / a.block));
  nch = (nv * a.S + 127) / 128;   // 128 table rows (sub-block columns) per chunk
}

// Snake order over rounds keeps every CTA's total work close to the mean.
__device__ __forceinline__ int route_unit_rank(int q) {
  return q * gridDim.x + ((q & 1) ? (gridDim.x - 1 - blockIdx.x) : blockIdx.x);
}

// Bounded wait on a phase that must already be in flight (teardown drain).
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity, uint32_t* err) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > kWaitLimitNs) {
      atomicCAS(err, 0u, SITE_DRAIN);
      return;
    }
  }
}

// Merges this row's buffered candidates into its top list: a descending
// register list of (score, block), KSEL long, of which the first k count.
// Candidates are inserted one at a time in arrival order (ascending block
// index) and an equal score is placed after the entries already held, so a
// lower block index wins ties.  Each insertion is a branchless shift over the
// list with independent compares; the loop runs to the warp's largest count
// (lanes past their own count insert -inf, which changes nothing).
// Inserts (x, xi) into the descending list at its place among entries
// J0 .. KSEL-1 (x not above entry J0 - 1): the entries from the insertion
// point shift down by one, the last drops out; an equal score goes after
// the entries already held.
template <int KSEL, int J0>
__device__ __forceinline__ void insert_tail(float (&Ls)[KSEL], int (&Li)[KSEL], float x, int xi) {
  bool gt[KSEL];
#pragma unroll
  for (int j = J0; j < KSEL; ++j) gt[j] = x > Ls[j];
#pragma unroll
  for (int j = KSEL - 1; j > J0; --j) {
    Ls[j] = gt[j - 1] ? Ls[j - 1] : (gt[j] ? x : Ls[j]);
    Li[j] = gt[j - 1] ? Li[j - 1] : (gt[j] ? xi : Li[j]);
  }
  Ls[J0] = gt[J0] ? x : Ls[J0];
  Li[J0] = gt[J0] ? xi : Li[J0];
}

template <int KSEL>
__device__ __forceinline__ void merge_candidates(float (&Ls)[KSEL], int (&Li)[KSEL], int& cnt, float& thr,
                                                 const uint2* my_cand, int k, bool empty_list) {
  if constexpr (KSEL == 32) {
    // the first merge of a row (its list still empty, at most 32 candidates):
    // one 32-key sorting network instead of 32 insertions; the keys order
    // (score desc, block asc), the insertions' order
    if (empty_list) {
      uint64_t key[32];
#pragma unroll
      for (int t = 0; t < 32; ++t) {
        const uint2 e = t < cnt ? my_cand[t * 128] : make_uint2(0u, 0u);
        key[t] = t < cnt ? make_key(e.x, e.y) : 0ull;
      }
      bitonic_sort_desc<32>(key);
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        Ls[j] = key[j] ? key_score(key[j]) : -INFINITY;
        Li[j] = key[j] ? static_cast<int>(key_block(key[j])) : -1;
      }
      cnt = 0;
      float kth = INFINITY;
#pragma unroll
      for (int j = 0; j < KSEL; ++j)
        if (j < k) kth = fminf(kth, Ls[j]);
      thr = kth;
      return;
    }
  }
  int n = cnt;
#pragma unroll
  for (int o = 16; o; o >>= 1) n = max(n, __shfl_xor_sync(0xFFFFFFFFu, n, o));
#pragma unroll 1
  for (int t = 0; t < n; ++t) {
    float x = -INFINITY;
    int xi = 0;
    if (t < cnt) {
      const uint2 e = my_cand[t * 128];
      x = __uint_as_float(e.x);
      xi = static_cast<int>(e.y);
    }
    insert_tail<KSEL, 0>(Ls, Li, x, xi);
  }
  cnt = 0;
  // the k-th best (the list is descending: the least of its first k)
  float kth = INFINITY;
#pragma unroll
  for (int j = 0; j < KSEL; ++j)
    if (j < k) kth = fminf(kth, Ls[j]);
  thr = kth;
}

// Appends the scores above the threshold (strictly: an equal score comes
// from a higher block index and would rank below the k-th) to the row's
// candidate buffer, in block order: independent compares build a take mask,
// then one store per set bit.  v holds the scores of blocks c0 .. c0+N-1.
template <int N, bool MASK>
__device__ __forceinline__ void filter_n(const uint32_t (&v)[N], int c0, int nvis, float thr,
                                         int& cnt, uint2* my_cand) {
  uint32_t take = 0;
#pragma unroll
  for (int t = 0; t < N; ++t) {
    bool tk = __uint_as_float(v[t]) > thr;
    if (MASK) tk = tk && (c0 + t < nvis);
    take |= tk ? (1u << t) : 0u;
  }
  // one store per taken score, lowest column first (block order)
  for (uint32_t m = take; m; m &= m - 1u) {
    const int t = __ffs(static_cast<int>(m)) - 1;
    uint32_t vt = v[0];
#pragma unroll
    for (int u = 1; u < N; ++u) vt = (t == u) ? v[u] : vt;
    my_cand[cnt * 128] = make_uint2(vt, static_cast<uint32_t>(c0 + t));
    ++cnt;
  }
}

// Block scores of 16 sub-block columns, S per block: the largest of each
// block's S sub-block scores (the scores are finite, so fmaxf is the max).
template <int S>
__device__ __forceinline__ void pool_columns(const uint32_t (&v)[16], uint32_t (&w)[16 / S]) {
#pragma unroll
  for (int t = 0; t < 16 / S; ++t) {
    float m = __uint_as_float(v[t * S]);
#pragma unroll
    for (int s = 1; s < S; ++s) m = fmaxf(m, __uint_as_float(v[t * S + s]));
    w[t] = __float_as_uint(m);
  }
}

// Filters one 16-column TMEM group of a row: c0 is the group's first
// column, so its blocks start at c0 / S.
template <int S>
__device__ __forceinline__ void filter_group(const uint32_t (&v)[16], int c0, int nvis, float thr,
                                             int& cnt, uint2* my_cand) {
  constexpr int N = 16 / S;
  const int b0 = c0 / S;
  uint32_t w[N];
  if constexpr (S == 1) {
#pragma unroll
    for (int t = 0; t < 16; ++t) w[t] = v[t];
  } else {
    pool_columns<S>(v, w);
  }
  // the group's largest score against the threshold first: most groups of
  // most rows hold no candidate once the threshold is high (the scores are
  // finite, so fmaxf is the maximum)
  float mx = __uint_as_float(w[0]);
#pragma unroll
  for (int t = 1; t < N; ++t) mx = fmaxf(mx, __uint_as_float(w[t]));
  if (!__any_sync(0xFFFFFFFFu, mx > thr)) return;
  if (__all_sync(0xFFFFFFFFu, b0 + N <= nvis))
    filter_n<N, false>(w, b0, nvis, thr, cnt, my_cand);
  else
    filter_n<N, true>(w, b0, nvis, thr, cnt, my_cand);
}

// Warp roles: 0 = TMA producer, 1 = MMA issuer (and TMEM owner), 2..5 and
// 6..9 = two epilogue groups, group g owning the unit's tile g (TMEM lane
// quadrant = warp % 4, one query row per thread).
template <int KF, int KSEL>
__global__ void __launch_bounds__(TiledCfg<KF>::THREADS, 1)
    route_tiled_kernel(const __grid_constant__ CUtensorMap tmF, const __grid_constant__ CUtensorMap tmT,
                       const __grid_constant__ CUtensorMap tmS, const RouteTiledArgs a) {
  using C = TiledCfg<KF>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + C::NAB * C::A_BYTES;
  uint2* cand = reinterpret_cast<uint2*>(sB + C::NS * C::BOX_BYTES);
  uint64_t* bars = reinterpret_cast<uint64_t*>(cand + C::RT * C::CAP * 128);
  uint64_t* a_full = bars;
  uint64_t* a_empty = a_full + C::NAB;
  uint64_t* b_full = a_empty + C::NAB;
  uint64_t* b_empty = b_full + C::NS;
  uint64_t* acc_full = b_empty + C::NS;
  uint64_t* acc_empty = acc_full + C::NACC;
  uint64_t* mma_done = acc_empty + C::NACC;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NAB; ++i) { mbar_init(&a_full[i], 1); mbar_init(&a_empty[i], 1); }
    for (int i = 0; i < C::NS; ++i) { mbar_init(&b_full[i], 1); mbar_init(&b_empty[i], 1); }
    for (int i = 0; i < C::NACC; ++i) { mbar_init(&acc_full[i], 1); mbar_init(&acc_empty[i], 4); }
    mbar_init(mma_done, 1);
    fence_barrier_init();
    tma_prefetch_desc(&tmF);
    tma_prefetch_desc(&tmT);
    if (a.n_snap) tma_prefetch_desc(&tmS);
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
    if (lane == 0) {
      uint32_t a_cnt = 0, b_cnt = 0;
      bool ok = true;
      for (int q = 0; ok; ++q) {
        const int r = route_unit_rank(q);
        if (r >= a.n_units) break;
        int bg, row0, nch;
        route_unit(a, r, bg, row0, nch);
        if (nch == 0 || unit_skipped(a, bg, row0)) continue;
        const int ab = a_cnt % C::NAB;
        if (!mbar_wait(&a_empty[ab], ((a_cnt / C::NAB) & 1) ^ 1, a.err, SITE_ROUTE_PRODUCER)) { ok = false; break; }
        mbar_arrive_expect_tx(&a_full[ab], C::A_BYTES);
        const int frow = bg * a.n_q + row0;   // rows past this (batch, kv-head) are never used
#pragma unroll
        for (int rt = 0; rt < C::RT; ++rt)
#pragma unroll
          for (int ks = 0; ks < C::A_BOXES; ++ks)
            tma_load_2d(sA + ab * C::A_BYTES + rt * C::A_TILE + ks * C::BOX_BYTES, &tmF, &a_full[ab], ks * 64,
                        frow + rt * 128);
        ++a_cnt;
        const int trow = bg * a.nb * a.S;
        const int snap = unit_snap(a, row0);
        // chunk -1: the unit's seed rows (when it has a snapshot)
        for (int j = (snap >= 0 ? -1 : 0); j < nch && ok; ++j) {
#pragma unroll
          for (int ks = 0; ks < C::A_BOXES; ++ks) {
            const int s = b_cnt % C::NS;
            if (!mbar_wait(&b_empty[s], ((b_cnt / C::NS) & 1) ^ 1, a.err, SITE_ROUTE_PRODUCER)) { ok = false; break; }
            mbar_arrive_expect_tx(&b_full[s], C::BOX_BYTES);
            if (j < 0)
              tma_load_2d(sB + s * C::BOX_BYTES, &tmS, &b_full[s], ks * 64, (bg * a.n_snap + snap) * kSeedRows);
            else
              tma_load_2d(sB + s * C::BOX_BYTES, &tmT, &b_full[s], ks * 64, trow + j * 128);
            ++b_cnt;
          }
        }
      }
      if (!ok) {   // make sure no copy is still landing in shared memory
        for (uint32_t n = (b_cnt > C::NS ? b_cnt - C::NS : 0); n < b_cnt; ++n)
          drain_wait(&b_full[n % C::NS], (n / C::NS) & 1, a.err);
        for (uint32_t n = (a_cnt > C::NAB ? a_cnt - C::NAB : 0); n < a_cnt; ++n)
          drain_wait(&a_full[n % C::NAB], (n / C::NAB) & 1, a.err);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t IDESC = umma_idesc_bf16(128, 128);
      uint32_t a_cnt = 0, b_cnt = 0, ch_cnt = 0;
      bool ok = true;
      const uint32_t sA_u = smem_u32(sA), sB_u = smem_u32(sB);
      for (int q = 0; ok; ++q) {
        const int r = route_unit_rank(q);
        if (r >= a.n_units) break;
        int bg, row0, nch;
        route_unit(a, r, bg, row0, nch);
        if (nch == 0 || unit_skipped(a, bg, row0)) continue;
        const int ab = a_cnt % C::NAB;
        if (!mbar_wait(&a_full[ab], (a_cnt / C::NAB) & 1, a.err, SITE_ROUTE_MMA)) { ok = false; break; }
        tc_fence_after();
        for (int j = (unit_snap(a, row0) >= 0 ? -1 : 0); j < nch && ok; ++j) {
          // chunk slot: accumulators 2 slot + rt, one per tile
          const int slot = ch_cnt & 1;
          const uint32_t par = ((ch_cnt >> 1) & 1) ^ 1;
          if (!mbar_wait(&acc_empty[2 * slot], par, a.err, SITE_ROUTE_MMA) ||
              !mbar_wait(&acc_empty[2 * slot + 1], par, a.err, SITE_ROUTE_MMA)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int ks = 0; ks < C::A_BOXES; ++ks) {
            const int s = b_cnt % C::NS;
            if (!mbar_wait(&b_full[s], (b_cnt / C::NS) & 1, a.err, SITE_ROUTE_MMA)) { ok = false; break; }
            tc_fence_after();
            const uint32_t bslice = sB_u + s * C::BOX_BYTES;
#pragma unroll
            for (int rt = 0; rt < C::RT; ++rt) {
              const uint32_t d_tmem = tmem_base + (2 * slot + rt) * 128;
              const uint32_t atile = sA_u + ab * C::A_BYTES + rt * C::A_TILE + ks * C::BOX_BYTES;
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                umma_bf16(d_tmem, umma_desc_sw128(atile + kk * 32), umma_desc_sw128(bslice + kk * 32), IDESC,
                          (ks | kk) != 0 ? 1u : 0u);
            }
            umma_commit(&b_empty[s]);
            ++b_cnt;
          }
          if (!ok) break;
          umma_commit(&acc_full[2 * slot]);
          umma_commit(&acc_full[2 * slot + 1]);
          ++ch_cnt;
        }
        if (!ok) break;
        umma_commit(&a_empty[ab]);
        ++a_cnt;
      }
      umma_commit(mma_done);        // all issued MMAs complete before TMEM is freed
      drain_wait(mma_done, 0, a.err);
    }
  } else {
    const int grp = (warp - 2) >> 2;   // the unit's tile this group owns
    const int eq = warp & 3;
    const int row = eq * 32 + lane;
    uint2* my_cand = cand + grp * (C::CAP * 128) + row;
    uint32_t ch_cnt = 0;
    bool ok = true;
    for (int q = 0; ok; ++q) {
      const int r = route_unit_rank(q);
      if (r >= a.n_units) break;
      int bg, row0, nch;
      route_unit(a, r, bg, row0, nch);
      if (unit_skipped(a, bg, row0)) continue;
      const int i = row0 + grp * 128 + row;
      const bool valid = i < a.n_q;
      const int nvis = valid ? static_cast<int>(min(static_cast<int64_t>(a.nb), (a.q_offset + i + 1) / a.block)) : 0;
      float Ls[KSEL];
      int Li[KSEL];
#pragma unroll
      for (int j = 0; j < KSEL; ++j) { Ls[j] = -INFINITY; Li[j] = -1; }
      float thr = -INFINITY;
      float floor_thr = -INFINITY;   // the seeds' lower bound on the k-th best score
      int cnt = 0;
      bool empty_list = true;   // warp-uniform: no merge of this unit yet
      const int snap = unit_snap(a, row0);
      if (snap >= 0) {
        // chunk -1: the scores of the snapshot's 128 seed blocks, all visible
        // to every row of the unit, in ng = 128 / gs disjoint groups of gs
        // consecutive columns (ng the least power of two >= topk).  Each
        // group's largest score belongs to a distinct block, so at least ng
        // >= topk blocks score at least the least of the ng maxima: a lower
        // bound on the row's k-th best score.  The threshold sits a little
        // below it, so a block scoring exactly that much still passes.
        const int acc = 2 * (ch_cnt & 1) + grp;
        ok = __all_sync(0xFFFFFFFFu, mbar_wait(&acc_full[acc], (ch_cnt >> 1) & 1, a.err, SITE_ROUTE_EPILOGUE));
        if (!ok) break;
        tc_fence_after();
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(eq * 32) << 16) + acc * 128;
        int ng = 1;
        while (ng < a.topk) ng <<= 1;
        const int gs = kSeedRows / ng;
        float mn = INFINITY, gmax = -INFINITY;
#pragma unroll 1
        for (int sub = 0; sub < kSeedRows / 16; ++sub) {
          uint32_t v[16];
          tmem_ld16(taddr + sub * 16, v);
          tmem_wait_ld();
#pragma unroll
          for (int t = 0; t < 16; ++t) {
            gmax = fmaxf(gmax, __uint_as_float(v[t]));
            if (((sub * 16 + t + 1) & (gs - 1)) == 0) { mn = fminf(mn, gmax); gmax = -INFINITY; }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[acc]);
        floor_thr = mn - (fabsf(mn) * 0x1p-16f + 0x1p-24f);
        thr = floor_thr;
        ++ch_cnt;
      }
      for (int j = 0; j < nch; ++j) {
        const int acc = 2 * (ch_cnt & 1) + grp;
        ok = __all_sync(0xFFFFFFFFu, mbar_wait(&acc_full[acc], (ch_cnt >> 1) & 1, a.err, SITE_ROUTE_EPILOGUE));
        if (!ok) break;
        tc_fence_after();
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(eq * 32) << 16) + acc * 128;
#pragma unroll 1
        for (int sub = 0; sub < 8; ++sub) {
          uint32_t v[16];
          tmem_ld16(taddr + sub * 16, v);
          tmem_wait_ld();
          if (sub == 7) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[acc]);
          }
          const int c0 = j * 128 + sub * 16;
          if (a.S == 1)
            filter_group<1>(v, c0, nvis, thr, cnt, my_cand);
          else if (a.S == 2)
            filter_group<2>(v, c0, nvis, thr, cnt, my_cand);
          else
            filter_group<4>(v, c0, nvis, thr, cnt, my_cand);
          if (__any_sync(0xFFFFFFFFu, cnt > C::CAP - 16)) {
            merge_candidates<KSEL>(Ls, Li, cnt, thr, my_cand, a.topk, empty_list);
            thr = fmaxf(thr, floor_thr);
            empty_list = false;
          }
        }
        ++ch_cnt;
      }
      if (!ok) break;
      if (__any_sync(0xFFFFFFFFu, cnt > 0)) merge_candidates<KSEL>(Ls, Li, cnt, thr, my_cand, a.topk, empty_list);
      if (valid) {
        uint32_t ob[KSEL];
        float os[KSEL];
#pragma unroll
        for (int j = 0; j < KSEL; ++j) {
          const bool use = (j < a.topk) && Li[j] >= 0;
          ob[j] = use ? static_cast<uint32_t>(Li[j]) : 0xFFFFFFFFu;
          os[j] = use ? Ls[j] : -INFINITY;
        }
        bitonic_sort_asc_u32<KSEL>(ob, os);
        const int b = bg / a.h_kv, g = bg % a.h_kv;
        const int64_t o = ((static_cast<int64_t>(b) * a.n_q + i) * a.h_kv + g) * a.topk;
        // four entries per store when the row's entries are 16-byte aligned
        if ((a.topk & 3) == 0 && (reinterpret_cast<uintptr_t>(a.block_idx) & 15) == 0 &&
            (reinterpret_cast<uintptr_t>(a.top_scores) & 15) == 0) {
#pragma unroll
          for (int j = 0; j < KSEL; j += 4) {
            if (j < a.topk) {
              int4 w;
              w.x = ob[j] == 0xFFFFFFFFu ? -1 : static_cast<int32_t>(ob[j]);
              w.y = ob[j + 1] == 0xFFFFFFFFu ? -1 : static_cast<int32_t>(ob[j + 1]);
              w.z = ob[j + 2] == 0xFFFFFFFFu ? -1 : static_cast<int32_t>(ob[j + 2]);
              w.w = ob[j + 3] == 0xFFFFFFFFu ? -1 : static_cast<int32_t>(ob[j + 3]);
              *reinterpret_cast<int4*>(a.block_idx + o + j) = w;
              if (a.top_scores)
                *reinterpret_cast<float4*>(a.top_scores + o + j) = make_float4(os[j], os[j + 1], os[j + 2], os[j + 3]);
            }
          }
        } else {
#pragma unroll
          for (int j = 0; j < KSEL; ++j) {
            if (j < a.topk) {
              a.block_idx[o + j] = ob[j] == 0xFFFFFFFFu ? -1 : static_cast<int32_t>(ob[j]);
              if (a.top_scores) a.top_scores[o + j] = os[j];
            }
          }
        }
      }
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

template <int KF, int KSEL>
cudaError_t run_tiled(const ssa_params& p, const CUtensorMap& tmF, const CUtensorMap& tmT, const CUtensorMap* tmS,
                      int n_snap, int32_t* idx, float* scores, const int32_t* unit_need, const LaunchCtx& c) {
  using C = TiledCfg<KF>;
  RouteTiledArgs a;
  a.batch = p.batch; a.n_q = p.n_q; a.h_kv = p.h_kv; a.nb = p.n_kv / p.block;
  a.block = p.block; a.topk = p.topk; a.S = rows_per_block(p);
  a.n_tiles = (p.n_q + 255) / 256;   // 256-row units per (batch, kv-head)
  a.n_units = p.batch * p.h_kv * a.n_tiles;
  a.q_offset = p.q_offset;
  a.block_idx = idx; a.top_scores = scores; a.err = c.err;
  a.unit_need = unit_need;
  a.n_snap = tmS ? n_snap : 0;
  cudaError_t e = cudaFuncSetAttribute(route_tiled_kernel<KF, KSEL>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
  if (e != cudaSuccess) return e;
  const int grid = a.n_units < c.sm_count ? a.n_units : c.sm_count;
  route_tiled_kernel<KF, KSEL><<<grid, C::THREADS, C::SMEM, c.stream>>>(tmF, tmT, tmS ? *tmS : tmT, a);
  note_launch();
  return cudaGetLastError();
}

// ------------------------------------------------------------------ row-wise routers

struct RowArgs {
  int32_t n_q, h_kv, nb, block, topk;
  int32_t S;                 // summary rows (sub-blocks) per block
  int64_t q_offset;
  float half_beta;
  int32_t* block_idx;
  float* top_scores;
  const uint8_t* skip;       // optional [b, n_q, h_kv]: rows whose byte is nonzero are skipped
};

// Writes the top-k of keys[0..n) (distinct and nonzero: a block index in
// the low half) in ascending block order.  A radix select, most significant
// 8-bit digit first, finds the k-th largest key: per digit, a histogram of
// the keys that share the digits decided so far (warp-aggregated
// shared-memory atomics), then one warp finds the digit holding the k-th key.
// It stops at the first digit whose keys are all needed, so the keys >= the
// decided prefix (lower digits zero) are exactly the k largest; they are
// collected and ranked by block index.
__device__ void select_and_write(const uint64_t* keys, int n, const RowArgs& a, int64_t out) {
  __shared__ uint32_t hist[256];
  __shared__ uint64_t s_prefix;
  __shared__ int s_krem, s_done, s_nsel;
  __shared__ uint64_t sel[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int k = min(a.topk, n);
  if (tid == 0) { s_prefix = 0; s_krem = a.topk; s_done = n <= a.topk; s_nsel = 0; }
  __syncthreads();   // also orders the callers' key writes before the reads below
  uint64_t mask = 0;
  for (int shift = 56; shift >= 0 && !s_done; shift -= 8) {
    for (int j = tid; j < 256; j += blockDim.x) hist[j] = 0;
    __syncthreads();
    const uint64_t prefix = s_prefix;
    for (int c0 = warp * 32; c0 < n; c0 += blockDim.x) {   // warp-uniform trip count
      const int c = c0 + lane;
      const uint64_t key = c < n ? keys[c] : 0;
      const bool in = c < n && (key & mask) == prefix;
      const uint32_t digit = in ? static_cast<uint32_t>(key >> shift) & 255u : 256u;
      const uint32_t same = __match_any_sync(0xFFFFFFFFu, digit);
      if (in && lane == __ffs(static_cast<int>(same)) - 1) atomicAdd(&hist[digit], __popc(same));
    }
    __syncthreads();
    if (warp == 0) {
      uint32_t h[8], sum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) { h[j] = hist[lane * 8 + j]; sum += h[j]; }
      uint32_t suf = sum;   // keys in this lane's digits and all higher ones
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_down_sync(0xFFFFFFFFu, suf, o);
        if (lane + o < 32) suf += v;
      }
      const uint32_t krem = static_cast<uint32_t>(s_krem);
      const uint32_t above = suf - sum;
      if (above < krem && krem <= suf) {   // the k-th key's digit is in this lane's range
        uint32_t cum = above;
        int d = lane * 8;
        uint32_t cnt = 0;
#pragma unroll
        for (int j = 7; j >= 0; --j) {
          if (cnt == 0 && cum + h[j] >= krem) { d = lane * 8 + j; cnt = h[j]; }
          else if (cnt == 0) cum += h[j];
        }
        s_prefix = prefix | (static_cast<uint64_t>(d) << shift);
        s_krem = static_cast<int>(krem - cum);
        s_done = cnt == krem - cum;
      }
    }
    __syncthreads();
    mask |= 0xFFull << shift;
  }
  const uint64_t T = s_prefix;   // 0 when every key is taken
  for (int c = tid; c < n; c += blockDim.x) {
    const uint64_t key = keys[c];
    if (key >= T) {
      const int slot = atomicAdd(&s_nsel, 1);
      if (slot < 32) sel[slot] = key;
    }
  }
  __syncthreads();
  if (warp == 0) {
    const uint64_t key = lane < k ? sel[lane] : 0;
    const uint32_t blk = key ? key_block(key) : 0xFFFFFFFFu;
    // valid entries are ranked by block index; empty slots follow, in lane order
    const uint32_t vmask = __ballot_sync(0xFFFFFFFFu, key != 0);
    int rank = 0;
    for (int o = 0; o < 32; ++o) {
      const uint32_t other = __shfl_sync(0xFFFFFFFFu, blk, o);
      rank += (other < blk) ? 1 : 0;
    }
    if (!key) rank = __popc(vmask) + __popc(~vmask & ((1u << lane) - 1u));
    if (lane < a.topk) {
      a.block_idx[out + rank] = key ? static_cast<int32_t>(blk) : -1;
      if (a.top_scores) a.top_scores[out + rank] = key ? key_score(key) : -INFINITY;
    }
  }
}

// bf16 table, one CTA per (query row, kv-head, batch).  Lane l of every warp
// holds features [FPL*l, FPL*l + FPL) of the row and dots them with the
// matching slice of a table row; a warp reduction gives the block score.
template <int D, int G>
__global__ void __launch_bounds__(256) route_rowwise_bf16_kernel(const __nv_bfloat16* __restrict__ Q,
                                                                 const __nv_bfloat16* __restrict__ T,
                                                                 const RowArgs a) {
  constexpr int FPL = 2 * D / 32;   // features per lane: 8 (d=128) or 4 (d=64)
  extern __shared__ uint64_t keys[];
  const int i = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  if (a.skip && a.skip[(static_cast<int64_t>(b) * a.n_q + i) * a.h_kv + g]) return;   // whole CTA
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
  const int64_t pos = a.q_offset + i;
  const int nvis = static_cast<int>(min(static_cast<int64_t>(a.nb), (pos + 1) / a.block));
  const int h_q = a.h_kv * G;
  const bool second = lane >= 16;
  const int dim0 = (lane % 16) * FPL;
  float f[FPL];
  {
    float qs[FPL], qq[FPL];
#pragma unroll
    for (int v = 0; v < FPL; ++v) { qs[v] = 0.f; qq[v] = 0.f; }
    const __nv_bfloat16* q = Q + ((static_cast<int64_t>(b) * a.n_q + i) * h_q + static_cast<int64_t>(g) * G) * D + dim0;
#pragma unroll
    for (int h = 0; h < G; ++h) {
#pragma unroll
      for (int v = 0; v < FPL; ++v) {
        const float x = __bfloat162float(q[h * D + v]);
        qs[v] = __fadd_rn(qs[v], x);
        qq[v] = __fmaf_rn(x, x, qq[v]);
      }
    }
#pragma unroll
    for (int v = 0; v < FPL; ++v) {
      const float raw = second ? __fmul_rn(a.half_beta, qq[v]) : qs[v];
      f[v] = __bfloat162float(__float2bfloat16_rn(raw));
    }
  }
  // table rows are sub-blocks (S per block); a warp scores two runs of 4
  // consecutive rows per pass (each run holds 4 / S whole blocks), its eight
  // row loads issued together: past the last row a lane reads row 0 and the
  // score is dropped
  const int nrows = nvis * a.S;
  const __nv_bfloat16* trow = T + (static_cast<int64_t>(b) * a.h_kv + g) * a.nb * a.S * (2 * D) + lane * FPL;
  for (int c0 = warp * 8; c0 < nrows; c0 += 64) {
    uint4 raw[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int c = c0 + u < nrows ? c0 + u : 0;
      const __nv_bfloat16* t = trow + static_cast<int64_t>(c) * (2 * D);
      if (FPL == 8) {
        raw[u] = __ldg(reinterpret_cast<const uint4*>(t));
      } else {
        const uint2 r2 = __ldg(reinterpret_cast<const uint2*>(t));
        raw[u] = make_uint4(r2.x, r2.y, 0u, 0u);
      }
    }
    float part[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const uint32_t w[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
      part[u] = 0.f;
#pragma unroll
      for (int j = 0; j < FPL / 2; ++j) {
        part[u] = __fmaf_rn(f[2 * j], __uint_as_float(w[j] << 16), part[u]);
        part[u] = __fmaf_rn(f[2 * j + 1], __uint_as_float(w[j] & 0xFFFF0000u), part[u]);
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) part[u] += __shfl_xor_sync(0xFFFFFFFFu, part[u], o);
    }
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      float* pq = part + 4 * q;
      // a block's score is the largest of its sub-blocks' scores
      if (a.S >= 2) { pq[0] = fmaxf(pq[0], pq[1]); pq[1] = fmaxf(pq[2], pq[3]); }
      if (a.S == 4) pq[0] = fmaxf(pq[0], pq[1]);
      const int nper = 4 / a.S;
      for (int u = 0; u < nper; ++u) {
        const int c = (c0 + 4 * q) / a.S + u;
        if (lane == 0 && c < nvis) keys[c] = make_key(__float_as_uint(pq[u]), c);
      }
    }
  }
  const int64_t out = ((static_cast<int64_t>(b) * a.n_q + i) * a.h_kv + g) * a.topk;
  select_and_write(keys, nvis, a, out);
}

// float32 summaries: s_c = sum_h (<q_h, mu_c> + (beta/2) q_h^T Sigma_c q_h).
// One warp per block; lane l owns rows s = l, l+32, ... of Sigma_c (full)
// or dimensions l, l+32, ... (diagonal).
template <int D, int G, bool FULL>
__global__ void __launch_bounds__(256) route_rowwise_f32_kernel(const float* __restrict__ Q,
                                                                const float* __restrict__ MU,
                                                                const float* __restrict__ SG,
                                                                const RowArgs a) {
  extern __shared__ uint64_t keys[];
  __shared__ float qsm[G][D];
  const int i = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int lane = threadIdx.x % 32, warp = threadIdx.x / 32;
  const int64_t pos = a.q_offset + i;
  const int nvis = static_cast<int>(min(static_cast<int64_t>(a.nb), (pos + 1) / a.block));
  const int h_q = a.h_kv * G;
  const float* q = Q + ((static_cast<int64_t>(b) * a.n_q + i) * h_q + static_cast<int64_t>(g) * G) * D;
  for (int e = threadIdx.x; e < G * D; e += blockDim.x) qsm[e / D][e % D] = q[e];
  __syncthreads();
  // summary rows are sub-blocks, S per block; a warp scores a block's S
  // rows and keeps the largest
  const int64_t bgrow = (static_cast<int64_t>(b) * a.h_kv + g) * a.nb * a.S;
  for (int cb = warp; cb < nvis; cb += 8) {
    float best = -INFINITY;
    for (int sb = 0; sb < a.S; ++sb) {
      const int64_t c = static_cast<int64_t>(cb) * a.S + sb;
      const float* mu = MU + (bgrow + c) * D;
      float acc = 0.f;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float lin = 0.f, quad = 0.f;
#pragma unroll
        for (int ss = 0; ss < D / 32; ++ss) {
          const int s = lane + 32 * ss;
          const float qv = qsm[h][s];
          lin = __fmaf_rn(qv, __ldg(mu + s), lin);
          if (FULL) {
            const float* srow = SG + ((bgrow + c) * D + s) * D;
            float u = 0.f;
#pragma unroll 8
            for (int t = 0; t < D; ++t) u = __fmaf_rn(__ldg(srow + t), qsm[h][t], u);
            quad = __fmaf_rn(qv, u, quad);
          } else {
            quad = __fmaf_rn(qv * qv, __ldg(SG + (bgrow + c) * D + s), quad);
          }
        }
        acc += lin + a.half_beta * quad;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
      best = fmaxf(best, acc);
    }
    if (lane == 0) keys[cb] = make_key(__float_as_uint(best), cb);
  }
  const int64_t out = ((static_cast<int64_t>(b) * a.n_q + i) * a.h_kv + g) * a.topk;
  select_and_write(keys, nvis, a, out);
}

// float32 summaries for runs of query rows: a CTA takes 32/G consecutive
// queries (32 (query, head) pairs) of one kv-head and walks the blocks,
// staging each block's mu_c and Sigma_c in shared memory once for all of
// them (the row-wise kernel reads them once per query).  Eight threads share
// a (query, head) pair, each taking every eighth row of Sigma_c; the block
// scores of each query stay in shared memory, and a warp per query sorts
// them and writes its top k.  Sub-block rows are max-pooled per block.
template <int D, int G, bool FULL>
__global__ void __launch_bounds__(256) route_qtile_f32_kernel(const float* __restrict__ Q,
                                                              const float* __restrict__ MU,
                                                              const float* __restrict__ SG, const RowArgs a,
                                                              int n2) {
  constexpr int QT = 32 / G;            // queries per CTA
  constexpr int SP = FULL ? D + 1 : D;  // padded Sigma row (bank spread)
  extern __shared__ uint64_t keys[];    // [QT][n2]
  float* qs = reinterpret_cast<float*>(keys + QT * n2);   // [32][D]
  float* sgs = qs + 32 * D;                               // [D][SP] or [D]
  float* mus = sgs + (FULL ? D * SP : D);                 // [D]
  float* sc = mus + D;                                    // [32] (query, head) scores
  const int i0 = blockIdx.x * QT, g = blockIdx.y, b = blockIdx.z;
  const int h_q = a.h_kv * G;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // the tile's (query, head) rows of Q; rows past n_q are zero.  Full Sigma:
  // stored transposed, qs[t * 32 + r]
  for (int e = threadIdx.x; e < 32 * D; e += 256) {
    const int r = e / D, t = e % D, qq = r / G, h = r % G;
    const int i = i0 + qq;
    const float v = i < a.n_q ? Q[((static_cast<int64_t>(b) * a.n_q + i) * h_q + static_cast<int64_t>(g) * G + h) * D + t]
                              : 0.f;
    qs[FULL ? t * 32 + r : e] = v;
  }
  const int64_t last = a.q_offset + min(i0 + QT, a.n_q) - 1;
  const int ncmax = static_cast<int>(min(static_cast<int64_t>(a.nb), (last + 1) / a.block));
  const int64_t bgrow = (static_cast<int64_t>(b) * a.h_kv + g) * a.nb * a.S;
  if constexpr (FULL) {
    // Register-tiled: thread (sg, rg) accumulates U[s][r] = sum_t Sigma[t][s] q_r[t]
    // for its D/16 columns s and two rows r (q^T Sigma^T q = q^T Sigma q), from
    // contiguous Sigma rows; the next summary row is fetched into registers
    // while this one is used.
    constexpr int SPT = D / 16;
    constexpr int NPF = D * D / 4 / 256;
    float* red = sc + 32;   // [16][32] partial scores
    const int sg = threadIdx.x >> 4, r0 = (threadIdx.x & 15) * 2, s0 = sg * SPT;
    const int nrow = ncmax * a.S;
    float4 pf[NPF];
    float4 pm = make_float4(0.f, 0.f, 0.f, 0.f);
    auto fetch = [&](int u) {
      const float4* src = reinterpret_cast<const float4*>(SG + (bgrow + u) * D * D);
#pragma unroll
      for (int j = 0; j < NPF; ++j) pf[j] = __ldg(src + threadIdx.x + j * 256);
      if (threadIdx.x < D / 4) pm = __ldg(reinterpret_cast<const float4*>(MU + (bgrow + u) * D) + threadIdx.x);
    };
    auto stage = [&]() {
      float4* dst = reinterpret_cast<float4*>(sgs);
#pragma unroll
      for (int j = 0; j < NPF; ++j) dst[threadIdx.x + j * 256] = pf[j];
      if (threadIdx.x < D / 4) reinterpret_cast<float4*>(mus)[threadIdx.x] = pm;
    };
    if (nrow > 0) {
      fetch(0);
      stage();
    }
    float best = -INFINITY;   // threads < QT: the query's best sub-block score
    const int iq = i0 + static_cast<int>(threadIdx.x);   // threads < QT: their query's visible blocks
    const int nvq = threadIdx.x < QT && iq < a.n_q
                        ? static_cast<int>(min(static_cast<int64_t>(a.nb), (a.q_offset + iq + 1) / a.block)) : 0;
    for (int u = 0; u < nrow; ++u) {
      __syncthreads();   // row u staged, the previous row's scores consumed
      if (u + 1 < nrow) fetch(u + 1);
      float acc[SPT][2];
#pragma unroll
      for (int i = 0; i < SPT; ++i) { acc[i][0] = 0.f; acc[i][1] = 0.f; }
#pragma unroll 4
      for (int t = 0; t < D; ++t) {
        float sv[SPT];
#pragma unroll
        for (int i = 0; i < SPT; i += 4) {
          const float4 x = *reinterpret_cast<const float4*>(sgs + t * D + s0 + i);
          sv[i] = x.x; sv[i + 1] = x.y; sv[i + 2] = x.z; sv[i + 3] = x.w;
        }
        const float2 qv = *reinterpret_cast<const float2*>(qs + t * 32 + r0);
#pragma unroll
        for (int i = 0; i < SPT; ++i) {
          acc[i][0] = __fmaf_rn(sv[i], qv.x, acc[i][0]);
          acc[i][1] = __fmaf_rn(sv[i], qv.y, acc[i][1]);
        }
      }
      // this thread's columns of <q, mu> + (beta/2) q^T Sigma q for its two rows
      float p0 = 0.f, p1 = 0.f;
#pragma unroll
      for (int i = 0; i < SPT; ++i) {
        const float2 qv = *reinterpret_cast<const float2*>(qs + (s0 + i) * 32 + r0);
        const float m = mus[s0 + i];
        p0 = __fmaf_rn(qv.x, __fmaf_rn(a.half_beta, acc[i][0], m), p0);
        p1 = __fmaf_rn(qv.y, __fmaf_rn(a.half_beta, acc[i][1], m), p1);
      }
      *reinterpret_cast<float2*>(red + sg * 32 + r0) = make_float2(p0, p1);
      __syncthreads();   // partials written, row u read
      if (threadIdx.x < 32) {
        float v = 0.f;
#pragma unroll
        for (int j = 0; j < 16; ++j) v += red[j * 32 + threadIdx.x];
        sc[threadIdx.x] = v;
      }
      if (u + 1 < nrow) stage();
      __syncthreads();
      // the group's score of each query for this summary row: its heads'
      // scores summed in head order; the block keeps its largest sub-block
      const int cb = u / a.S, sb = u % a.S;
      if (threadIdx.x < QT) {
        float gsum = 0.f;
#pragma unroll
        for (int h = 0; h < G; ++h) gsum += sc[threadIdx.x * G + h];
        best = fmaxf(best, gsum);
        if (sb == a.S - 1) {
          const int qq = threadIdx.x;
          keys[qq * n2 + cb] = cb < nvq ? make_key(__float_as_uint(best), cb) : 0ull;
          best = -INFINITY;
        }
      }
    }
  } else {
  const int r = threadIdx.x >> 3, part = threadIdx.x & 7;   // (query, head) row, its eighth
  for (int cb = 0; cb < ncmax; ++cb) {
    float best = -INFINITY;   // threads < QT: the query's best sub-block score
    for (int sb = 0; sb < a.S; ++sb) {
      const int64_t row = bgrow + static_cast<int64_t>(cb) * a.S + sb;
      __syncthreads();   // the previous summary row is consumed
      for (int e = threadIdx.x; e < D; e += 256) mus[e] = MU[row * D + e];
      if (FULL) {
        for (int e = threadIdx.x; e < D * D; e += 256) sgs[(e / D) * SP + e % D] = SG[row * D * D + e];
      } else {
        for (int e = threadIdx.x; e < D; e += 256) sgs[e] = SG[row * D + e];
      }
      __syncthreads();
      const float* q = qs + r * D;
      float lin = 0.f, quad = 0.f;
#pragma unroll 4
      for (int s2 = part; s2 < D; s2 += 8) {
        const float qv = q[s2];
        lin = __fmaf_rn(qv, mus[s2], lin);
        if (FULL) {
          const float* srow = sgs + s2 * SP;
          float u = 0.f;
#pragma unroll 8
          for (int t = 0; t < D; ++t) u = __fmaf_rn(srow[t], q[t], u);
          quad = __fmaf_rn(qv, u, quad);
        } else {
          quad = __fmaf_rn(qv * qv, sgs[s2], quad);
        }
      }
      float v = lin + a.half_beta * quad;
#pragma unroll
      for (int o = 4; o; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
      // the group's score of each query for this summary row: its heads'
      // scores summed in head order; the block keeps its largest sub-block
      if (part == 0) sc[r] = v;
      __syncthreads();
      if (threadIdx.x < QT) {
        float acc = 0.f;
#pragma unroll
        for (int h = 0; h < G; ++h) acc += sc[threadIdx.x * G + h];
        best = fmaxf(best, acc);
      }
    }
    if (threadIdx.x < QT) {
      const int qq = threadIdx.x, i = i0 + qq;
      const int64_t pos = a.q_offset + i;
      const bool vis = i < a.n_q && cb < min(static_cast<int64_t>(a.nb), (pos + 1) / a.block);
      keys[qq * n2 + cb] = vis ? make_key(__float_as_uint(best), cb) : 0ull;
    }
  }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < QT * n2; e += 256)
    if (e % n2 >= ncmax) keys[e] = 0ull;
  __syncthreads();
  // a warp per query: bitonic sort of its n2 keys (descending), then the top
  // k in ascending block order
  for (int qq = warp; qq < QT; qq += 8) {
    const int i = i0 + qq;
    if (i >= a.n_q) continue;   // warp-uniform
    uint64_t* kq = keys + qq * n2;
    for (int size = 2; size <= n2; size <<= 1) {
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        for (int t = lane; t < n2 / 2; t += 32) {
          const int x = 2 * t - (t & (stride - 1));
          const int y = x + stride;
          const bool desc = (x & size) == 0;
          const uint64_t kx = kq[x], ky = kq[y];
          if (desc ? (kx < ky) : (kx > ky)) { kq[x] = ky; kq[y] = kx; }
        }
        __syncwarp();
      }
    }
    const uint64_t key = (lane < a.topk && lane < n2) ? kq[lane] : 0ull;
    const uint32_t blk = key ? key_block(key) : 0xFFFFFFFFu;
    const uint32_t vmask = __ballot_sync(0xFFFFFFFFu, key != 0);
    int rank = 0;
    for (int o = 0; o < 32; ++o) {
      const uint32_t other = __shfl_sync(0xFFFFFFFFu, blk, o);
      rank += (other < blk) ? 1 : 0;
    }
    if (!key) rank = __popc(vmask) + __popc(~vmask & ((1u << lane) - 1u));
    const int64_t out = ((static_cast<int64_t>(b) * a.n_q + i) * a.h_kv + g) * a.topk;
    if (lane < a.topk) {
      a.block_idx[out + rank] = key ? static_cast<int32_t>(blk) : -1;
      if (a.top_scores) a.top_scores[out + rank] = key ? key_score(key) : -INFINITY;
    }
  }
}

RowArgs row_args(const ssa_params& p, int32_t* idx, float* scores) {
  RowArgs a;
  a.n_q = p.n_q; a.h_kv = p.h_kv; a.nb = p.n_kv / p.block; a.block = p.block; a.topk = p.topk;
  a.S = rows_per_block(p);
  a.q_offset = p.q_offset;
  a.half_beta = p.beta * 0.5f;   // exact
  a.block_idx = idx; a.top_scores = scores;
  a.skip = nullptr;
  return a;
}

template <int D, int G>
cudaError_t run_features(const ssa_params& p, const void* Q, void* F, const LaunchCtx& c) {
  constexpr int RPC = 256 / (D / 8);
  const int64_t rows = static_cast<int64_t>(p.batch) * p.h_kv * p.n_q;
  const int64_t grid = (rows + RPC - 1) / RPC;
  features_kernel<D, G><<<static_cast<unsigned>(grid), 256, 0, c.stream>>>(
      static_cast<const __nv_bfloat16*>(Q), static_cast<__nv_bfloat16*>(F), rows, p.n_q, p.h_kv,
      p.beta * 0.5f);
  note_launch();
  return cudaGetLastError();
}

template <int D>
cudaError_t features_g(const ssa_params& p, const void* Q, void* F, const LaunchCtx& c) {
  switch (p.h_q / p.h_kv) {
    case 1: return run_features<D, 1>(p, Q, F, c);
    case 2: return run_features<D, 2>(p, Q, F, c);
    case 4: return run_features<D, 4>(p, Q, F, c);
    case 8: return run_features<D, 8>(p, Q, F, c);
  }
  return cudaErrorInvalidValue;
}

int row_smem_bytes(const ssa_params& p) {
  int n2 = 1;
  while (n2 < p.n_kv / p.block) n2 <<= 1;
  return n2 * 8;
}

template <int D, int G>
cudaError_t run_rowwise_bf16(const ssa_params& p, const void* Q, const void* T, int32_t* idx,
                             float* scores, const uint8_t* skip, const LaunchCtx& c) {
  RowArgs ra = row_args(p, idx, scores);
  ra.skip = skip;
  const int smem = row_smem_bytes(p);
  cudaError_t e = cudaFuncSetAttribute(route_rowwise_bf16_kernel<D, G>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.n_q, p.h_kv, p.batch);
  route_rowwise_bf16_kernel<D, G><<<grid, 256, smem, c.stream>>>(
      static_cast<const __nv_bfloat16*>(Q), static_cast<const __nv_bfloat16*>(T), ra);
  note_launch();
  return cudaGetLastError();
}

template <int D>
cudaError_t rowwise_bf16_g(const ssa_params& p, const void* Q, const void* T, int32_t* idx,
                           float* scores, const uint8_t* skip, const LaunchCtx& c) {
  switch (p.h_q / p.h_kv) {
    case 1: return run_rowwise_bf16<D, 1>(p, Q, T, idx, scores, skip, c);
    case 2: return run_rowwise_bf16<D, 2>(p, Q, T, idx, scores, skip, c);
    case 4: return run_rowwise_bf16<D, 4>(p, Q, T, idx, scores, skip, c);
    case 8: return run_rowwise_bf16<D, 8>(p, Q, T, idx, scores, skip, c);
  }
  return cudaErrorInvalidValue;
}

// Shared memory of route_qtile_f32_kernel, 0 when it does not fit.
template <int D, int G, bool FULL>
int qtile_smem_bytes(const ssa_params& p) {
  int n2 = 1;
  while (n2 < p.n_kv / p.block) n2 <<= 1;
  const int64_t bytes = static_cast<int64_t>(32 / G) * n2 * 8 + 32 * D * 4 +
                        (FULL ? static_cast<int64_t>(D) * (D + 1) : D) * 4 + D * 4 + 32 * 4 +
                        (FULL ? 16 * 32 * 4 : 0);
  return bytes <= 160 * 1024 ? static_cast<int>(bytes) : 0;
}

template <int D, int G, bool FULL>
cudaError_t run_rowwise_f32(const ssa_params& p, const void* Q, const float* mu, const float* sg,
                            int32_t* idx, float* scores, const LaunchCtx& c) {
  if (const int qs = qtile_smem_bytes<D, G, FULL>(p)) {   // runs of queries share each block's summary
    int n2 = 1;
    while (n2 < p.n_kv / p.block) n2 <<= 1;
    cudaError_t e = cudaFuncSetAttribute(route_qtile_f32_kernel<D, G, FULL>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, qs);
    if (e != cudaSuccess) return e;
    constexpr int QT = 32 / G;
    dim3 grid((p.n_q + QT - 1) / QT, p.h_kv, p.batch);
    route_qtile_f32_kernel<D, G, FULL><<<grid, 256, qs, c.stream>>>(
        static_cast<const float*>(Q), mu, sg, row_args(p, idx, scores), n2);
    note_launch();
    return cudaGetLastError();
  }
  const int smem = row_smem_bytes(p);
  cudaError_t e = cudaFuncSetAttribute(route_rowwise_f32_kernel<D, G, FULL>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(p.n_q, p.h_kv, p.batch);
  route_rowwise_f32_kernel<D, G, FULL><<<grid, 256, smem, c.stream>>>(
      static_cast<const float*>(Q), mu, sg, row_args(p, idx, scores));
  note_launch();
  return cudaGetLastError();
}

template <int D, bool FULL>
cudaError_t rowwise_f32_g(const ssa_params& p, const void* Q, const float* mu, const float* sg,
                          int32_t* idx, float* scores, const LaunchCtx& c) {
  switch (p.h_q / p.h_kv) {
    case 1: return run_rowwise_f32<D, 1, FULL>(p, Q, mu, sg, idx, scores, c);
    case 2: return run_rowwise_f32<D, 2, FULL>(p, Q, mu, sg, idx, scores, c);
    case 4: return run_rowwise_f32<D, 4, FULL>(p, Q, mu, sg, idx, scores, c);
    case 8: return run_rowwise_f32<D, 8, FULL>(p, Q, mu, sg, idx, scores, c);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

int route_tiled_smem_bytes(int d, int /*topk*/) {
  return d == 128 ? TiledCfg<256>::SMEM : TiledCfg<128>::SMEM;
}

cudaError_t launch_features(const ssa_params& p, const void* Q, void* F, const LaunchCtx& c) {
  if (p.d == 128) return features_g<128>(p, Q, F, c);
  if (p.d == 64) return features_g<64>(p, Q, F, c);
  return cudaErrorInvalidValue;
}

cudaError_t launch_route_tiled(const ssa_params& p, const CUtensorMap& tmF, const CUtensorMap& tmT,
                               int32_t* idx, float* scores, const LaunchCtx& c, const int32_t* unit_need,
                               const CUtensorMap* tmS, int n_snap) {
  const int ksel = p.topk <= 8 ? 8 : (p.topk <= 16 ? 16 : 32);
  if (rows_per_block(p) != 1) tmS = nullptr;   // seeds are whole-block rows
  if (p.d == 128) {
    if (ksel == 8) return run_tiled<256, 8>(p, tmF, tmT, tmS, n_snap, idx, scores, unit_need, c);
    if (ksel == 16) return run_tiled<256, 16>(p, tmF, tmT, tmS, n_snap, idx, scores, unit_need, c);
    return run_tiled<256, 32>(p, tmF, tmT, tmS, n_snap, idx, scores, unit_need, c);
  }
  if (p.d == 64) {
    if (ksel == 8) return run_tiled<128, 8>(p, tmF, tmT, tmS, n_snap, idx, scores, unit_need, c);
    if (ksel == 16) return run_tiled<128, 16>(p, tmF, tmT, tmS, n_snap, idx, scores, unit_need, c);
    return run_tiled<128, 32>(p, tmF, tmT, tmS, n_snap, idx, scores, unit_need, c);
  }
  return cudaErrorInvalidValue;
}

// ------------------------------------------------------------------ seeds

// Snapshots per (batch, kv-head) the prefix scan holds in shared memory
// (2 x 512 lists of 32 keys = 256 KB would not fit; 2 x 384 = 192 KB does):
// problems with more blocks route without seeds.
constexpr size_t kMaxSnap = 384;

size_t route_seed_bytes(const ssa_params& p) {
  if (rows_per_block(p) != 1 || p.dtype != SSA_BF16) return 0;
  const size_t bgs = static_cast<size_t>(p.batch) * p.h_kv;
  const size_t nb = static_cast<size_t>(p.n_kv / p.block);
  const size_t n_snap = nb / 32;
  if (n_snap == 0 || n_snap > kMaxSnap) return 0;
  auto ru = [](size_t x) { return (x + 255) & ~size_t(255); };
  const size_t rows = bgs * n_snap * kSeedRows;
  return ru(bgs * nb * 4) + ru(rows * 4) + ru(rows * 2 * p.d * 2);
}

RouteSeeds route_seed_layout(const ssa_params& p, void* base) {
  RouteSeeds s{};
  const size_t bgs = static_cast<size_t>(p.batch) * p.h_kv;
  const size_t nb = static_cast<size_t>(p.n_kv / p.block);
  s.n_snap = static_cast<int32_t>(nb / 32);
  auto ru = [](size_t x) { return (x + 255) & ~size_t(255); };
  uint8_t* b = static_cast<uint8_t*>(base);
  s.var = reinterpret_cast<float*>(b);
  s.blk = reinterpret_cast<int32_t*>(b + ru(bgs * nb * 4));
  s.tab = b + ru(bgs * nb * 4) + ru(bgs * s.n_snap * kSeedRows * 4);
  return s;
}

namespace {

// Warp per routing row: the sum of its variance half (any order: the seeds
// only need some blocks, and every choice of them gives a valid bound).
template <int D>
__global__ void __launch_bounds__(256) seed_var_kernel(const __nv_bfloat16* __restrict__ T, float* __restrict__ var,
                                                       int64_t rows) {
  const int64_t row = (static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x) >> 5;
  if (row >= rows) return;   // warp-uniform
  const int lane = threadIdx.x & 31;
  const __nv_bfloat16* v = T + row * (2 * D) + D;
  float acc = 0.f;
#pragma unroll
  for (int t = lane; t < D; t += 32) acc += __bfloat162float(v[t]);
#pragma unroll
  for (int o = 16; o; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
  if (lane == 0) var[row] = acc;
}

// Lane l of the warp ends with the l-th largest of the warp's 32 keys.
__device__ __forceinline__ uint64_t warp_sort_desc(uint64_t key) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      const uint64_t other = __shfl_xor_sync(0xFFFFFFFFu, key, stride);
      const bool desc = (lane & size) == 0 || size == 32;
      const bool low = (lane & stride) == 0;
      key = (low == desc) ? (key > other ? key : other) : (key < other ? key : other);
    }
  }
  return key;
}

// CTA per (batch, kv-head): every 32-block batch's keys (variance desc,
// then block asc) sorted by one warp, then a Hillis-Steele prefix scan over
// the batches of each residue class mod 4, each step keeping the larger 32
// of two sorted lists (an associative merge): list s ends as the 32 best
// keys of batches s, s-4, s-8, ...  Snapshot s (blocks 0 .. 32 (s+1) - 1)
// takes lists s, s-1, s-2, s-3 — four disjoint sets of blocks — as its 128
// seeds, ordered so that every group of 4 consecutive seeds holds one of the
// 32 largest variance sums (below).  Two shared buffers of n_snap lists of
// 32 keys (n_snap <= kMaxSnap).
__device__ __forceinline__ uint64_t merge_top32(uint64_t a, uint64_t b_desc) {
  // a, b: descending runs held one element per lane; the larger 32 of the
  // 64 form a bitonic sequence a[l] max b[31 - l], sorted once more
  const int lane = threadIdx.x & 31;
  const uint64_t rev = __shfl_sync(0xFFFFFFFFu, b_desc, 31 - lane);
  return warp_sort_desc(a > rev ? a : rev);
}

__global__ void __launch_bounds__(1024) seed_prefix_kernel(const float* __restrict__ var, int32_t* __restrict__ blk,
                                                           int nb, int n_snap) {
  extern __shared__ uint64_t lists[];   // [2][n_snap][32]
  const int bg = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  uint64_t* cur = lists;
  uint64_t* nxt = lists + n_snap * 32;
  for (int s = warp; s < n_snap; s += nw) {
    const int c = s * 32 + lane;
    cur[s * 32 + lane] = warp_sort_desc(
        make_key(__float_as_uint(var[static_cast<int64_t>(bg) * nb + c]), static_cast<uint32_t>(c)));
  }
  __syncthreads();
  for (int off = 4; off < n_snap; off <<= 1) {
    for (int s = warp; s < n_snap; s += nw) {
      const uint64_t mine = cur[s * 32 + lane];
      nxt[s * 32 + lane] = s >= off ? merge_top32(mine, cur[(s - off) * 32 + lane]) : mine;
    }
    __syncthreads();
    uint64_t* t = cur; cur = nxt; nxt = t;
  }
  // snapshot s: the nl = min(4, s + 1) lists s, s-1, .. ranked together by
  // key (the keys are distinct); seed column 4 j + t holds rank j + 32 t, or
  // rank j again when that rank does not exist, so group j of 4 consecutive
  // columns holds rank j, one of the 32 largest variances
  for (int s = warp; s < n_snap; s += nw) {
    const int nl = s + 1 < 4 ? s + 1 : 4;
    int32_t* out = blk + (static_cast<int64_t>(bg) * n_snap + s) * kSeedRows;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      if (r >= nl) break;   // warp-uniform
      const uint64_t key = cur[(s - r) * 32 + lane];
      int rank = lane;
      for (int q = 0; q < nl; ++q) {
        if (q == r) continue;
        const uint64_t* L = cur + (s - q) * 32;   // descending: count the keys above `key`
        int lo = 0, hi = 32;
        while (lo < hi) {
          const int mid = (lo + hi) >> 1;
          if (L[mid] > key) lo = mid + 1; else hi = mid;
        }
        rank += lo;
      }
      const int32_t b = static_cast<int32_t>(key_block(key));
      out[(rank & 31) * 4 + (rank >> 5)] = b;
      if (rank < 32)
        for (int t = nl; t < 4; ++t) out[rank * 4 + t] = b;
    }
  }
}

// Warp per seed row: copies the routing row of its block.
template <int D>
__global__ void __launch_bounds__(256) seed_gather_kernel(const __nv_bfloat16* __restrict__ T,
                                                          const int32_t* __restrict__ blk,
                                                          __nv_bfloat16* __restrict__ tab, int64_t rows, int nb,
                                                          int per_bg) {
  const int64_t r = (static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x) >> 5;
  if (r >= rows) return;   // warp-uniform
  const int lane = threadIdx.x & 31;
  const int64_t bg = r / per_bg;
  const int c = blk[r];
  constexpr int PER = 2 * D / 32;   // bf16 values per lane
  const __nv_bfloat16* src = T + (bg * nb + c) * (2 * D) + lane * PER;
  __nv_bfloat16* dst = tab + r * (2 * D) + lane * PER;
  if constexpr (PER == 8)
    *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
  else
    *reinterpret_cast<uint2*>(dst) = *reinterpret_cast<const uint2*>(src);
}

}  // namespace

cudaError_t launch_route_seeds(const ssa_params& p, const void* table, const RouteSeeds& s, const LaunchCtx& c) {
  const int bgs = p.batch * p.h_kv;
  const int nb = p.n_kv / p.block;
  const __nv_bfloat16* T = static_cast<const __nv_bfloat16*>(table);
  const int64_t rows = static_cast<int64_t>(bgs) * nb;
  const unsigned g1 = static_cast<unsigned>((rows * 32 + 255) / 256);
  if (p.d == 128) seed_var_kernel<128><<<g1, 256, 0, c.stream>>>(T, s.var, rows);
  else seed_var_kernel<64><<<g1, 256, 0, c.stream>>>(T, s.var, rows);
  note_launch();
  const int psmem = 2 * s.n_snap * 32 * static_cast<int>(sizeof(uint64_t));
  cudaError_t e = cudaFuncSetAttribute(seed_prefix_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, psmem);
  if (e != cudaSuccess) return e;
  seed_prefix_kernel<<<static_cast<unsigned>(bgs), 1024, psmem, c.stream>>>(s.var, s.blk, nb, s.n_snap);
  note_launch();
  const int64_t srows = static_cast<int64_t>(bgs) * s.n_snap * kSeedRows;
  const unsigned g3 = static_cast<unsigned>((srows * 32 + 255) / 256);
  __nv_bfloat16* tab = static_cast<__nv_bfloat16*>(s.tab);
  if (p.d == 128) seed_gather_kernel<128><<<g3, 256, 0, c.stream>>>(T, s.blk, tab, srows, nb, s.n_snap * kSeedRows);
  else seed_gather_kernel<64><<<g3, 256, 0, c.stream>>>(T, s.blk, tab, srows, nb, s.n_snap * kSeedRows);
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_route_rowwise_bf16(const ssa_params& p, const void* Q, const void* table,
                                      int32_t* idx, float* scores, const LaunchCtx& c, const uint8_t* skip) {
  if (p.d == 128) return rowwise_bf16_g<128>(p, Q, table, idx, scores, skip, c);
  if (p.d == 64) return rowwise_bf16_g<64>(p, Q, table, idx, scores, skip, c);
  return cudaErrorInvalidValue;
}

cudaError_t launch_route_rowwise_f32(const ssa_params& p, const void* Q, const float* mu,
                                     const float* sigma, int32_t* idx, float* scores,
                                     const LaunchCtx& c) {
  const bool full = p.sigma == SSA_SIGMA_FULL;
  if (p.d == 128) return full ? rowwise_f32_g<128, true>(p, Q, mu, sigma, idx, scores, c)
                              : rowwise_f32_g<128, false>(p, Q, mu, sigma, idx, scores, c);
  if (p.d == 64) return full ? rowwise_f32_g<64, true>(p, Q, mu, sigma, idx, scores, c)
                             : rowwise_f32_g<64, false>(p, Q, mu, sigma, idx, scores, c);
  return cudaErrorInvalidValue;
}

}  // namespace ssa

// Hierarchical routing: a tree level of nodes over the block summaries, a
// per-row probe of the best nodes, and the row's certificate.
//
// The page "Subquadratic Sparse Attention (SSA)" names a tree router with a
// recursive radius (artifact list, Barnes-Hut style), branch-and-bound exact
// selection under an admissible bound (same list) and per-query certificates
// with escalation ("Certified Causal Cascade" entry), without fixing their
// rules.  The rules built here:
//
//   node N = blocks N*M .. N*M+M-1 (complete nodes only), summarised from the
//   blocks' bf16 routing rows T_c = [mu_c ; s_c] by
//     centre m_N = bf16(f32(mean_c mu_c)),  cap v_N = max_c s_c (per dim),
//     radius R_N = max_c ||mu_c - m_N||_2   (float64, rounded up to float32);
//   for features f = [f_s ; f_q] with f_q >= 0 every block of N scores
//     f . T_c <= f . [m_N ; v_N] + ||f_s|| R_N.
//
// A row ranks its complete visible nodes by w_N = f . [m_N ; v_N] (the
// block router run over the node table, tensor-core tiles or one CTA per
// row, keeping the top probe+1 with their scores),
// scores the blocks of the best `probe` nodes and the visible blocks outside
// complete nodes exactly, and keeps their top-k.  It is certified when no
// complete visible node is left, or when the k-th kept score exceeds
// w_(probe+1) + ||f_s|| R* + 2^-12 ||f|| T* (R*: largest radius, T*: largest
// row 2-norm of the (batch, kv-head); the last term covers float32 rounding
// of both scores): every unexpanded block then scores below the kept set, so
// the kept set is the exact top-k.
//
// A second tree level groups M consecutive nodes into a super-node S with
//   centre m_S = bf16(f32(mean_N m_N)),  cap v_S = max_N v_N,
//   radius R_S = max_N (||m_N - m_S||_2 + R_N)   (the recursive radius: by
//   the triangle inequality every block mean of S lies within it of m_S),
// so f . T_c <= f . [m_S ; v_S] + ||f_s|| R_S for every block of S.  A row
// then ranks its complete visible super-nodes, ranks the nodes of the best
// `probe` (and the nodes outside complete super-nodes) by their exact node
// scores, and probes the best `probe` of those as above; it is certified
// when the k-th kept score also exceeds the best unexpanded super-node's
// w_S + ||f_s|| R2* + 2^-12 ||f|| T* (R2*: largest super-node radius).
#include <cuda_bf16.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace ssa {
namespace {

// Lane l holds elements [FPL*l, FPL*l + FPL) of a 2D-long routing row:
// lanes 0..15 the mean half, lanes 16..31 the variance half.
template <int FPL>
__device__ __forceinline__ void load_slice(const __nv_bfloat16* p, float (&v)[FPL]) {
  if constexpr (FPL == 8) {
    const uint4 raw = __ldg(reinterpret_cast<const uint4*>(p));
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[2 * j] = __uint_as_float(w[j] << 16);
      v[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
    }
  } else {
    const uint2 raw = __ldg(reinterpret_cast<const uint2*>(p));
    const uint32_t w[2] = {raw.x, raw.y};
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      v[2 * j] = __uint_as_float(w[j] << 16);
      v[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
    }
  }
}

// The raw bf16 pairs of a lane's slice (FPL / 2 words; the rest unused).
template <int FPL>
__device__ __forceinline__ uint4 load_raw(const __nv_bfloat16* p) {
  if constexpr (FPL == 8) {
    return __ldg(reinterpret_cast<const uint4*>(p));
  } else {
    const uint2 r = __ldg(reinterpret_cast<const uint2*>(p));
    return make_uint4(r.x, r.y, 0u, 0u);
  }
}

template <int FPL>
__device__ __forceinline__ float dot_raw(const float (&f)[FPL], uint4 raw, float acc) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int j = 0; j < FPL / 2; ++j) {
    acc = __fmaf_rn(f[2 * j], __uint_as_float(w[j] << 16), acc);
    acc = __fmaf_rn(f[2 * j + 1], __uint_as_float(w[j] & 0xFFFF0000u), acc);
  }
  return acc;
}

template <int FPL>
__device__ __forceinline__ void store_slice(__nv_bfloat16* p, const float (&v)[FPL]) {
  uint32_t w[FPL / 2];
#pragma unroll
  for (int j = 0; j < FPL / 2; ++j)
    w[j] = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(v[2 * j]))) |
           (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(v[2 * j + 1]))) << 16);
  if constexpr (FPL == 8)
    *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
  else
    *reinterpret_cast<uint2*>(p) = make_uint2(w[0], w[1]);
}

__device__ __forceinline__ double warp_sum_d(double x) {
#pragma unroll
  for (int o = 16; o; o >>= 1) x += __shfl_xor_sync(0xFFFFFFFFu, x, o);
  return x;
}

__device__ __forceinline__ float warp_sum_f(float x) {
#pragma unroll
  for (int o = 16; o; o >>= 1) x += __shfl_xor_sync(0xFFFFFFFFu, x, o);
  return x;
}

__device__ __forceinline__ uint64_t warp_min_u64(uint64_t x) {
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    const uint64_t y = __shfl_xor_sync(0xFFFFFFFFu, x, o);
    x = y < x ? y : x;
  }
  return x;
}

// ------------------------------------------------------------------ nodes

// One warp per (batch * kv-head, node); node index nn covers the trailing
// blocks that belong to no complete node (their row norms only).
template <int D>
__global__ void __launch_bounds__(256) hier_nodes_kernel(const HierNodeArgs a) {
  constexpr int FPL = 2 * D / 32;
  const int lane = threadIdx.x & 31;
  const int64_t w = static_cast<int64_t>(blockIdx.x) * 8 + threadIdx.x / 32;
  if (w >= static_cast<int64_t>(a.bgs) * (a.nn + 1)) return;
  const int bg = static_cast<int>(w / (a.nn + 1)), N = static_cast<int>(w % (a.nn + 1));
  const bool mean_half = lane < 16;
  const __nv_bfloat16* trow = a.T + static_cast<int64_t>(bg) * a.nb * (2 * D) + lane * FPL;
  const int c0 = N * a.M;
  const int c1 = N < a.nn ? c0 + a.M : a.nb;
  double sum[FPL];
  float cap[FPL];
#pragma unroll
  for (int e = 0; e < FPL; ++e) { sum[e] = 0.0; cap[e] = -INFINITY; }
  double row2max = 0.0;
#pragma unroll 4
  for (int c = c0; c < c1; ++c) {
    float v[FPL];
    load_slice<FPL>(trow + static_cast<int64_t>(c) * (2 * D), v);
    double r2 = 0.0;
#pragma unroll
    for (int e = 0; e < FPL; ++e) {
      r2 += static_cast<double>(v[e]) * v[e];
      sum[e] += v[e];
      cap[e] = fmaxf(cap[e], v[e]);
    }
    row2max = fmax(row2max, warp_sum_d(r2));
  }
  if (N < a.nn) {
    float m[FPL];
#pragma unroll
    for (int e = 0; e < FPL; ++e)   // sum / M is exact (M a power of two)
      m[e] = mean_half ? __bfloat162float(__float2bfloat16_rn(__double2float_rn(sum[e] / a.M))) : cap[e];
    store_slice<FPL>(a.NT + (static_cast<int64_t>(bg) * a.nn + N) * (2 * D) + lane * FPL, m);
    double n2 = 0.0;
#pragma unroll
    for (int e = 0; e < FPL; ++e) n2 += static_cast<double>(m[e]) * m[e];
    row2max = fmax(row2max, warp_sum_d(n2));
    double d2max = 0.0;
#pragma unroll 4
    for (int c = c0; c < c1; ++c) {
      float v[FPL];
      load_slice<FPL>(trow + static_cast<int64_t>(c) * (2 * D), v);
      double d2 = 0.0;
#pragma unroll
      for (int e = 0; e < FPL; ++e) {
        const double t = static_cast<double>(v[e]) - m[e];
        d2 += mean_half ? t * t : 0.0;
      }
      d2max = fmax(d2max, warp_sum_d(d2));
    }
    const float R = __double2float_ru(sqrt(d2max));
    if (lane == 0) {
      a.radius[static_cast<int64_t>(bg) * a.nn + N] = R;
      atomicMax(&a.bound[2 * bg], __float_as_uint(R));   // non-negative floats order as their bits
    }
  }
  if (lane == 0) atomicMax(&a.bound[2 * bg + 1], __float_as_uint(__double2float_ru(sqrt(row2max))));
}

// One warp per (batch * kv-head, super-node).
template <int D>
__global__ void __launch_bounds__(256) hier_supers_kernel(const HierSuperArgs a) {
  constexpr int FPL = 2 * D / 32;
  const int lane = threadIdx.x & 31;
  const int64_t w = static_cast<int64_t>(blockIdx.x) * 8 + threadIdx.x / 32;
  if (w >= static_cast<int64_t>(a.bgs) * a.ns) return;
  const int bg = static_cast<int>(w / a.ns), S = static_cast<int>(w % a.ns);
  const bool mean_half = lane < 16;
  const __nv_bfloat16* nrow = a.NT + static_cast<int64_t>(bg) * a.nn * (2 * D) + lane * FPL;
  const int n0 = S * a.M;
  double sum[FPL];
  float cap[FPL];
#pragma unroll
  for (int e = 0; e < FPL; ++e) { sum[e] = 0.0; cap[e] = -INFINITY; }
#pragma unroll 4
  for (int c = n0; c < n0 + a.M; ++c) {
    float v[FPL];
    load_slice<FPL>(nrow + static_cast<int64_t>(c) * (2 * D), v);
#pragma unroll
    for (int e = 0; e < FPL; ++e) {
      sum[e] += v[e];
      cap[e] = fmaxf(cap[e], v[e]);
    }
  }
  float m[FPL];
#pragma unroll
  for (int e = 0; e < FPL; ++e)   // sum / M is exact (M a power of two)
    m[e] = mean_half ? __bfloat162float(__float2bfloat16_rn(__double2float_rn(sum[e] / a.M))) : cap[e];
  store_slice<FPL>(a.ST + (static_cast<int64_t>(bg) * a.ns + S) * (2 * D) + lane * FPL, m);
  double n2 = 0.0;
#pragma unroll
  for (int e = 0; e < FPL; ++e) n2 += static_cast<double>(m[e]) * m[e];
  n2 = warp_sum_d(n2);
  double rmax = 0.0;
#pragma unroll 4
  for (int c = n0; c < n0 + a.M; ++c) {
    float v[FPL];
    load_slice<FPL>(nrow + static_cast<int64_t>(c) * (2 * D), v);
    double d2 = 0.0;
#pragma unroll
    for (int e = 0; e < FPL; ++e) {
      const double t = static_cast<double>(v[e]) - m[e];
      d2 += mean_half ? t * t : 0.0;
    }
    d2 = warp_sum_d(d2);
    rmax = fmax(rmax, sqrt(d2) + static_cast<double>(a.radius[static_cast<int64_t>(bg) * a.nn + c]));
  }
  const float R = __double2float_ru(rmax);
  if (lane == 0) {
    a.sradius[static_cast<int64_t>(bg) * a.ns + S] = R;
    atomicMax(&a.sbound[bg], __float_as_uint(R));   // non-negative floats order as their bits
    atomicMax(&a.bound[2 * bg + 1], __float_as_uint(__double2float_ru(sqrt(n2))));
  }
}

// ------------------------------------------------------------------ probe

constexpr int kProbeMaxCand = 512;   // (probe + 1) * M
constexpr int kProbeWarps = 8;

// Exact scores f . R_c of a row's n_cand candidate rows of a [rows, 2D]
// table (tb points at row 0, this lane's slice), as keys (score, row) in
// keys[0 .. n_cand): candidate t < nexpc is child t % M of the entry
// my_exp holds in lane t / M (the expanded entries, ascending); the rest are
// the consecutive rows tail0 ...  32 at a time: lane u accumulates its slice
// of candidate t0+u, then a transposing butterfly leaves the whole score of
// candidate t0+l in lane l.
template <int FPL>
__device__ __forceinline__ void score_candidates(const float (&f)[FPL], const __nv_bfloat16* tb, int my_exp,
                                                 int log2M, int nexpc, int tail0, int n_cand, uint64_t* keys) {
  const int lane = threadIdx.x & 31;
  const int Mm1 = (1 << log2M) - 1;
  for (int t0 = 0; t0 < n_cand; t0 += 32) {
    float acc[32];
#pragma unroll
    for (int u0 = 0; u0 < 32; u0 += 8) {
      // eight independent row loads in flight; past the last candidate a
      // lane reads row 0 and the score is discarded
      uint4 raw[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int t = t0 + u0 + u;
        const int e = __shfl_sync(0xFFFFFFFFu, my_exp, min(t >> log2M, 31));
        int c = t < nexpc ? (e << log2M) + (t & Mm1) : tail0 + (t - nexpc);
        c = t < n_cand ? c : 0;
        raw[u] = load_raw<FPL>(tb + static_cast<int64_t>(c) * (FPL * 32));
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) acc[u0 + u] = dot_raw<FPL>(f, raw[u], 0.f);
    }
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      const bool up = (lane & o) != 0;
#pragma unroll
      for (int u = 0; u < o; ++u) {
        const float send = up ? acc[u] : acc[u + o];
        const float keep = up ? acc[u + o] : acc[u];
        acc[u] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, o);
      }
    }
    const int t = t0 + lane;
    const int e = __shfl_sync(0xFFFFFFFFu, my_exp, min(t >> log2M, 31));
    if (t < n_cand) {
      const int c = t < nexpc ? (e << log2M) + (t & Mm1) : tail0 + (t - nexpc);
      keys[t] = make_key(__float_as_uint(acc[0]), static_cast<uint32_t>(c));
    }
  }
  __syncwarp();
}

// The best kcount (<= 32) of keys[0 .. n_cand) under (score desc, index
// asc): k rounds of a warp arg-max, the score half and the index half of
// the key each by one warp reduction (keys are unique: one row each); a
// lane keeps its best key cached.  Lane j < the returned count gets the
// j-th best in `kept`.  Consumes keys.
__device__ __forceinline__ int warp_top_keys(uint64_t* keys, int n_cand, int kcount, uint64_t& kept) {
  const int lane = threadIdx.x & 31;
  int nkept = 0;
  uint64_t m = 0;
  int at = -1;
  for (int t = lane; t < n_cand; t += 32) {
    const uint64_t x = keys[t];
    if (x > m) { m = x; at = t; }
  }
  for (int j = 0; j < kcount; ++j) {
    const uint32_t hi = static_cast<uint32_t>(m >> 32);
    const uint32_t top = __reduce_max_sync(0xFFFFFFFFu, hi);
    if (top == 0) break;   // no candidates left
    const uint32_t lo = __reduce_max_sync(0xFFFFFFFFu, hi == top ? static_cast<uint32_t>(m) : 0u);
    const uint64_t best = (static_cast<uint64_t>(top) << 32) | lo;
    if (lane == j) kept = best;
    ++nkept;
    if (m == best) {   // the owner drops it and rescans its candidates
      keys[at] = 0;
      m = 0;
      at = -1;
      for (int t = lane; t < n_cand; t += 32) {
        const uint64_t x = keys[t];
        if (x > m) { m = x; at = t; }
      }
    }
    __syncwarp();
  }
  return nkept;
}

// From a list of the probe+1 best entries (lane l < probe+1: index and
// score, ascending index, -1 padded) of the nv candidate entries of a level
// (indices below `range`): whether every candidate is expanded (nv <= probe), the
// entries to expand (all listed ones, or all but the last under (score
// desc, index asc), whose score is then the best unexpanded score w_next)
// in lanes 0 .. nexp-1 of my_exp, ascending; list_ok when the list holds
// the expected number of valid entries.
struct Expansion {
  bool complete, list_ok;
  float w_next;
  int nexp, my_exp;
};

__device__ __forceinline__ Expansion expand_list(int idx, float score, int range, int nv, int probe) {
  const int lane = threadIdx.x & 31;
  Expansion x;
  x.complete = nv <= probe;
  const bool valid = idx >= 0 && idx < range;
  const int nvalid = __popc(__ballot_sync(0xFFFFFFFFu, valid));
  x.list_ok = x.complete ? nvalid == nv : nvalid == probe + 1;
  const uint64_t k = valid ? make_key(__float_as_uint(score), idx) : ~0ull;
  const uint64_t kmin = warp_min_u64(k);
  const int excl = x.complete ? -1 : static_cast<int>(key_block(kmin));
  x.w_next = x.complete ? -INFINITY : key_score(kmin);
  const bool expd = valid && idx != excl;
  const uint32_t emask = __ballot_sync(0xFFFFFFFFu, expd);
  x.nexp = __popc(emask);
  uint32_t m = emask;
  for (int t = 0; t < lane && m; ++t) m &= m - 1u;   // drop the j lowest set bits
  const int src = (lane < x.nexp && m) ? __ffs(static_cast<int>(m)) - 1 : 0;
  x.my_exp = __shfl_sync(0xFFFFFFFFu, idx, src);
  return x;
}

// One warp per (batch * kv-head, query row).
template <int D>
__global__ void __launch_bounds__(256) hier_probe_kernel(const HierProbeArgs a) {
  constexpr int FPL = 2 * D / 32;
  __shared__ uint64_t keys_all[kProbeWarps][kProbeMaxCand];
  const int lane = threadIdx.x & 31;
  uint64_t* keys = keys_all[threadIdx.x / 32];
  const int64_t w = static_cast<int64_t>(blockIdx.x) * kProbeWarps + threadIdx.x / 32;
  if (w >= static_cast<int64_t>(a.bgs) * a.n_q) return;
  const int bg = static_cast<int>(w / a.n_q), i = static_cast<int>(w % a.n_q);
  const int b = bg / a.h_kv, g = bg % a.h_kv;
  // key positions fit 31 bits and B, M are powers of two: shifts
  const int pos1 = static_cast<int>(a.q_offset) + i + 1;
  const int lbb = __ffs(a.block) - 1;
  const int nv = min(a.nb, pos1 >> lbb);
  const int nvn = min(a.nn, pos1 >> (lbb + __ffs(a.M) - 1));
  const int64_t row = (static_cast<int64_t>(b) * a.n_q + i) * a.h_kv + g;

  float f[FPL];
  load_slice<FPL>(a.F + (static_cast<int64_t>(bg) * a.n_q + i) * (2 * D) + lane * FPL, f);
  float f2 = 0.f;
#pragma unroll
  for (int e = 0; e < FPL; ++e) f2 = __fmaf_rn(f[e], f[e], f2);
  const float fs2 = warp_sum_f(lane < 16 ? f2 : 0.f);
  f2 = warp_sum_f(f2);

  // the row's candidate nodes (every complete visible node, or with two
  // levels those of its expanded super-nodes and outside complete ones) and
  // the probe+1 best of them (ascending node index, -1 padded); when the
  // list is full its last entry under (score desc, index asc) stays
  // unexpanded and bounds every unexpanded candidate
  const int P1 = a.probe + 1;
  const int ncn = a.n_cand ? a.n_cand[row] : nvn;
  int nidx = -1;
  float nsc = -INFINITY;
  if (ncn > 0 && lane < P1) {
    nidx = a.node_idx[row * P1 + lane];
    nsc = a.node_score[row * P1 + lane];
  }
  const Expansion x = expand_list(nidx, nsc, nvn, ncn, a.probe);
  const bool complete = x.complete, list_ok = x.list_ok;
  const float w_next = x.w_next;
  const int nexp = x.nexp, my_exp = x.my_exp;
  const int log2M = __ffs(a.M) - 1;
  const int nexpb = nexp << log2M;
  const int n_cand = nexpb + (nv - nvn * a.M);

  score_candidates<FPL>(f, a.T + static_cast<int64_t>(bg) * a.nb * (2 * D) + lane * FPL, my_exp, log2M, nexpb,
                        nvn * a.M, n_cand, keys);
  uint64_t kept = 0;
  const int nkept = warp_top_keys(keys, n_cand, a.topk, kept);
  const uint64_t kth = __shfl_sync(0xFFFFFFFFu, kept, max(a.topk - 1, 0));
  const float tau = nkept == a.topk ? key_score(kth) : -INFINITY;
  const float margin = 0x1p-12f * sqrtf(f2) * a.bound[2 * bg + 1];
  const float bound = w_next + sqrtf(fs2) * a.bound[2 * bg] + margin;
  // two levels: the best unexpanded super-node bounds the blocks of all
  // unexpanded super-nodes (+inf when the first probe's list was short)
  const float w2 = a.w2_next ? a.w2_next[row] : -INFINITY;
  const bool ok2 = !(w2 > -INFINITY) || tau > w2 + sqrtf(fs2) * a.sbound[bg] + margin;
  const bool certified = list_ok && (complete || tau > bound) && ok2;

  // kept blocks in ascending order, -1 padded
  const uint32_t blk = (lane < nkept) ? key_block(kept) : 0xFFFFFFFFu;
  int rank = 0;
#pragma unroll 8
  for (int o = 0; o < 32; ++o) rank += (__shfl_sync(0xFFFFFFFFu, blk, o) < blk) ? 1 : 0;
  if (lane < a.topk) {
    int32_t* out = a.block_idx + row * a.topk;
    if (lane < nkept)
      out[rank] = static_cast<int32_t>(blk);
    else
      out[lane] = -1;
  }
  if (lane == 0) {
    if (a.cert) a.cert[row] = certified ? 1 : 0;
    if (!certified && a.unit_need) a.unit_need[static_cast<int64_t>(bg) * a.n_tiles + i / 256] = 1;
  }
}

// Two levels, first probe: one warp per (batch * kv-head, query row).
template <int D>
__global__ void __launch_bounds__(256) hier_probe2_kernel(const HierProbe2Args a) {
  constexpr int FPL = 2 * D / 32;
  __shared__ uint64_t keys_all[kProbeWarps][kProbeMaxCand];
  const int lane = threadIdx.x & 31;
  uint64_t* keys = keys_all[threadIdx.x / 32];
  const int64_t w = static_cast<int64_t>(blockIdx.x) * kProbeWarps + threadIdx.x / 32;
  if (w >= static_cast<int64_t>(a.bgs) * a.n_q) return;
  const int bg = static_cast<int>(w / a.n_q), i = static_cast<int>(w % a.n_q);
  const int b = bg / a.h_kv, g = bg % a.h_kv;
  // key positions fit 31 bits and B, M are powers of two: shifts
  const int pos1 = static_cast<int>(a.q_offset) + i + 1;
  const int lbb = __ffs(a.block) - 1, log2M = __ffs(a.M) - 1;
  const int nvn = min(a.nn, pos1 >> (lbb + log2M));
  const int nvs = min(a.ns, pos1 >> (lbb + 2 * log2M));
  const int64_t row = (static_cast<int64_t>(b) * a.n_q + i) * a.h_kv + g;
  float f[FPL];
  load_slice<FPL>(a.F + (static_cast<int64_t>(bg) * a.n_q + i) * (2 * D) + lane * FPL, f);

  // the super-node router's probe+1 best (ascending, -1 padded)
  const int P1 = a.probe + 1;
  int sidx = -1;
  float ssc = -INFINITY;
  if (a.sup_idx && nvs > 0 && lane < P1) {
    sidx = a.sup_idx[row * P1 + lane];
    ssc = a.sup_score[row * P1 + lane];
  }
  const Expansion x = expand_list(sidx, ssc, nvs, nvs, a.probe);
  // candidate nodes: the children of the expanded super-nodes, then the
  // complete visible nodes outside complete visible super-nodes
  const int nexpc = x.nexp << log2M;
  const int n_cand = nexpc + (nvn - nvs * a.M);
  score_candidates<FPL>(f, a.NT + static_cast<int64_t>(bg) * a.nn * (2 * D) + lane * FPL, x.my_exp, log2M, nexpc,
                        nvs * a.M, n_cand, keys);
  uint64_t kept = 0;
  const int nkept = warp_top_keys(keys, n_cand, P1, kept);
  // the kept nodes in ascending order with their scores, -1 padded
  const uint32_t nd = (lane < nkept) ? key_block(kept) : 0xFFFFFFFFu;
  int rank = 0;
#pragma unroll 8
  for (int o = 0; o < 32; ++o) rank += (__shfl_sync(0xFFFFFFFFu, nd, o) < nd) ? 1 : 0;
  if (lane < P1) {
    if (lane < nkept) {
      a.node_idx[row * P1 + rank] = static_cast<int32_t>(nd);
      a.node_score[row * P1 + rank] = key_score(kept);
    } else {
      a.node_idx[row * P1 + lane] = -1;
      a.node_score[row * P1 + lane] = -INFINITY;
    }
  }
  if (lane == 0) {
    a.n_cand[row] = n_cand;
    // a short super-node list certifies nothing
    a.w2_next[row] = x.list_ok ? x.w_next : INFINITY;
  }
}

}  // namespace

cudaError_t launch_hier_nodes(const ssa_params& p, const HierNodeArgs& a, const LaunchCtx& c) {
  const int64_t warps = static_cast<int64_t>(a.bgs) * (a.nn + 1);
  const int64_t grid = (warps + 7) / 8;
  if (grid == 0) return cudaSuccess;
  if (grid > 2147483647) return cudaErrorInvalidValue;
  if (p.d == 128)
    hier_nodes_kernel<128><<<static_cast<unsigned>(grid), 256, 0, c.stream>>>(a);
  else if (p.d == 64)
    hier_nodes_kernel<64><<<static_cast<unsigned>(grid), 256, 0, c.stream>>>(a);
  else
    return cudaErrorInvalidValue;
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_hier_probe(const ssa_params& p, const HierProbeArgs& a, const LaunchCtx& c) {
  const int64_t warps = static_cast<int64_t>(a.bgs) * a.n_q;
  const int64_t grid = (warps + kProbeWarps - 1) / kProbeWarps;
  if (grid == 0) return cudaSuccess;
  if (grid > 2147483647) return cudaErrorInvalidValue;
  if ((a.probe + 1) * a.M > kProbeMaxCand || a.topk > 32 || a.probe + 1 > 32) return cudaErrorInvalidValue;
  if (p.d == 128)
    hier_probe_kernel<128><<<static_cast<unsigned>(grid), kProbeWarps * 32, 0, c.stream>>>(a);
  else if (p.d == 64)
    hier_probe_kernel<64><<<static_cast<unsigned>(grid), kProbeWarps * 32, 0, c.stream>>>(a);
  else
    return cudaErrorInvalidValue;
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_hier_supers(const ssa_params& p, const HierSuperArgs& a, const LaunchCtx& c) {
  const int64_t warps = static_cast<int64_t>(a.bgs) * a.ns;
  const int64_t grid = (warps + 7) / 8;
  if (grid == 0) return cudaSuccess;
  if (grid > 2147483647) return cudaErrorInvalidValue;
  if (p.d == 128)
    hier_supers_kernel<128><<<static_cast<unsigned>(grid), 256, 0, c.stream>>>(a);
  else if (p.d == 64)
    hier_supers_kernel<64><<<static_cast<unsigned>(grid), 256, 0, c.stream>>>(a);
  else
    return cudaErrorInvalidValue;
  note_launch();
  return cudaGetLastError();
}

cudaError_t launch_hier_probe2(const ssa_params& p, const HierProbe2Args& a, const LaunchCtx& c) {
  const int64_t warps = static_cast<int64_t>(a.bgs) * a.n_q;
  const int64_t grid = (warps + kProbeWarps - 1) / kProbeWarps;
  if (grid == 0) return cudaSuccess;
  if (grid > 2147483647) return cudaErrorInvalidValue;
  if ((a.probe + 1) * a.M > kProbeMaxCand || a.probe + 1 > 32) return cudaErrorInvalidValue;
  if (p.d == 128)
    hier_probe2_kernel<128><<<static_cast<unsigned>(grid), kProbeWarps * 32, 0, c.stream>>>(a);
  else if (p.d == 64)
    hier_probe2_kernel<64><<<static_cast<unsigned>(grid), kProbeWarps * 32, 0, c.stream>>>(a);
  else
    return cudaErrorInvalidValue;
  note_launch();
  return cudaGetLastError();
}

}  // namespace ssa

// Step (i) of the layer: per-block key summaries (and the outlier channel's
// rows).
//
// "routes ... using only per-block summary statistics"
// [Subquadratic Sparse Attention (SSA), opening section]; the routing score
// needs the block mean mu_c and the covariance Sigma_c of the block's keys
// ["The idea in one screen", routing-score equation].  Normalisation is by
// the number of keys summarised (population moments).
//
// A unit is a block of B keys, or a sub-block of B / S keys when each block
// is summarised S times.  bf16 keys: one warp per (batch, kv-head, unit),
// lane l owning dimensions d/32 l .. d/32 (l+1) - 1, one pass over the rows
// with float64 sums.  float32 keys: one CTA per unit, the mean and then the
// centred second moments reduced in float64.  Every partial sum of the mean
// is exact in float64, so mu is the exact block mean and its float32 /
// bfloat16 roundings are reproducible bit for bit.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.h"

namespace ssa {
namespace {

template <typename T>
__device__ __forceinline__ void load_vec(const T* p, float (&x)[16 / sizeof(T)]);

template <>
__device__ __forceinline__ void load_vec<float>(const float* p, float (&x)[4]) {
  const float4 v = __ldg(reinterpret_cast<const float4*>(p));
  x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
}

template <>
__device__ __forceinline__ void load_vec<__nv_bfloat16>(const __nv_bfloat16* p, float (&x)[8]) {
  const uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// Diagonal summaries.  Thread (rg, cg) owns VEC consecutive dimensions of
// rows rg, rg + RG, rg + 2 RG, ...
template <typename T, int D, int BLK>
__global__ void __launch_bounds__(256) summary_diag_kernel(const T* __restrict__ K,
                                                           float* __restrict__ mu,
                                                           float* __restrict__ sig,
                                                           __nv_bfloat16* __restrict__ table,
                                                           int n_kv, int h_kv, int nb, int rstride) {
  constexpr int VEC = 16 / sizeof(T);
  constexpr int CG = D / VEC;
  constexpr int RG = 256 / CG;
  constexpr int RPT = BLK / RG;
  static_assert(RPT * RG == BLK, "block must be a multiple of the row groups");
  __shared__ double red[RG][D];
  __shared__ double mean_s[D];

  const int c = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int cg = threadIdx.x % CG, rg = threadIdx.x / CG;
  const int64_t row_stride = static_cast<int64_t>(h_kv) * D;
  const T* base = K + ((static_cast<int64_t>(b) * n_kv + static_cast<int64_t>(c) * BLK) * h_kv + g) * D +
                  cg * VEC;

  float x[RPT][VEC];
#pragma unroll
  for (int t = 0; t < RPT; ++t) load_vec<T>(base + (rg + t * RG) * row_stride, x[t]);

#pragma unroll
  for (int v = 0; v < VEC; ++v) {
    double s = 0.0;
#pragma unroll
    for (int t = 0; t < RPT; ++t) s += static_cast<double>(x[t][v]);
    red[rg][cg * VEC + v] = s;
  }
  __syncthreads();
  if (threadIdx.x < D) {
    double s = 0.0;
#pragma unroll 4
    for (int r = 0; r < RG; ++r) s += red[r][threadIdx.x];
    mean_s[threadIdx.x] = s / BLK;
  }
  __syncthreads();
#pragma unroll
  for (int v = 0; v < VEC; ++v) {
    const double m = mean_s[cg * VEC + v];
    double s = 0.0;
#pragma unroll
    for (int t = 0; t < RPT; ++t) {
      const double e = static_cast<double>(x[t][v]) - m;
      s = fma(e, e, s);
    }
    red[rg][cg * VEC + v] = s;
  }
  __syncthreads();
  if (threadIdx.x < D) {
    double s = 0.0;
#pragma unroll 4
    for (int r = 0; r < RG; ++r) s += red[r][threadIdx.x];
    const float m32 = __double2float_rn(mean_s[threadIdx.x]);
    const float v32 = __double2float_rn(s / BLK);
    const int64_t row = ((static_cast<int64_t>(b) * h_kv + g) * nb + c) * rstride;
    if (mu) mu[row * D + threadIdx.x] = m32;
    if (sig) sig[row * D + threadIdx.x] = v32;
    if (table) {
      table[row * 2 * D + threadIdx.x] = __float2bfloat16_rn(m32);
      table[row * 2 * D + D + threadIdx.x] = __float2bfloat16_rn(v32);
    }
  }
}

// bf16 diagonal summaries, a warp per unit.  The variance comes from sums
// of the keys shifted by the unit's first key, sum (x - x0) and
// sum (x - x0)^2: for bf16 keys each shifted value and its square are exact
// in float64 and so are their sums over a unit, so the one-pass formula
// (sum (x-x0)^2 - (sum (x-x0))^2 / n) / n differs from the centred two-pass
// sum only in the final float64 roundings.
template <int D, int BLK>
__global__ void __launch_bounds__(256) summary_bf16_warp_kernel(const __nv_bfloat16* __restrict__ K,
                                                                 float* __restrict__ mu, float* __restrict__ sig,
                                                                 __nv_bfloat16* __restrict__ table, int n_kv,
                                                                 int h_kv, int nu, int64_t units, int rstride) {
  constexpr int VPL = D / 32;   // dimensions per lane: 4 (d = 128) or 2 (d = 64)
  constexpr int UNROLL = 16;    // rows loaded before they are summed
  static_assert(BLK % UNROLL == 0, "unit size");
  const int lane = threadIdx.x & 31;
  int64_t x = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);   // unit
  if (x >= units) return;   // warp-uniform
  const int c = static_cast<int>(x % nu);
  const int64_t bg = x / nu;
  const int g = static_cast<int>(bg % h_kv), b = static_cast<int>(bg / h_kv);
  const int64_t row_stride = static_cast<int64_t>(h_kv) * D;
  const __nv_bfloat16* base = K + ((static_cast<int64_t>(b) * n_kv + static_cast<int64_t>(c) * BLK) * h_kv + g) * D +
                              lane * VPL;
  auto load = [&](int r, float (&v)[VPL]) {
    if (VPL == 4) {
      const uint2 w = __ldg(reinterpret_cast<const uint2*>(base + r * row_stride));
      v[0] = __uint_as_float(w.x << 16); v[1] = __uint_as_float(w.x & 0xFFFF0000u);
      v[2] = __uint_as_float(w.y << 16); v[3] = __uint_as_float(w.y & 0xFFFF0000u);
    } else {
      const uint32_t w = __ldg(reinterpret_cast<const uint32_t*>(base + r * row_stride));
      v[0] = __uint_as_float(w << 16); v[1] = __uint_as_float(w & 0xFFFF0000u);
    }
  };
  float x0[VPL];
  load(0, x0);
  double s0[VPL], s1[VPL], s2[VPL];   // sum x, sum (x - x0), sum (x - x0)^2
#pragma unroll
  for (int v = 0; v < VPL; ++v) { s0[v] = 0.0; s1[v] = 0.0; s2[v] = 0.0; }
#pragma unroll 1
  for (int r0 = 0; r0 < BLK; r0 += UNROLL) {
    float xv[UNROLL][VPL];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) load(r0 + u, xv[u]);
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
#pragma unroll
      for (int v = 0; v < VPL; ++v) {
        const double xd = static_cast<double>(xv[u][v]);
        const double t = xd - static_cast<double>(x0[v]);
        s0[v] += xd;
        s1[v] += t;
        s2[v] = fma(t, t, s2[v]);
      }
    }
  }
  float m32[VPL], v32[VPL];
#pragma unroll
  for (int v = 0; v < VPL; ++v) {
    m32[v] = __double2float_rn(s0[v] / BLK);
    v32[v] = __double2float_rn((s2[v] - s1[v] * s1[v] / BLK) / BLK);
  }
  const int64_t x_in = x;
  x = x_in * rstride;   // output row
  if (mu) {
#pragma unroll
    for (int v = 0; v < VPL; ++v) mu[x * D + lane * VPL + v] = m32[v];
  }
  if (sig) {
#pragma unroll
    for (int v = 0; v < VPL; ++v) sig[x * D + lane * VPL + v] = v32[v];
  }
  if (table) {
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
      table[x * 2 * D + lane * VPL + v] = __float2bfloat16_rn(m32[v]);
      table[x * 2 * D + D + lane * VPL + v] = __float2bfloat16_rn(v32[v]);
    }
  }
}

// Full covariance (float32 problems).  The block is staged centred in
// shared memory as float64; thread e computes entries e, e+256, ...
template <int D, int BLK>
__global__ void __launch_bounds__(256) summary_full_kernel(const float* __restrict__ K,
                                                           float* __restrict__ mu,
                                                           float* __restrict__ sig,
                                                           int n_kv, int h_kv, int nb, int rstride) {
  extern __shared__ double xs[];   // [BLK][D]
  __shared__ double mean_s[D];
  const int c = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int64_t row_stride = static_cast<int64_t>(h_kv) * D;
  const float* base = K + ((static_cast<int64_t>(b) * n_kv + static_cast<int64_t>(c) * BLK) * h_kv + g) * D;
  for (int e = threadIdx.x; e < BLK * D; e += 256) {
    const int r = e / D, t = e % D;
    xs[e] = static_cast<double>(__ldg(base + r * row_stride + t));
  }
  __syncthreads();
  if (threadIdx.x < D) {
    double s = 0.0;
    for (int r = 0; r < BLK; ++r) s += xs[r * D + threadIdx.x];
    mean_s[threadIdx.x] = s / BLK;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < BLK * D; e += 256) xs[e] -= mean_s[e % D];
  __syncthreads();
  const int64_t row = ((static_cast<int64_t>(b) * h_kv + g) * nb + c) * rstride;
  if (mu && threadIdx.x < D) mu[row * D + threadIdx.x] = __double2float_rn(mean_s[threadIdx.x]);
  if (sig) {
    for (int e = threadIdx.x; e < D * D; e += 256) {
      const int s_ = e / D, t = e % D;
      double acc = 0.0;
      for (int r = 0; r < BLK; ++r) acc = fma(xs[r * D + s_], xs[r * D + t], acc);
      sig[row * D * D + e] = __double2float_rn(acc / BLK);
    }
  }
}

// Outlier rows, a warp per (batch, kv-head, block): the block's key of
// largest 2-norm — squared norms summed in float64 (exact for bf16 keys;
// float32 keys' squares are exact too), equal norms to the earlier key —
// written as summary row 2c + 1: mu = the key, sigma = 0 (d values, or the
// d x d zero matrix), route table [bf16(key) ; 0].
template <typename T, int D>
__global__ void __launch_bounds__(256) outlier_kernel(const T* __restrict__ K, float* __restrict__ mu,
                                                      float* __restrict__ sig, __nv_bfloat16* __restrict__ table,
                                                      int n_kv, int h_kv, int nb, int B, int full, int64_t units) {
  constexpr int VPL = D / 32;
  const int lane = threadIdx.x & 31;
  const int64_t x = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (x >= units) return;   // warp-uniform
  const int c = static_cast<int>(x % nb);
  const int64_t bg = x / nb;
  const int g = static_cast<int>(bg % h_kv), b = static_cast<int>(bg / h_kv);
  const int64_t row_stride = static_cast<int64_t>(h_kv) * D;
  const T* base = K + ((static_cast<int64_t>(b) * n_kv + static_cast<int64_t>(c) * B) * h_kv + g) * D + lane * VPL;
  double best = -1.0;
  int brow = 0;
#pragma unroll 4
  for (int r = 0; r < B; ++r) {
    double n2 = 0.0;
#pragma unroll
    for (int v = 0; v < VPL; ++v) {
      const double kv = static_cast<double>(static_cast<float>(base[r * row_stride + v]));
      n2 = fma(kv, kv, n2);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) n2 += __shfl_xor_sync(0xFFFFFFFFu, n2, o);
    if (n2 > best) { best = n2; brow = r; }   // the same on every lane
  }
  const int64_t row = x * 2 + 1;
#pragma unroll
  for (int v = 0; v < VPL; ++v) {
    const float kv = static_cast<float>(base[brow * row_stride + v]);
    const int t = lane * VPL + v;
    if (mu) mu[row * D + t] = kv;
    if (sig && !full) sig[row * D + t] = 0.f;
    if (table) {
      table[row * 2 * D + t] = __float2bfloat16_rn(kv);
      table[row * 2 * D + D + t] = __float2bfloat16_rn(0.f);
    }
  }
  if (sig && full)
    for (int e = lane; e < D * D; e += 32) sig[row * D * D + e] = 0.f;
}

template <typename T, int D>
cudaError_t run_outlier(const ssa_params& p, const void* K, float* mu, float* sig, void* table,
                        const LaunchCtx& c) {
  const int nb = p.n_kv / p.block;
  const int64_t units = static_cast<int64_t>(p.batch) * p.h_kv * nb;
  const int64_t grid = (units + 7) / 8;
  if (grid > 2147483647) return cudaErrorInvalidValue;
  outlier_kernel<T, D><<<static_cast<unsigned>(grid), 256, 0, c.stream>>>(
      static_cast<const T*>(K), mu, sig, static_cast<__nv_bfloat16*>(table), p.n_kv, p.h_kv, nb, p.block,
      p.sigma == SSA_SIGMA_FULL ? 1 : 0, units);
  note_launch();
  return cudaGetLastError();
}

// A launch summarises units of BLK keys: whole blocks, or the sub-blocks of
// B / S keys when S > 1 (unit c*S + s is sub-block s of block c, so the rows
// come out in that order with no index arithmetic of their own).
template <typename T, int D, int BLK>
cudaError_t run_diag(const ssa_params& p, const void* K, float* mu, float* sig, void* table,
                     const LaunchCtx& c) {
  const int nu = p.n_kv / BLK;
  if constexpr (sizeof(T) == 2) {   // bf16: a warp per unit
    const int64_t units = static_cast<int64_t>(p.batch) * p.h_kv * nu;
    const int64_t grid = (units + 7) / 8;
    if (grid > 2147483647) return cudaErrorInvalidValue;
    summary_bf16_warp_kernel<D, BLK><<<static_cast<unsigned>(grid), 256, 0, c.stream>>>(
        reinterpret_cast<const __nv_bfloat16*>(K), mu, sig, static_cast<__nv_bfloat16*>(table), p.n_kv, p.h_kv, nu,
        units, p.outlier ? 2 : 1);
    note_launch();
    return cudaGetLastError();
  } else {   // float32: a CTA per unit
    dim3 grid(nu, p.h_kv, p.batch);
    summary_diag_kernel<T, D, BLK><<<grid, 256, 0, c.stream>>>(
        static_cast<const T*>(K), mu, sig, static_cast<__nv_bfloat16*>(table), p.n_kv, p.h_kv, nu,
        p.outlier ? 2 : 1);
    note_launch();
    return cudaGetLastError();
  }
}

template <int D, int BLK>
cudaError_t run_full(const ssa_params& p, const void* K, float* mu, float* sig, const LaunchCtx& c) {
  const int nu = p.n_kv / BLK;
  const int smem = BLK * D * static_cast<int>(sizeof(double));
  cudaError_t e = cudaFuncSetAttribute(summary_full_kernel<D, BLK>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(nu, p.h_kv, p.batch);
  summary_full_kernel<D, BLK><<<grid, 256, smem, c.stream>>>(static_cast<const float*>(K), mu, sig,
                                                             p.n_kv, p.h_kv, nu, p.outlier ? 2 : 1);
  note_launch();
  return cudaGetLastError();
}

template <int D>
cudaError_t full_u(int unit, const ssa_params& p, const void* K, float* mu, float* sig, const LaunchCtx& c) {
  if (unit == 32) return run_full<D, 32>(p, K, mu, sig, c);
  if (unit == 64) return run_full<D, 64>(p, K, mu, sig, c);
  if (unit == 128) return run_full<D, 128>(p, K, mu, sig, c);
  return cudaErrorInvalidValue;
}

template <typename T, int D>
cudaError_t diag_u(int unit, const ssa_params& p, const void* K, float* mu, float* sig, void* table,
                   const LaunchCtx& c) {
  if (unit == 32) return run_diag<T, D, 32>(p, K, mu, sig, table, c);
  if (unit == 64) return run_diag<T, D, 64>(p, K, mu, sig, table, c);
  if (unit == 128) return run_diag<T, D, 128>(p, K, mu, sig, table, c);
  return cudaErrorInvalidValue;
}

}  // namespace

namespace {
cudaError_t launch_block_rows(const ssa_params& p, const void* K, float* mu, float* sigma, void* table,
                              const LaunchCtx& c);
}  // namespace

// The block (or sub-block) summary rows, then with the outlier channel each
// block's outlier row after its summary row.
cudaError_t launch_summary(const ssa_params& p, const void* K, float* mu, float* sigma,
                           void* table, const LaunchCtx& c) {
  cudaError_t e = launch_block_rows(p, K, mu, sigma, table, c);
  if (e != cudaSuccess || !p.outlier) return e;
  if (p.subblocks != 1) return cudaErrorInvalidValue;
  if (p.dtype == SSA_BF16) {
    if (p.d == 128) return run_outlier<__nv_bfloat16, 128>(p, K, mu, sigma, table, c);
    if (p.d == 64) return run_outlier<__nv_bfloat16, 64>(p, K, mu, sigma, table, c);
  } else {
    if (p.d == 128) return run_outlier<float, 128>(p, K, mu, sigma, nullptr, c);
    if (p.d == 64) return run_outlier<float, 64>(p, K, mu, sigma, nullptr, c);
  }
  return cudaErrorInvalidValue;
}

namespace {
cudaError_t launch_block_rows(const ssa_params& p, const void* K, float* mu, float* sigma, void* table,
                              const LaunchCtx& c) {
  if (p.subblocks < 1 || p.block % p.subblocks != 0) return cudaErrorInvalidValue;
  const int unit = p.block / p.subblocks;
  if (p.sigma == SSA_SIGMA_FULL) {
    if (p.d == 64) return full_u<64>(unit, p, K, mu, sigma, c);
    if (p.d == 128) return full_u<128>(unit, p, K, mu, sigma, c);
    return cudaErrorInvalidValue;
  }
  if (p.dtype == SSA_BF16) {
    if (p.d == 128) return diag_u<__nv_bfloat16, 128>(unit, p, K, mu, sigma, table, c);
    if (p.d == 64) return diag_u<__nv_bfloat16, 64>(unit, p, K, mu, sigma, table, c);
  } else {
    if (p.d == 128) return diag_u<float, 128>(unit, p, K, mu, sigma, nullptr, c);
    if (p.d == 64) return diag_u<float, 64>(unit, p, K, mu, sigma, nullptr, c);
  }
  return cudaErrorInvalidValue;
}
}  // namespace

}  // namespace ssa

// Step (i) of the layer: per-block key summaries.
//
// "routes ... using only per-block summary statistics"
// [Subquadratic Sparse Attention (SSA), opening section]; the routing score
// needs the block mean mu_c and the covariance Sigma_c of the block's keys
// ["The idea in one screen", routing-score equation].  Normalisation is by
// the number of keys summarised (population moments).
//
// One CTA per (batch, kv-head, unit), a unit being a block of B keys, or a
// sub-block of B / S keys when each block is summarised S times.  The block's B x d keys are read once
// with 16-byte coalesced loads into registers; the mean and then the centred
// second moments are reduced in float64.  For bf16 and float32 keys every
// partial sum of the mean is exact in float64, so mu is the exact block mean
// and its float32 / bfloat16 roundings are reproducible bit for bit.
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
                                                           int n_kv, int h_kv, int nb) {
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
    const int64_t row = (static_cast<int64_t>(b) * h_kv + g) * nb + c;
    if (mu) mu[row * D + threadIdx.x] = m32;
    if (sig) sig[row * D + threadIdx.x] = v32;
    if (table) {
      table[row * 2 * D + threadIdx.x] = __float2bfloat16_rn(m32);
      table[row * 2 * D + D + threadIdx.x] = __float2bfloat16_rn(v32);
    }
  }
}

// Full covariance (float32 problems).  The block is staged centred in
// shared memory as float64; thread e computes entries e, e+256, ...
template <int D, int BLK>
__global__ void __launch_bounds__(256) summary_full_kernel(const float* __restrict__ K,
                                                           float* __restrict__ mu,
                                                           float* __restrict__ sig,
                                                           int n_kv, int h_kv, int nb) {
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
  const int64_t row = (static_cast<int64_t>(b) * h_kv + g) * nb + c;
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

// A launch summarises units of BLK keys: whole blocks, or the sub-blocks of
// B / S keys when S > 1 (unit c*S + s is sub-block s of block c, so the rows
// come out in that order with no index arithmetic of their own).
template <typename T, int D, int BLK>
cudaError_t run_diag(const ssa_params& p, const void* K, float* mu, float* sig, void* table,
                     const LaunchCtx& c) {
  const int nu = p.n_kv / BLK;
  dim3 grid(nu, p.h_kv, p.batch);
  summary_diag_kernel<T, D, BLK><<<grid, 256, 0, c.stream>>>(
      static_cast<const T*>(K), mu, sig, static_cast<__nv_bfloat16*>(table), p.n_kv, p.h_kv, nu);
  note_launch();
  return cudaGetLastError();
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
                                                             p.n_kv, p.h_kv, nu);
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

cudaError_t launch_summary(const ssa_params& p, const void* K, float* mu, float* sigma,
                           void* table, const LaunchCtx& c) {
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

}  // namespace ssa

// Host-side launchers of the SSA kernels (one per translation unit), called
// by the C ABI in ssa_api.cu after it has validated the arguments.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "ssa.h"

namespace ssa {

struct LaunchCtx {
  cudaStream_t stream;
  int device;
  int sm_count;
  uint32_t* err;   // device failure word
};

// Counts every kernel launched through the library.
void note_launch();

// step (i): block summaries
cudaError_t launch_summary(const ssa_params& p, const void* K, float* mu, float* sigma,
                           void* table, const LaunchCtx& c);

// step (i): routing features for the tiled router, [b, h_kv, n_q, 2d] bf16
cudaError_t launch_features(const ssa_params& p, const void* Q, void* F, const LaunchCtx& c);

// step (i): tcgen05 tile router with fused streaming top-k
cudaError_t launch_route_tiled(const ssa_params& p, const CUtensorMap& tmF, const CUtensorMap& tmT,
                               int32_t* block_idx, float* top_scores, const LaunchCtx& c);

// step (i): one CTA per query row (bf16 table)
cudaError_t launch_route_rowwise_bf16(const ssa_params& p, const void* Q, const void* table,
                                      int32_t* block_idx, float* top_scores, const LaunchCtx& c);

// step (i): one CTA per query row (float32 summaries, diagonal or full)
cudaError_t launch_route_rowwise_f32(const ssa_params& p, const void* Q, const float* mu,
                                     const float* sigma, int32_t* block_idx, float* top_scores,
                                     const LaunchCtx& c);

// steps (ii)+(iii): TMA tile-gather attention, bf16
cudaError_t launch_attn_bf16(const ssa_params& p, const CUtensorMap& tmK, const CUtensorMap& tmV,
                             const CUtensorMap& tmQ, const void* Q, const int32_t* block_idx, void* O,
                             float* lse, int32_t* bad, const LaunchCtx& c);

// steps (ii)+(iii): float32 attention
cudaError_t launch_attn_f32(const ssa_params& p, const void* Q, const void* K, const void* V,
                            const int32_t* block_idx, void* O, float* lse, int32_t* bad,
                            const LaunchCtx& c);

// Shared-memory bytes of the tiled router / gather attention (for checks).
int route_tiled_smem_bytes(int d, int topk);
int attn_bf16_smem_bytes(int d);

}  // namespace ssa

// Host-side launchers of the SSA kernels (one per translation unit), called
// by the C ABI in ssa_api.cu after it has validated the arguments.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
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

// Seeds of the tile router (one summary row per block): after every 32
// blocks of a (batch, kv-head), snapshot s holds 128 blocks among blocks
// 0 .. 32 (s + 1) - 1 — the 32 of largest variance sum (ties to the lower
// block) in each of four disjoint sets of 32-block batches — and their
// routing rows.  A unit of query rows whose first row sees snapshot s
// scores those rows first: the least of the maxima over disjoint groups of
// them is a lower bound on every row's k-th best score, the filter's
// starting threshold.
struct RouteSeeds {
  int32_t n_snap;            // snapshots per (batch, kv-head): nb / 32
  float* var;                // [bgs][nb] variance sums of the routing rows
  int32_t* blk;              // [bgs][n_snap][128] seed blocks
  void* tab;                 // [bgs * n_snap * 128][2d] bf16 seed rows
};
size_t route_seed_bytes(const ssa_params& p);
// The feature rows alone: the least workspace of ssa_route_topk's tiled router.
size_t route_min_workspace(const ssa_params& p);   // workspace of the three arrays, 256-byte aligned each
RouteSeeds route_seed_layout(const ssa_params& p, void* base);
cudaError_t launch_route_seeds(const ssa_params& p, const void* table, const RouteSeeds& s, const LaunchCtx& c);

// step (i): tcgen05 tile router with fused streaming top-k; tmS (when not
// NULL) maps the seed rows of `seeds`
cudaError_t launch_route_tiled(const ssa_params& p, const CUtensorMap& tmF, const CUtensorMap& tmT,
                               int32_t* block_idx, float* top_scores, const LaunchCtx& c,
                               const int32_t* unit_need = nullptr, const CUtensorMap* tmS = nullptr,
                               int n_snap = 0);

// step (i): one CTA per query row (bf16 table)
cudaError_t launch_route_rowwise_bf16(const ssa_params& p, const void* Q, const void* table,
                                      int32_t* block_idx, float* top_scores, const LaunchCtx& c,
                                      const uint8_t* skip = nullptr);

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

// Block-major attention plan: per-block lists of the (query, slot) entries
// that selected each key block, cut into tiles of 128 / G queries.
// Query rows per CTA of the selection inversion.
constexpr int kPlanRows = 1024;

// Summary rows per block: the S sub-blocks, plus the outlier row.
inline int rows_per_block(const ssa_params& p) { return p.subblocks + (p.outlier ? 1 : 0); }

struct BlockPlan {
  int32_t bgs, n_q, h_kv, nb, block, topk, window, qpt, nchunk;
  // paired slots (64-key blocks): tile keys are single blocks (0 .. nb-1)
  // and pairs of hot blocks (nb + pair_index(h1, h2)); otherwise the key
  // is the block and nkey = nb
  int32_t pair, nkey;
  int32_t* hot_id;     // [bgs][nb] hot number of each block, -1 when not hot (pair mode)
  int32_t* hot_blk;    // [bgs][kHotBlocks] block of each hot number (pair mode)
  int64_t q_offset;
  int32_t* chist;      // [bgs][nchunk][nkey] slot counts, then their column scans
  int32_t *count, *blk_off, *tile_off;   // [bgs][nkey]
  int32_t *bg_ents, *bg_tiles;           // [bgs]
  int32_t *ent_base, *tile_base;         // [bgs + 1]
  int32_t* entries;                      // make_entry(query row, slot)
  int4* tiles;                           // {bg, block, first entry, entries}
  uint32_t* win;                         // [bgs * n_q] uncovered window blocks of each row
  uint2* rowinfo;                        // [bgs * n_q] {selected-slot mask, skipped block_idx entries}
  // balanced split of the tiles over the block kernel's CTAs
  int32_t max_tiles, grid;               // tile capacity; CTAs (<= kMaxBlockGrid)
  uint8_t* tcost;                        // [max_tiles] estimated cost of each tile
  int32_t* csum;                         // [ceil(max_tiles / 256)] cost per 256 tiles, then its scan
  int32_t* t_start;                      // [grid + 1] first tile of each CTA
};

// Upper bound on the block kernel's grid (one CTA per SM).
constexpr int kMaxBlockGrid = 1024;

cudaError_t launch_block_plan(const ssa_params& p, const int32_t* block_idx, const BlockPlan& pl,
                              const LaunchCtx& c);

// tcgen05 block tiles -> per-(query, head, slot) normalised partial outputs
// partO [items][topk][G][d] (float16, row-scaled by 2^-e) and partL
// [items][stride] of (base-2 log-sum-exp, 2^e).
// tmQ: Q as [b * n_q, h_q, d], 128-byte-swizzled boxes of 64 dims x 8 heads
// (used when G = 8).
cudaError_t launch_attn_block(const ssa_params& p, const BlockPlan& pl, const void* Q,
                              const CUtensorMap& tmK, const CUtensorMap& tmV, const CUtensorMap& tmQ,
                              void* partO, void* partL, const LaunchCtx& c);

// The causal window, densely: one partial per (query, head, window chunk)
// at slot topk + chunk, same format as the block tiles' partials.  tmQ: Q as
// [b * n_q, h_q, d], 128-byte-swizzled boxes of 64 dims x G heads x 128/G
// query rows; tmK, tmV as for the block tiles.
cudaError_t launch_attn_window(const ssa_params& p, const BlockPlan& pl, const CUtensorMap& tmQ,
                               const CUtensorMap& tmK, const CUtensorMap& tmV, void* partO, void* partL,
                               const LaunchCtx& c);

// Per (query, kv-head): the softmax merge of the slot partials into O, lse.
// win, rowinfo: the plan's per-row window blocks and slot records.
cudaError_t launch_attn_merge(const ssa_params& p, const uint32_t* win, const uint2* rowinfo,
                              const void* partO, const void* partL, void* O, float* lse, int32_t* bad,
                              const LaunchCtx& c);

// Hierarchical routing (hier.cu).  Node summaries of the bf16 routing table:
// one warp per (batch * kv-head, node).
struct HierNodeArgs {
  int32_t bgs, nb, nn, M;      // M blocks per node, nn = nb / M complete nodes
  const __nv_bfloat16* T;      // [bgs, nb, 2d] block routing rows
  __nv_bfloat16* NT;           // [bgs, nn, 2d] node rows [centre ; cap]
  float* radius;               // [bgs, nn]
  uint32_t* bound;             // [bgs, 2] float bits (largest radius, largest row norm); zeroed first
};
cudaError_t launch_hier_nodes(const ssa_params& p, const HierNodeArgs& a, const LaunchCtx& c);

// The tree's second level: one warp per (batch * kv-head, super-node) of M
// consecutive nodes.
struct HierSuperArgs {
  int32_t bgs, nn, ns, M;      // ns = nn / M complete super-nodes
  const __nv_bfloat16* NT;     // [bgs, nn, 2d] node rows
  const float* radius;         // [bgs, nn] node radii
  __nv_bfloat16* ST;           // [bgs, ns, 2d] super-node rows [centre ; cap]
  float* sradius;              // [bgs, ns] recursive radii
  uint32_t* sbound;            // [bgs] float bits: largest super-node radius; zeroed first
  uint32_t* bound;             // [bgs, 2] of the nodes: the row-norm half is raised to the super rows'
};
cudaError_t launch_hier_supers(const ssa_params& p, const HierSuperArgs& a, const LaunchCtx& c);

// Two-level routing, first probe: one warp per (batch * kv-head, query row)
// expands the row's best super-nodes and ranks their nodes (and the nodes
// outside complete super-nodes) by their exact node scores, keeping the best
// probe+1 in the layout the node router gives the block probe.
struct HierProbe2Args {
  int32_t n_q, h_kv, bgs, nn, ns, M, block, probe;
  int64_t q_offset;
  const __nv_bfloat16* F;      // [bgs, n_q, 2d] routing features
  const __nv_bfloat16* NT;     // [bgs, nn, 2d] node rows
  const int32_t* sup_idx;      // [b, n_q, h_kv, probe+1] best super-nodes, ascending, -1 padded (null: none)
  const float* sup_score;      // same layout, their scores
  int32_t* node_idx;           // [b, n_q, h_kv, probe+1] out: best candidate nodes, ascending, -1 padded
  float* node_score;           // same layout, their scores
  int32_t* n_cand;             // [b, n_q, h_kv] out: candidate nodes of the row
  float* w2_next;              // [b, n_q, h_kv] out: best unexpanded super-node score, -inf if none
};
cudaError_t launch_hier_probe2(const ssa_params& p, const HierProbe2Args& a, const LaunchCtx& c);

// The per-row probe of the best nodes and the certificate: one warp per
// (batch * kv-head, query row).
struct HierProbeArgs {
  int32_t n_q, h_kv, bgs, nb, nn, M, block, topk, probe, n_tiles;
  int64_t q_offset;
  const __nv_bfloat16* F;      // [bgs, n_q, 2d] routing features
  const __nv_bfloat16* T;      // [bgs, nb, 2d] block routing rows
  const int32_t* node_idx;     // [b, n_q, h_kv, probe+1] best nodes, ascending, -1 padded
  const float* node_score;     // same layout, their scores f . [centre ; cap]
  const float* bound;          // [bgs, 2]
  int32_t* block_idx;          // [b, n_q, h_kv, topk]
  uint8_t* cert;               // [b, n_q, h_kv] (may be null)
  int32_t* unit_need;          // [bgs, n_tiles] set to 1 for units holding an uncertified row (may be null)
  // two levels (null for one): the row's candidate nodes and best
  // unexpanded super-node score from the first probe, and the largest
  // super-node radius of each (batch * kv-head)
  const int32_t* n_cand;       // [b, n_q, h_kv]
  const float* w2_next;        // [b, n_q, h_kv]
  const float* sbound;         // [bgs]
};
cudaError_t launch_hier_probe(const ssa_params& p, const HierProbeArgs& a, const LaunchCtx& c);

// One CTA whose bounded wait never completes (the failure-path self-test).
cudaError_t launch_selftest_wait(const LaunchCtx& c);


// Shared-memory bytes of the tiled router / gather attention (for checks).
int route_tiled_smem_bytes(int d, int topk);
int attn_bf16_smem_bytes(int d);

}  // namespace ssa

// C ABI of libssa: argument validation, workspace carving, TMA descriptor
// encoding and kernel dispatch.  See include/ssa.h for the contract.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "invert.cuh"
#include "kernels.h"
#include "ssa.h"

namespace ssa {

static std::atomic<uint64_t> g_launches{0};
void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

}  // namespace ssa

// Device failure word (one per device that loads the library).
__device__ uint32_t g_ssa_device_error;

namespace {

using ssa::LaunchCtx;

constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool ready = false;
  int sm_count = 0;
  uint32_t* err = nullptr;
};

std::mutex g_dev_mu;
DeviceInfo g_dev[kMaxDevices];

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

ssa_status make_ctx(void* stream, LaunchCtx& c) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SSA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    if (cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return SSA_ERR_CUDA;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_ssa_device_error) != cudaSuccess) return SSA_ERR_CUDA;
    d.err = static_cast<uint32_t*>(p);
    d.ready = true;
  }
  c.stream = static_cast<cudaStream_t>(stream);
  c.device = dev;
  c.sm_count = d.sm_count;
  c.err = d.err;
  return SSA_OK;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t round_up(size_t x) { return (x + 255) & ~size_t(255); }

int64_t nb_of(const ssa_params& p) { return p.block > 0 ? p.n_kv / p.block : 0; }
// Summary rows per (batch, kv-head): one per sub-block.
int64_t summary_rows(const ssa_params& p) { return nb_of(p) * ssa::rows_per_block(p); }
size_t esize(const ssa_params& p) { return p.dtype == SSA_BF16 ? 2 : 4; }

bool is_empty(const ssa_params& p) { return p.batch == 0 || p.n_q == 0; }

// Shape / support checks shared by every call.
ssa_status check_params(const ssa_params* pp) {
  if (!pp) return SSA_ERR_INVALID_ARG;
  const ssa_params& p = *pp;
  if (p.batch < 0 || p.n_q < 0 || p.n_kv < 0 || p.h_q < 1 || p.h_kv < 1 || p.d < 1 || p.block < 1 ||
      p.topk < 1 || p.window < 1)
    return SSA_ERR_INVALID_ARG;
  if (p.h_q % p.h_kv != 0 || p.n_kv % p.block != 0) return SSA_ERR_INVALID_ARG;
  if (p.subblocks < 1 || p.block % p.subblocks != 0 || (p.outlier != 0 && p.outlier != 1))
    return SSA_ERR_INVALID_ARG;
  if (p.q_offset < 0 || p.q_offset + p.n_q > p.n_kv) return SSA_ERR_INVALID_ARG;
  if ((p.dtype != SSA_F32 && p.dtype != SSA_BF16) || (p.sigma != SSA_SIGMA_DIAG && p.sigma != SSA_SIGMA_FULL) ||
      p.route_impl < SSA_ROUTE_AUTO || p.route_impl > SSA_ROUTE_ROWWISE)
    return SSA_ERR_INVALID_ARG;
  if (!isfinite(p.beta) || !isfinite(p.scale) || !(p.scale > 0.f)) return SSA_ERR_INVALID_ARG;
  const int G = p.h_q / p.h_kv;
  if (p.d != 64 && p.d != 128) return SSA_ERR_UNSUPPORTED;
  if (p.block != 64 && p.block != 128) return SSA_ERR_UNSUPPORTED;
  if ((p.subblocks != 1 && p.subblocks != 2 && p.subblocks != 4) || p.block / p.subblocks < 32)
    return SSA_ERR_UNSUPPORTED;
  if (p.outlier && p.subblocks != 1) return SSA_ERR_UNSUPPORTED;
  if (G != 1 && G != 2 && G != 4 && G != 8) return SSA_ERR_UNSUPPORTED;
  if (p.topk > 32 || p.window > 4032) return SSA_ERR_UNSUPPORTED;
  if (p.dtype == SSA_BF16 && p.sigma != SSA_SIGMA_DIAG) return SSA_ERR_UNSUPPORTED;
  // index ranges used by the kernels and the TMA coordinates
  const int64_t rows_kv = static_cast<int64_t>(p.batch) * p.n_kv;
  const int64_t rows_q = static_cast<int64_t>(p.batch) * p.h_kv * p.n_q;
  const int64_t rows_t = static_cast<int64_t>(p.batch) * p.h_kv * summary_rows(p);
  if (rows_kv > INT32_MAX || rows_q > INT32_MAX || rows_t > INT32_MAX) return SSA_ERR_UNSUPPORTED;
  if (p.batch > 65535 || p.h_kv > 65535 || nb_of(p) > 2147483647) return SSA_ERR_UNSUPPORTED;
  return SSA_OK;
}

bool use_tiled(const ssa_params& p) {
  if (p.dtype != SSA_BF16) return false;
  if (p.route_impl == SSA_ROUTE_TILED) return true;
  if (p.route_impl == SSA_ROUTE_ROWWISE) return false;
  return p.n_q >= 128;
}

bool rowwise_fits(const ssa_params& p) {
  int64_t n2 = 1;
  while (n2 < nb_of(p)) n2 <<= 1;
  return n2 * 8 <= 200 * 1024 && p.n_q <= 2147483647 && p.h_kv <= 65535;
}

size_t features_bytes(const ssa_params& p) {
  return use_tiled(p) ? round_up(static_cast<size_t>(p.batch) * p.h_kv * p.n_q * 2 * p.d * 2) : 0;
}
// Route workspace: the feature rows (required by the tiled router), then
// the router's seed arrays (used when the caller's workspace holds them).
size_t route_ws_bytes(const ssa_params& p) {
  return features_bytes(p) + (use_tiled(p) ? ssa::route_seed_bytes(p) : 0);
}
size_t table_bytes(const ssa_params& p) {
  return p.dtype == SSA_BF16 ? round_up(static_cast<size_t>(p.batch) * p.h_kv * summary_rows(p) * 2 * p.d * 2) : 0;
}
size_t mu_bytes(const ssa_params& p) {
  return p.dtype == SSA_F32 ? round_up(static_cast<size_t>(p.batch) * p.h_kv * summary_rows(p) * p.d * 4) : 0;
}
size_t sigma_bytes(const ssa_params& p) {
  if (p.dtype != SSA_F32) return 0;
  const size_t per = p.sigma == SSA_SIGMA_FULL ? static_cast<size_t>(p.d) * p.d : p.d;
  return round_up(static_cast<size_t>(p.batch) * p.h_kv * summary_rows(p) * per * 4);
}
size_t idx_bytes(const ssa_params& p) {
  return round_up(static_cast<size_t>(p.batch) * p.n_q * p.h_kv * p.topk * 4);
}

ssa_status from_cuda(cudaError_t e) { return e == cudaSuccess ? SSA_OK : SSA_ERR_CUDA; }

// Block-major attention applies to long bf16 problems whose query heads
// fill a 128-row tensor-core tile in groups of G, whose row slots (selected
// blocks plus window chunks) fit the 6-bit slot field of an entry and whose
// window blocks fit a 32-bit mask, and whose per-block counters fit the
// inversion's shared memory.
bool use_block_attn(const ssa_params& p) {
  const int G = p.h_q / p.h_kv;
  const int64_t nb = p.n_kv / p.block;
  return p.dtype == SSA_BF16 && p.d == 128 && (G == 1 || G == 2 || G == 4 || G == 8) && p.topk * G <= 128 &&
         ssa::window_slots(p.window, p.block) <= 32 && nb <= 16384 && p.n_q >= 1024 && p.n_q < (1 << 25);
}

// Paired slots: the block-major attention evaluates two selected blocks per
// slot (128-key tiles for 64-key blocks, 256-key tiles for 128-key blocks).
bool pair_mode(const ssa_params& p) { return p.block == 64 || p.block == 128; }

struct AttnLayout {
  size_t chist, count, blk_off, tile_off, bg_ents, bg_tiles, ent_base, tile_base, entries, tiles, tcost, csum,
      t_start, win, rowinfo, hot_id, hot_blk, part_o, part_l, total;
  int nchunk, nsl, nkey;
  size_t max_tiles;
};

AttnLayout attn_layout(const ssa_params& p) {
  AttnLayout L{};
  if (!use_block_attn(p)) return L;
  const size_t bgs = static_cast<size_t>(p.batch) * p.h_kv;
  const size_t nb = static_cast<size_t>(nb_of(p));
  const size_t G = static_cast<size_t>(p.h_q / p.h_kv);
  const size_t qpt = 128 / G;
  L.nchunk = (p.n_q + ssa::kPlanRows - 1) / ssa::kPlanRows;
  L.nsl = p.topk + ssa::window_chunks(p.window, p.h_q / p.h_kv);
  const size_t items = bgs * p.n_q;
  const size_t sel = items * L.nsl;                       // entries, at most
  const size_t nkey = nb + (pair_mode(p) ? static_cast<size_t>(ssa::kPairKeys) : 0);
  L.nkey = static_cast<int>(nkey);
  const size_t max_tiles = (sel + qpt - 1) / qpt + bgs * nkey;
  size_t off = 0;
  L.chist = off; off += round_up(bgs * L.nchunk * nkey * 4);
  L.count = off; off += round_up(bgs * nkey * 4);
  L.blk_off = off; off += round_up(bgs * nkey * 4);
  L.tile_off = off; off += round_up(bgs * nkey * 4);
  L.bg_ents = off; off += round_up(bgs * 4);
  L.bg_tiles = off; off += round_up(bgs * 4);
  L.ent_base = off; off += round_up((bgs + 1) * 4);
  L.tile_base = off; off += round_up((bgs + 1) * 4);
  L.entries = off; off += round_up(sel * 4);
  L.tiles = off; off += round_up(max_tiles * 16);
  L.max_tiles = max_tiles;
  L.tcost = off; off += round_up(max_tiles);
  L.csum = off; off += round_up((max_tiles + 255) / 256 * 4);
  L.t_start = off; off += round_up((ssa::kMaxBlockGrid + 1) * 4);
  L.win = off; off += round_up(items * 4);
  L.rowinfo = off; off += round_up(items * 8);
  L.hot_id = off; off += pair_mode(p) ? round_up(bgs * nb * 4) : 0;
  L.hot_blk = off; off += pair_mode(p) ? round_up(bgs * ssa::kHotBlocks * 4) : 0;
  L.part_o = off; off += round_up(sel * G * p.d * 2);
  L.part_l = off; off += round_up(sel * G * 8);
  L.total = off;
  return L;
}

// 2D bf16 map of a [rows, cols] row-major matrix, 64 x box_rows boxes, 128B swizzle.
bool encode_2d(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2D bf16 map of a [rows, cols] row-major matrix, unswizzled boxes of 64 x box_rows.
bool encode_rows(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {cols, rows};
  const cuuint64_t strides[1] = {cols * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3D bf16 map of K or V viewed as [b*n_kv, h_kv, d]; boxes of 64 keys x 1 head x 64 dims.
bool encode_kv(CUtensorMap* m, const void* base, const ssa_params& p) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(p.d), static_cast<cuuint64_t>(p.h_kv),
                              static_cast<cuuint64_t>(p.batch) * p.n_kv};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(p.d) * 2, static_cast<cuuint64_t>(p.h_kv) * p.d * 2};
  const cuuint32_t box[3] = {64, 1, 64};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3D bf16 map of Q viewed as [b*n_q, h_q, d]; 128-byte-swizzled boxes of
// 64 dims x 8 heads x 1 query row.
bool encode_q_heads(CUtensorMap* m, const void* base, const ssa_params& p) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(p.d), static_cast<cuuint64_t>(p.h_q),
                              static_cast<cuuint64_t>(p.batch) * p.n_q};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(p.d) * 2, static_cast<cuuint64_t>(p.h_q) * p.d * 2};
  const cuuint32_t box[3] = {64, 8, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3D bf16 map of Q viewed as [b*n_q, h_q, d]; 128-byte-swizzled boxes of
// 64 dims x `heads` heads x `rows` query rows.
bool encode_q_tile(CUtensorMap* m, const void* base, const ssa_params& p, int heads, int rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(p.d), static_cast<cuuint64_t>(p.h_q),
                              static_cast<cuuint64_t>(p.batch) * p.n_q};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(p.d) * 2, static_cast<cuuint64_t>(p.h_q) * p.d * 2};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(heads), static_cast<cuuint32_t>(rows)};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

ssa_status do_summary(const ssa_params& p, const void* K, float* mu, float* sigma, void* table,
                      const LaunchCtx& c) {
  if (p.batch == 0 || p.n_kv == 0) return SSA_OK;
  if (!mu && !sigma && !table) return SSA_OK;
  return from_cuda(ssa::launch_summary(p, K, mu, sigma, table, c));
}

ssa_status do_route(const ssa_params& p, const void* Q, const float* mu, const float* sigma,
                    const void* table, int32_t* idx, float* scores, void* ws, size_t ws_bytes,
                    const LaunchCtx& c) {
  if (is_empty(p)) return SSA_OK;
  if (p.dtype == SSA_F32) {
    if (!rowwise_fits(p)) return SSA_ERR_UNSUPPORTED;
    return from_cuda(ssa::launch_route_rowwise_f32(p, Q, mu, sigma, idx, scores, c));
  }
  if (!use_tiled(p)) {
    if (!rowwise_fits(p)) return SSA_ERR_UNSUPPORTED;
    return from_cuda(ssa::launch_route_rowwise_bf16(p, Q, table, idx, scores, c));
  }
  const size_t need = features_bytes(p);
  if (ws_bytes < need || (need && !ws) || !aligned16(ws)) return SSA_ERR_WORKSPACE;
  ssa_status st = from_cuda(ssa::launch_features(p, Q, ws, c));
  if (st != SSA_OK) return st;
  CUtensorMap tmF, tmT;
  const uint64_t kf = 2 * static_cast<uint64_t>(p.d);
  if (!encode_2d(&tmF, ws, kf, static_cast<uint64_t>(p.batch) * p.h_kv * p.n_q, 128) ||
      !encode_2d(&tmT, table, kf, static_cast<uint64_t>(p.batch) * p.h_kv * summary_rows(p), 128))
    return SSA_ERR_CUDA;
  const size_t sb = ssa::route_seed_bytes(p);
  if (sb && ws_bytes >= need + sb) {
    const ssa::RouteSeeds S = ssa::route_seed_layout(p, static_cast<uint8_t*>(ws) + need);
    if ((st = from_cuda(ssa::launch_route_seeds(p, table, S, c))) != SSA_OK) return st;
    const uint64_t srows = static_cast<uint64_t>(p.batch) * p.h_kv * S.n_snap * 128;   // 128 seed rows each
    CUtensorMap tmS;
    if (!encode_2d(&tmS, S.tab, kf, srows, 128)) return SSA_ERR_CUDA;
    return from_cuda(ssa::launch_route_tiled(p, tmF, tmT, idx, scores, c, nullptr, &tmS, S.n_snap));
  }
  return from_cuda(ssa::launch_route_tiled(p, tmF, tmT, idx, scores, c));
}

ssa::BlockPlan block_plan(const ssa_params& p, const AttnLayout& L, uint8_t* w) {
  ssa::BlockPlan pl;
  pl.bgs = p.batch * p.h_kv;
  pl.n_q = p.n_q;
  pl.h_kv = p.h_kv;
  pl.nb = static_cast<int32_t>(nb_of(p));
  pl.block = p.block;
  pl.topk = p.topk;
  pl.window = p.window;
  pl.qpt = 128 / (p.h_q / p.h_kv);
  pl.nchunk = L.nchunk;
  pl.pair = pair_mode(p) ? 1 : 0;
  pl.nkey = L.nkey;
  pl.hot_id = pl.pair ? reinterpret_cast<int32_t*>(w + L.hot_id) : nullptr;
  pl.hot_blk = pl.pair ? reinterpret_cast<int32_t*>(w + L.hot_blk) : nullptr;
  pl.q_offset = p.q_offset;
  pl.chist = reinterpret_cast<int32_t*>(w + L.chist);
  pl.count = reinterpret_cast<int32_t*>(w + L.count);
  pl.blk_off = reinterpret_cast<int32_t*>(w + L.blk_off);
  pl.tile_off = reinterpret_cast<int32_t*>(w + L.tile_off);
  pl.bg_ents = reinterpret_cast<int32_t*>(w + L.bg_ents);
  pl.bg_tiles = reinterpret_cast<int32_t*>(w + L.bg_tiles);
  pl.ent_base = reinterpret_cast<int32_t*>(w + L.ent_base);
  pl.tile_base = reinterpret_cast<int32_t*>(w + L.tile_base);
  pl.entries = reinterpret_cast<int32_t*>(w + L.entries);
  pl.tiles = reinterpret_cast<int4*>(w + L.tiles);
  pl.win = reinterpret_cast<uint32_t*>(w + L.win);
  pl.rowinfo = reinterpret_cast<uint2*>(w + L.rowinfo);
  pl.max_tiles = static_cast<int32_t>(L.max_tiles);
  pl.grid = 0;   // set by the caller from the device's SM count
  pl.tcost = w + L.tcost;
  pl.csum = reinterpret_cast<int32_t*>(w + L.csum);
  pl.t_start = reinterpret_cast<int32_t*>(w + L.t_start);
  return pl;
}

struct AttnMaps {
  CUtensorMap K, V, Q, Qh;   // Q: unswizzled G-row boxes (gather path); Qh: 8-head boxes (G = 8 tiles)
  CUtensorMap Qw;            // G heads x 128/G query rows (window tiles)
};

bool encode_attn_maps(AttnMaps& m, const ssa_params& p, const void* Q, const void* K, const void* V) {
  const uint32_t G = static_cast<uint32_t>(p.h_q / p.h_kv);
  if (!encode_kv(&m.K, K, p) || !encode_kv(&m.V, V, p) ||
      !encode_rows(&m.Q, Q, p.d, static_cast<uint64_t>(p.batch) * p.n_q * p.h_q, G))
    return false;
  if (p.d == 128 && (G == 1 || G == 2 || G == 4 || G == 8) && !encode_q_tile(&m.Qw, Q, p, G, 128 / G)) return false;
  if (G == 8 && p.d == 128) return encode_q_heads(&m.Qh, Q, p);
  m.Qh = m.Q;
  return true;
}

// Block-major stages; the caller has checked that the problem qualifies and
// that `w` holds attn_layout(p).total bytes.
ssa_status attn_stage_plan(const ssa_params& p, const int32_t* idx, uint8_t* w, const LaunchCtx& c) {
  const AttnLayout L = attn_layout(p);
  ssa::BlockPlan pl = block_plan(p, L, w);
  pl.grid = c.sm_count;
  return from_cuda(ssa::launch_block_plan(p, idx, pl, c));
}

ssa_status attn_stage_blocks(const ssa_params& p, const void* Q, const AttnMaps& m, uint8_t* w, const LaunchCtx& c) {
  const AttnLayout L = attn_layout(p);
  ssa::BlockPlan pl = block_plan(p, L, w);
  pl.grid = c.sm_count;
  return from_cuda(ssa::launch_attn_block(p, pl, Q, m.K, m.V, m.Qh, w + L.part_o, w + L.part_l, c));
}

ssa_status attn_stage_window(const ssa_params& p, const AttnMaps& m, uint8_t* w, const LaunchCtx& c) {
  const AttnLayout L = attn_layout(p);
  ssa::BlockPlan pl = block_plan(p, L, w);
  pl.grid = c.sm_count;
  return from_cuda(ssa::launch_attn_window(p, pl, m.Qw, m.K, m.V, w + L.part_o, w + L.part_l, c));
}

ssa_status attn_stage_merge(const ssa_params& p, const int32_t* idx, void* O, float* lse, int32_t* bad,
                            const uint8_t* w, const LaunchCtx& c) {
  const AttnLayout L = attn_layout(p);
  (void)idx;   // the plan recorded each row's slots from block_idx
  return from_cuda(ssa::launch_attn_merge(p, reinterpret_cast<const uint32_t*>(w + L.win),
                                          reinterpret_cast<const uint2*>(w + L.rowinfo), w + L.part_o,
                                          w + L.part_l, O, lse, bad, c));
}

ssa_status do_attn(const ssa_params& p, const void* Q, const void* K, const void* V,
                   const int32_t* idx, void* O, float* lse, int32_t* bad, void* ws, size_t ws_bytes,
                   const LaunchCtx& c) {
  if (is_empty(p)) return SSA_OK;
  if (p.dtype == SSA_F32) return from_cuda(ssa::launch_attn_f32(p, Q, K, V, idx, O, lse, bad, c));
  AttnMaps m;
  if (!encode_attn_maps(m, p, Q, K, V)) return SSA_ERR_CUDA;
  const AttnLayout L = attn_layout(p);
  if (L.total == 0 || !ws || ws_bytes < L.total || !aligned16(ws))
    return from_cuda(ssa::launch_attn_bf16(p, m.K, m.V, m.Q, Q, idx, O, lse, bad, c));
  uint8_t* w = static_cast<uint8_t*>(ws);
  ssa_status st = attn_stage_plan(p, idx, w, c);
  if (st == SSA_OK) st = attn_stage_blocks(p, Q, m, w, c);
  if (st == SSA_OK) st = attn_stage_window(p, m, w, c);
  if (st == SSA_OK) st = attn_stage_merge(p, idx, O, lse, bad, w, c);
  return st;
}

struct ForwardLayout {
  size_t table, mu, sigma, feat, idx, attn, total;
};

ForwardLayout forward_layout(const ssa_params& p) {
  ForwardLayout L;
  size_t off = 0;
  L.table = off; off += table_bytes(p);
  L.mu = off; off += mu_bytes(p);
  L.sigma = off; off += sigma_bytes(p);
  L.feat = off; off += route_ws_bytes(p);
  L.idx = off; off += idx_bytes(p);
  L.attn = off; off += attn_layout(p).total;
  L.total = off;
  return L;
}

struct HostioLayout {
  size_t q, k, v, o, lse, ws, total;
};

HostioLayout hostio_layout(const ssa_params& p) {
  HostioLayout L;
  const size_t es = esize(p);
  size_t off = 0;
  L.q = off; off += round_up(static_cast<size_t>(p.batch) * p.n_q * p.h_q * p.d * es);
  L.k = off; off += round_up(static_cast<size_t>(p.batch) * p.n_kv * p.h_kv * p.d * es);
  L.v = off; off += round_up(static_cast<size_t>(p.batch) * p.n_kv * p.h_kv * p.d * es);
  L.o = off; off += round_up(static_cast<size_t>(p.batch) * p.n_q * p.h_q * p.d * es);
  L.lse = off; off += round_up(static_cast<size_t>(p.batch) * p.n_q * p.h_q * 4);
  L.ws = off; off += forward_layout(p).total;
  L.total = off;
  return L;
}

ssa_status forward_impl(const ssa_params& p, const void* Q, const void* K, const void* V, void* O,
                        float* lse, uint8_t* ws, size_t ws_bytes, const LaunchCtx& c) {
  const ForwardLayout L = forward_layout(p);
  if (ws_bytes < L.total || (L.total && !ws) || !aligned16(ws)) return SSA_ERR_WORKSPACE;
  void* table = table_bytes(p) ? ws + L.table : nullptr;
  float* mu = mu_bytes(p) ? reinterpret_cast<float*>(ws + L.mu) : nullptr;
  float* sg = sigma_bytes(p) ? reinterpret_cast<float*>(ws + L.sigma) : nullptr;
  int32_t* idx = reinterpret_cast<int32_t*>(ws + L.idx);
  ssa_status st = do_summary(p, K, mu, sg, table, c);
  if (st != SSA_OK) return st;
  st = do_route(p, Q, mu, sg, table, idx, nullptr, route_ws_bytes(p) ? ws + L.feat : nullptr,
                route_ws_bytes(p), c);
  if (st != SSA_OK) return st;
  const size_t aw = attn_layout(p).total;
  return do_attn(p, Q, K, V, idx, O, lse, nullptr, aw ? ws + L.attn : nullptr, aw, c);
}

// ------------------------------------------------------------------ hierarchical routing

int hier_levels(const ssa_hier_params& hp) { return hp.levels == 2 ? 2 : 1; }

struct HierNodeLayout {
  int64_t nn, ns;   // nodes; super-nodes (second level, else 0)
  size_t table, radius, bound, stable, sradius, sbound, total;
};

HierNodeLayout hier_node_layout(const ssa_params& p, const ssa_hier_params& hp) {
  HierNodeLayout L;
  const size_t bgs = static_cast<size_t>(p.batch) * p.h_kv;
  L.nn = nb_of(p) / hp.fanout;
  L.ns = hier_levels(hp) == 2 ? L.nn / hp.fanout : 0;
  size_t off = 0;
  L.table = off; off += round_up(bgs * L.nn * 2 * p.d * 2);
  L.radius = off; off += round_up(bgs * L.nn * 4);
  L.bound = off; off += round_up(bgs * 2 * 4);
  L.stable = off; off += round_up(bgs * L.ns * 2 * p.d * 2);
  L.sradius = off; off += round_up(bgs * L.ns * 4);
  L.sbound = off; off += hier_levels(hp) == 2 ? round_up(bgs * 4) : 0;
  L.total = off;
  return L;
}

struct HierLayout {
  size_t feat, nidx, nsc, cert, need, sidx, ssc, ncand, w2n, total;
};

int32_t route_tiles(const ssa_params& p) { return (p.n_q + 255) / 256; }

HierLayout hier_layout(const ssa_params& p, const ssa_hier_params& hp) {
  HierLayout L;
  const size_t rows = static_cast<size_t>(p.batch) * p.n_q * p.h_kv;
  const size_t bgs = static_cast<size_t>(p.batch) * p.h_kv;
  size_t off = 0;
  L.feat = off; off += round_up(rows * 2 * p.d * 2);
  L.nidx = off; off += round_up(rows * (hp.probe + 1) * 4);
  L.nsc = off; off += round_up(rows * (hp.probe + 1) * 4);
  L.cert = off; off += round_up(rows);
  L.need = off; off += (hp.escalate && use_tiled(p)) ? round_up(bgs * route_tiles(p) * 4) : 0;
  const bool two = hier_levels(hp) == 2;
  L.sidx = off; off += two ? round_up(rows * (hp.probe + 1) * 4) : 0;
  L.ssc = off; off += two ? round_up(rows * (hp.probe + 1) * 4) : 0;
  L.ncand = off; off += two ? round_up(rows * 4) : 0;
  L.w2n = off; off += two ? round_up(rows * 4) : 0;
  L.total = off;
  return L;
}

ssa_status check_hier(const ssa_params* p, const ssa_hier_params* hp) {
  ssa_status st = check_params(p);
  if (st != SSA_OK) return st;
  if (!hp || hp->levels < 0 || hp->levels > 2) return SSA_ERR_INVALID_ARG;
  const int M = hp->fanout;
  if (M < 1 || M > 64 || (M & (M - 1)) != 0) return SSA_ERR_INVALID_ARG;
  if (hp->probe < 1 || hp->probe > 31 || (hp->escalate != 0 && hp->escalate != 1)) return SSA_ERR_INVALID_ARG;
  if ((hp->probe + 1) * M > 512) return SSA_ERR_UNSUPPORTED;   // candidates per row of the probe kernel
  if (p->dtype != SSA_BF16 || p->subblocks != 1 || p->outlier) return SSA_ERR_UNSUPPORTED;
  if (!use_tiled(*p) && !rowwise_fits(*p)) return SSA_ERR_UNSUPPORTED;
  return SSA_OK;
}

// The node problem: nodes of M blocks act as blocks of M * B keys (and
// super-nodes of M nodes as blocks of M * M * B keys: span = M * M).
ssa_params node_params(const ssa_params& p, const ssa_hier_params& hp, int64_t nn, int span) {
  ssa_params pn = p;
  pn.block = p.block * span;
  pn.n_kv = static_cast<int32_t>(nn * pn.block);
  pn.topk = hp.probe + 1;
  pn.subblocks = 1;
  return pn;
}

ssa_status do_route_hier(const ssa_params& p, const ssa_hier_params& hp, const void* Q, const void* table,
                         const void* nodes, int32_t* idx, uint8_t* cert_out, uint8_t* ws, const LaunchCtx& c) {
  const HierNodeLayout NL = hier_node_layout(p, hp);
  const HierLayout H = hier_layout(p, hp);
  const uint8_t* nd = static_cast<const uint8_t*>(nodes);
  const uint64_t kf = 2 * static_cast<uint64_t>(p.d);
  const int64_t bgs = static_cast<int64_t>(p.batch) * p.h_kv;
  void* F = ws + H.feat;
  int32_t* nidx = reinterpret_cast<int32_t*>(ws + H.nidx);
  float* nsc = reinterpret_cast<float*>(ws + H.nsc);
  uint8_t* cert = cert_out ? cert_out : ws + H.cert;
  const bool tiled = use_tiled(p);
  ssa_status st = from_cuda(ssa::launch_features(p, Q, F, c));
  if (st != SSA_OK) return st;
  CUtensorMap tmF;
  if (tiled && !encode_2d(&tmF, F, kf, static_cast<uint64_t>(bgs) * p.n_q, 128)) return SSA_ERR_CUDA;
  // the best probe+1 entries of every row, with their scores, from the
  // block router run over a node or super-node table
  auto rank_rows = [&](const uint8_t* rows_table, int64_t n_rows, int span, int32_t* out_idx,
                       float* out_sc) -> ssa_status {
    const ssa_params pn = node_params(p, hp, n_rows, span);
    if (tiled) {
      CUtensorMap tmN;
      if (!encode_2d(&tmN, rows_table, kf, static_cast<uint64_t>(bgs * n_rows), 128)) return SSA_ERR_CUDA;
      return from_cuda(ssa::launch_route_tiled(pn, tmF, tmN, out_idx, out_sc, c));
    }
    return from_cuda(ssa::launch_route_rowwise_bf16(pn, Q, rows_table, out_idx, out_sc, c));
  };
  const bool two = hier_levels(hp) == 2;
  if (two) {
    // super-nodes first; the first probe ranks the candidate nodes exactly
    int32_t* sidx = reinterpret_cast<int32_t*>(ws + H.sidx);
    float* ssc = reinterpret_cast<float*>(ws + H.ssc);
    if (NL.ns > 0 && (st = rank_rows(nd + NL.stable, NL.ns, hp.fanout * hp.fanout, sidx, ssc)) != SSA_OK)
      return st;
    ssa::HierProbe2Args a2;
    a2.n_q = p.n_q; a2.h_kv = p.h_kv; a2.bgs = static_cast<int32_t>(bgs);
    a2.nn = static_cast<int32_t>(NL.nn); a2.ns = static_cast<int32_t>(NL.ns); a2.M = hp.fanout;
    a2.block = p.block; a2.probe = hp.probe; a2.q_offset = p.q_offset;
    a2.F = static_cast<const __nv_bfloat16*>(F);
    a2.NT = reinterpret_cast<const __nv_bfloat16*>(nd + NL.table);
    a2.sup_idx = NL.ns > 0 ? sidx : nullptr;
    a2.sup_score = NL.ns > 0 ? ssc : nullptr;
    a2.node_idx = nidx; a2.node_score = nsc;
    a2.n_cand = reinterpret_cast<int32_t*>(ws + H.ncand);
    a2.w2_next = reinterpret_cast<float*>(ws + H.w2n);
    if ((st = from_cuda(ssa::launch_hier_probe2(p, a2, c))) != SSA_OK) return st;
  } else if (NL.nn > 0 && (st = rank_rows(nd + NL.table, NL.nn, hp.fanout, nidx, nsc)) != SSA_OK) {
    return st;
  }
  int32_t* need = (hp.escalate && tiled) ? reinterpret_cast<int32_t*>(ws + H.need) : nullptr;
  if (need && cudaMemsetAsync(need, 0, static_cast<size_t>(bgs) * route_tiles(p) * 4, c.stream) != cudaSuccess)
    return SSA_ERR_CUDA;
  ssa::HierProbeArgs a;
  a.n_q = p.n_q; a.h_kv = p.h_kv; a.bgs = static_cast<int32_t>(bgs);
  a.nb = static_cast<int32_t>(nb_of(p)); a.nn = static_cast<int32_t>(NL.nn); a.M = hp.fanout;
  a.block = p.block; a.topk = p.topk; a.probe = hp.probe; a.n_tiles = route_tiles(p);
  a.q_offset = p.q_offset;
  a.F = static_cast<const __nv_bfloat16*>(F);
  a.T = static_cast<const __nv_bfloat16*>(table);
  a.node_idx = nidx; a.node_score = nsc;
  a.bound = reinterpret_cast<const float*>(nd + NL.bound);
  a.block_idx = idx; a.cert = cert; a.unit_need = need;
  a.n_cand = two ? reinterpret_cast<const int32_t*>(ws + H.ncand) : nullptr;
  a.w2_next = two ? reinterpret_cast<const float*>(ws + H.w2n) : nullptr;
  a.sbound = two ? reinterpret_cast<const float*>(nd + NL.sbound) : nullptr;
  if ((st = from_cuda(ssa::launch_hier_probe(p, a, c))) != SSA_OK) return st;
  if (!hp.escalate) return SSA_OK;
  if (tiled) {   // the units holding an uncertified row, over all their visible blocks
    CUtensorMap tmT;
    if (!encode_2d(&tmT, table, kf, static_cast<uint64_t>(bgs) * summary_rows(p), 128)) return SSA_ERR_CUDA;
    return from_cuda(ssa::launch_route_tiled(p, tmF, tmT, idx, nullptr, c, need));
  }
  return from_cuda(ssa::launch_route_rowwise_bf16(p, Q, table, idx, nullptr, c, cert));
}

}  // namespace

namespace ssa {
size_t route_min_workspace(const ssa_params& p) { return check_params(&p) == SSA_OK ? features_bytes(p) : 0; }
}  // namespace ssa

extern "C" {

const char* ssa_status_string(int32_t s) {
  switch (s) {
    case SSA_OK: return "SSA_OK";
    case SSA_ERR_INVALID_ARG: return "SSA_ERR_INVALID_ARG";
    case SSA_ERR_UNSUPPORTED: return "SSA_ERR_UNSUPPORTED";
    case SSA_ERR_WORKSPACE: return "SSA_ERR_WORKSPACE";
    case SSA_ERR_CUDA: return "SSA_ERR_CUDA";
    case SSA_ERR_DEVICE: return "SSA_ERR_DEVICE";
  }
  return "SSA_ERR_UNKNOWN";
}

int32_t ssa_version(void) { return 1000; }

uint64_t ssa_launch_count(void) { return ssa::g_launches.load(std::memory_order_relaxed); }

ssa_status ssa_device_error(uint32_t* code) {
  if (!code) return SSA_ERR_INVALID_ARG;
  *code = 0;
  if (cudaDeviceSynchronize() != cudaSuccess) return SSA_ERR_CUDA;
  uint32_t v = 0;
  if (cudaMemcpyFromSymbol(&v, g_ssa_device_error, sizeof(v)) != cudaSuccess) return SSA_ERR_CUDA;
  const uint32_t zero = 0;
  if (cudaMemcpyToSymbol(g_ssa_device_error, &zero, sizeof(zero)) != cudaSuccess) return SSA_ERR_CUDA;
  *code = v;
  return v ? SSA_ERR_DEVICE : SSA_OK;
}

ssa_status ssa_block_summary(const ssa_params* pp, const void* K, float* mu, float* sigma,
                             void* route_table, void* stream) {
  ssa_status st = check_params(pp);
  if (st != SSA_OK) return st;
  const ssa_params& p = *pp;
  if (p.dtype == SSA_F32 && route_table) return SSA_ERR_INVALID_ARG;
  if (p.batch == 0 || p.n_kv == 0) return SSA_OK;
  if (!K || !aligned16(K) || !aligned16(mu) || !aligned16(sigma) || !aligned16(route_table))
    return SSA_ERR_INVALID_ARG;
  LaunchCtx c;
  if ((st = make_ctx(stream, c)) != SSA_OK) return st;
  return do_summary(p, K, mu, sigma, route_table, c);
}

size_t ssa_route_workspace_size(const ssa_params* p) {
  if (check_params(p) != SSA_OK) return 0;
  return route_ws_bytes(*p);
}

ssa_status ssa_route_topk(const ssa_params* pp, const void* Q, const float* mu, const float* sigma,
                          const void* route_table, int32_t* block_idx, float* top_scores, void* ws,
                          size_t ws_bytes, void* stream) {
  ssa_status st = check_params(pp);
  if (st != SSA_OK) return st;
  const ssa_params& p = *pp;
  if (is_empty(p)) return SSA_OK;
  if (!Q || !block_idx || !aligned16(Q) || !aligned16(block_idx) || !aligned16(top_scores))
    return SSA_ERR_INVALID_ARG;
  if (p.dtype == SSA_F32 && (!mu || !sigma || !aligned16(mu) || !aligned16(sigma))) return SSA_ERR_INVALID_ARG;
  if (p.dtype == SSA_BF16 && (!route_table || !aligned16(route_table))) return SSA_ERR_INVALID_ARG;
  LaunchCtx c;
  if ((st = make_ctx(stream, c)) != SSA_OK) return st;
  return do_route(p, Q, mu, sigma, route_table, block_idx, top_scores, ws, ws_bytes, c);
}

size_t ssa_attn_workspace_size(const ssa_params* p) {
  if (check_params(p) != SSA_OK) return 0;
  return attn_layout(*p).total;
}

ssa_status ssa_sparse_attn(const ssa_params* pp, const void* Q, const void* K, const void* V,
                           const int32_t* block_idx, void* O, float* lse, int32_t* bad_index_count,
                           void* ws, size_t ws_bytes, void* stream) {
  ssa_status st = check_params(pp);
  if (st != SSA_OK) return st;
  const ssa_params& p = *pp;
  if (is_empty(p)) return SSA_OK;
  if (!Q || !K || !V || !block_idx || !O) return SSA_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(block_idx) || !aligned16(O) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u) || (reinterpret_cast<uintptr_t>(bad_index_count) & 3u))
    return SSA_ERR_INVALID_ARG;
  LaunchCtx c;
  if ((st = make_ctx(stream, c)) != SSA_OK) return st;
  return do_attn(p, Q, K, V, block_idx, O, lse, bad_index_count, ws, ws_bytes, c);
}

// Common checks of the three block-major stage calls.
ssa_status check_stage(const ssa_params* pp, const void* ws, size_t ws_bytes) {
  ssa_status st = check_params(pp);
  if (st != SSA_OK) return st;
  if (is_empty(*pp)) return SSA_OK;
  const AttnLayout L = attn_layout(*pp);
  if (L.total == 0) return SSA_ERR_UNSUPPORTED;
  if (!ws || ws_bytes < L.total || !aligned16(ws)) return SSA_ERR_WORKSPACE;
  return SSA_OK;
}

ssa_status ssa_attn_plan(const ssa_params* pp, const int32_t* block_idx, void* ws, size_t ws_bytes, void* stream) {
  ssa_status st = check_stage(pp, ws, ws_bytes);
  if (st != SSA_OK || is_empty(*pp)) return st;
  if (!block_idx || !aligned16(block_idx)) return SSA_ERR_INVALID_ARG;
  LaunchCtx c;
  if ((st = make_ctx(stream, c)) != SSA_OK) return st;
  return attn_stage_plan(*pp, block_idx, static_cast<uint8_t*>(ws), c);
}

ssa_status ssa_attn_blocks(const ssa_params* pp, const void* Q, const void* K, const void* V, void* ws,
                           size_t ws_bytes, void* stream) {
  ssa_status st = check_stage(pp, ws, ws_bytes);
  if (st != SSA_OK || is_empty(*pp)) return st;
  if (!Q || !K || !V || !aligned16(Q) || !aligned16(K) || !aligned16(V)) return SSA_ERR_INVALID_ARG;
  LaunchCtx c;
  if ((st = make_ctx(stream, c)) != SSA_OK) return st;
  AttnMaps m;
  if (!encode_attn_maps(m, *pp, Q, K, V)) return SSA_ERR_CUDA;
  return attn_stage_blocks(*pp, Q, m, static_cast<uint8_t*>(ws), c);
}

ssa_status ssa_attn_window(const ssa_params* pp, const void* Q, const void* K, const void* V, void* ws,
                           size_t ws_bytes, void* stream) {
  ssa_status st = check_stage(pp, ws, ws_bytes);
  if (st != SSA_OK || is_empty(*pp)) return st;
  if (!Q || !K || !V || !aligned16(Q) || !aligned16(K) || !aligned16(V)) return SSA_ERR_INVALID_ARG;
  LaunchCtx c;
  if ((st = make_ctx(stream, c)) != SSA_OK) return st;
  AttnMaps m;
  if (!encode_attn_maps(m, *pp, Q, K, V)) return SSA_ERR_CUDA;
  return attn_stage_window(*pp, m, static_cast<uint8_t*>(ws), c);
}

ssa_status ssa_attn_merge(const ssa_params* pp, const int32_t* block_idx, void* O, float* lse,
                          int32_t* bad_index_count, const void* ws, size_t ws_bytes, void* stream) {
  ssa_status st = check_stage(pp, ws, ws_bytes);
  if (st != SSA_OK || is_empty(*pp)) return st;
  if (!block_idx || !O || !aligned16(block_idx) || !aligned16(O) || (reinterpret_cast<uintptr_t>(lse) & 3u) ||
      (reinterpret_cast<uintptr_t>(bad_index_count) & 3u))
    return SSA_ERR_INVALID_ARG;
  LaunchCtx c;
  if ((st = make_ctx(stream, c)) != SSA_OK) return st;
  return attn_stage_merge(*pp, block_idx, O, lse, bad_index_count, static_cast<const uint8_t*>(ws), c);
}

size_t ssa_workspace_size(const ssa_params* p) {
  if (check_params(p) != SSA_OK) return 0;
  return forward_layout(*p).total;
}

ssa_status ssa_forward(const ssa_params* pp, const void* Q, const void* K, const void* V, void* O,
                       float* lse, void* ws, size_t ws_bytes, void* stream) {
  ssa_status st = check_params(pp);
  if (st != SSA_OK) return st;
  const ssa_params& p = *pp;
  if (is_empty(p)) return SSA_OK;
  if (!Q || !K || !V || !O || !aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) ||
      (reinterpret_cast<uintptr_t>(lse) & 3u))
    return SSA_ERR_INVALID_ARG;
  LaunchCtx c;
  if ((st = make_ctx(stream, c)) != SSA_OK) return st;
  return forward_impl(p, Q, K, V, O, lse, static_cast<uint8_t*>(ws), ws_bytes, c);
}

size_t ssa_hostio_buffer_size(const ssa_params* p) {
  if (check_params(p) != SSA_OK) return 0;
  return hostio_layout(*p).total;
}

ssa_status ssa_forward_hostio(const ssa_params* pp, const void* hQ, const void* hK, const void* hV,
                              void* hO, float* hlse, void* dev_buf, size_t dev_bytes, void* stream) {
  ssa_status st = check_params(pp);
  if (st != SSA_OK) return st;
  const ssa_params& p = *pp;
  if (is_empty(p)) return SSA_OK;
  if (!hQ || !hK || !hV || !hO) return SSA_ERR_INVALID_ARG;
  const HostioLayout L = hostio_layout(p);
  if (!dev_buf || dev_bytes < L.total || !aligned16(dev_buf)) return SSA_ERR_WORKSPACE;
  LaunchCtx c;
  if ((st = make_ctx(stream, c)) != SSA_OK) return st;
  uint8_t* d = static_cast<uint8_t*>(dev_buf);
  const size_t es = esize(p);
  const size_t qb = static_cast<size_t>(p.batch) * p.n_q * p.h_q * p.d * es;
  const size_t kb = static_cast<size_t>(p.batch) * p.n_kv * p.h_kv * p.d * es;
  const size_t lb = static_cast<size_t>(p.batch) * p.n_q * p.h_q * 4;
  if (cudaMemcpyAsync(d + L.q, hQ, qb, cudaMemcpyHostToDevice, c.stream) != cudaSuccess ||
      cudaMemcpyAsync(d + L.k, hK, kb, cudaMemcpyHostToDevice, c.stream) != cudaSuccess ||
      cudaMemcpyAsync(d + L.v, hV, kb, cudaMemcpyHostToDevice, c.stream) != cudaSuccess)
    return SSA_ERR_CUDA;
  st = forward_impl(p, d + L.q, d + L.k, d + L.v, d + L.o, reinterpret_cast<float*>(d + L.lse), d + L.ws,
                    L.total - L.ws, c);
  if (st != SSA_OK) return st;
  if (cudaMemcpyAsync(hO, d + L.o, qb, cudaMemcpyDeviceToHost, c.stream) != cudaSuccess) return SSA_ERR_CUDA;
  if (hlse && cudaMemcpyAsync(hlse, d + L.lse, lb, cudaMemcpyDeviceToHost, c.stream) != cudaSuccess)
    return SSA_ERR_CUDA;
  return SSA_OK;
}

size_t ssa_hier_nodes_size(const ssa_params* p, const ssa_hier_params* hp) {
  if (check_hier(p, hp) != SSA_OK) return 0;
  return hier_node_layout(*p, *hp).total;
}

ssa_status ssa_hier_nodes(const ssa_params* pp, const ssa_hier_params* hp, const void* route_table, void* nodes,
                          void* stream) {
  ssa_status st = check_hier(pp, hp);
  if (st != SSA_OK) return st;
  const ssa_params& p = *pp;
  if (p.batch == 0) return SSA_OK;
  if (!route_table || !nodes || !aligned16(route_table) || !aligned16(nodes)) return SSA_ERR_INVALID_ARG;
  LaunchCtx c;
  if ((st = make_ctx(stream, c)) != SSA_OK) return st;
  const HierNodeLayout L = hier_node_layout(p, *hp);
  uint8_t* nd = static_cast<uint8_t*>(nodes);
  const int64_t bgs = static_cast<int64_t>(p.batch) * p.h_kv;
  if (cudaMemsetAsync(nd + L.bound, 0, static_cast<size_t>(bgs) * 2 * 4, c.stream) != cudaSuccess)
    return SSA_ERR_CUDA;
  if (hier_levels(*hp) == 2 && cudaMemsetAsync(nd + L.sbound, 0, static_cast<size_t>(bgs) * 4, c.stream) != cudaSuccess)
    return SSA_ERR_CUDA;
  ssa::HierNodeArgs a;
  a.bgs = static_cast<int32_t>(bgs);
  a.nb = static_cast<int32_t>(nb_of(p));
  a.nn = static_cast<int32_t>(L.nn);
  a.M = hp->fanout;
  a.T = static_cast<const __nv_bfloat16*>(route_table);
  a.NT = reinterpret_cast<__nv_bfloat16*>(nd + L.table);
  a.radius = reinterpret_cast<float*>(nd + L.radius);
  a.bound = reinterpret_cast<uint32_t*>(nd + L.bound);
  if ((st = from_cuda(ssa::launch_hier_nodes(p, a, c))) != SSA_OK || hier_levels(*hp) != 2) return st;
  ssa::HierSuperArgs s2;
  s2.bgs = static_cast<int32_t>(bgs);
  s2.nn = static_cast<int32_t>(L.nn);
  s2.ns = static_cast<int32_t>(L.ns);
  s2.M = hp->fanout;
  s2.NT = reinterpret_cast<const __nv_bfloat16*>(nd + L.table);
  s2.radius = reinterpret_cast<const float*>(nd + L.radius);
  s2.ST = reinterpret_cast<__nv_bfloat16*>(nd + L.stable);
  s2.sradius = reinterpret_cast<float*>(nd + L.sradius);
  s2.sbound = reinterpret_cast<uint32_t*>(nd + L.sbound);
  s2.bound = reinterpret_cast<uint32_t*>(nd + L.bound);
  return from_cuda(ssa::launch_hier_supers(p, s2, c));
}

size_t ssa_route_hier_workspace_size(const ssa_params* p, const ssa_hier_params* hp) {
  if (check_hier(p, hp) != SSA_OK) return 0;
  return hier_layout(*p, *hp).total;
}

ssa_status ssa_route_hier(const ssa_params* pp, const ssa_hier_params* hp, const void* Q, const void* route_table,
                          const void* nodes, int32_t* block_idx, uint8_t* certified, void* ws, size_t ws_bytes,
                          void* stream) {
  ssa_status st = check_hier(pp, hp);
  if (st != SSA_OK) return st;
  const ssa_params& p = *pp;
  if (is_empty(p)) return SSA_OK;
  if (!Q || !route_table || !nodes || !block_idx || !aligned16(Q) || !aligned16(route_table) ||
      !aligned16(nodes) || !aligned16(block_idx))
    return SSA_ERR_INVALID_ARG;
  const HierLayout H = hier_layout(p, *hp);
  if (!ws || ws_bytes < H.total || !aligned16(ws)) return SSA_ERR_WORKSPACE;
  LaunchCtx c;
  if ((st = make_ctx(stream, c)) != SSA_OK) return st;
  return do_route_hier(p, *hp, Q, route_table, nodes, block_idx, certified, static_cast<uint8_t*>(ws), c);
}

ssa_status ssa_selftest_wait_timeout(void* stream) {
  LaunchCtx c;
  ssa_status st = make_ctx(stream, c);
  if (st != SSA_OK) return st;
  return from_cuda(ssa::launch_selftest_wait(c));
}

}  // extern "C"

// ssa_route_topk_static: the router with its scratch in a fixed device array.
//
// The tiled router needs scratch memory for the routing-feature rows it
// multiplies on the tensor cores.  ssa_route_topk takes that scratch from a
// caller-provided workspace.  This entry point is for callers that cannot
// hand out device memory at that point: code embedded in a host framework
// whose allocator owns the whole device pool (a raw cudaMalloc would fail or
// fragment it), or latency-sensitive loops where cudaMalloc's implicit device
// synchronisation is not acceptable.  Here the scratch is a file-scope device
// array of fixed size that exists on every GPU that loads the library, so the
// call allocates nothing.
//
// Behaviour:
//  * the array holds SSA_ROUTE_STATIC_SCRATCH_BYTES; a problem whose feature
//    rows need more is rejected with SSA_ERR_WORKSPACE before any launch;
//  * the first call on each device looks up the array's device address
//    (cudaGetSymbolAddress) with that device current, and caches it; make
//    that first call before any stream capture on the device;
//  * all calls share the one array and it keeps the last call's contents.
//    Nothing in it needs to start at zero (every call overwrites the rows it
//    reads), but two calls whose kernels overlap on the GPU (different
//    streams, or different host threads) race on it; serialise them;
//  * no cudaMalloc, cudaFree or allocating library routine is called.
#include <cuda_runtime.h>

#include <mutex>

#include "kernels.h"
#include "ssa.h"

namespace {

static __device__ __align__(256) unsigned char g_route_scratch[SSA_ROUTE_STATIC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (looked up once).
ssa_status scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SSA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_route_scratch) != cudaSuccess || !ptr) return SSA_ERR_CUDA;
    g_scratch_ptr[dev] = ptr;
  }
  *out = g_scratch_ptr[dev];
  return SSA_OK;
}

}  // namespace

extern "C" ssa_status ssa_route_topk_static(const ssa_params* p, const void* Q, const float* mu,
                                            const float* sigma, const void* route_table,
                                            int32_t* block_idx, float* top_scores, void* stream) {
  if (!p) return SSA_ERR_INVALID_ARG;
  // the feature rows must fit; the router's seed arrays are used when they
  // fit beside them
  const size_t need = ssa::route_min_workspace(*p);
  if (need > SSA_ROUTE_STATIC_SCRATCH_BYTES) return SSA_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (need > 0) {
    const ssa_status st = scratch_for_current_device(&scratch);
    if (st != SSA_OK) return st;
  }
  return ssa_route_topk(p, Q, mu, sigma, route_table, block_idx, top_scores, scratch,
                        need > 0 ? static_cast<size_t>(SSA_ROUTE_STATIC_SCRATCH_BYTES) : 0, stream);
}

// moe_dispatch_noalloc: the pack step for callers that cannot hand the library any
// scratch memory.
//
// Some callers cannot obtain device memory at the moment they need to pack tokens: code
// running inside a framework that owns every device allocation (a plugin handed only its
// input and output buffers), runtimes with a fixed memory budget decided before start-up,
// or hosts that must not call an allocator on their hot path (allocation can synchronise
// the device or take a global lock).  This variant therefore keeps its only scratch, the
// per-token-tile expert histogram, in a fixed array in the library's own device memory
// and takes no workspace argument.  The caller still passes inputs and outputs.
#include <mutex>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

// Largest histogram this entry point handles: num_tiles(T, E) * E int32 entries.  The
// array lives in every device that loads the library, until the process exits.
constexpr int kNoAllocHistEntries = 16384;  // 64 KiB
static __device__ __align__(256) int32_t g_noalloc_hist[kNoAllocHistEntries];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
int32_t* g_hist_ptr[kMaxDevices] = {};

// Device address of g_noalloc_hist on the current device.  In host code the symbol
// names a host-side stand-in, not device memory, so the address must be looked up, once
// per device, with that device current.
cudaError_t hist_address(int32_t** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_hist_ptr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_hist);
    if (e != cudaSuccess) return e;
    g_hist_ptr[dev] = static_cast<int32_t*>(p);
  }
  *out = g_hist_ptr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace moe

using namespace moe;

extern "C" moe_status moe_dispatch_noalloc(const moe_config* cfg, const void* x,
                                           const int32_t* ids, void* x_packed,
                                           int32_t* row_token, int32_t* route_row,
                                           int32_t* offsets, int32_t* demand, int32_t* status,
                                           moe_stream_t stream) {
  // Same argument checks as moe_dispatch (validation lives in api.cu; repeated here in
  // short form so this file stays independent of the workspace layout).
  if (cfg == nullptr || cfg->T < 1 || cfg->d < 1 || cfg->E < 1 || cfg->k < 1 || cfg->k > cfg->E ||
      (cfg->dtype != MOE_F32 && cfg->dtype != MOE_BF16))
    return MOE_ERR_INVALID;
  if ((cfg->layout != MOE_LAYOUT_RAGGED && cfg->layout != MOE_LAYOUT_PADDED) ||
      (cfg->overflow != MOE_OVERFLOW_DROP && cfg->overflow != MOE_OVERFLOW_REROUTE) ||
      (cfg->layout == MOE_LAYOUT_PADDED && cfg->capacity < 0))
    return MOE_ERR_INVALID;
  // The reroute policy ranks with the router's logits, which live in a workspace.
  if (cfg->overflow == MOE_OVERFLOW_REROUTE) return MOE_ERR_UNSUPPORTED;
  if (cfg->E > 256 || cfg->k > 32 || cfg->T > (1 << 24)) return MOE_ERR_UNSUPPORTED;
  if (static_cast<long long>(cfg->T) * cfg->k > (1 << 30) ||
      (cfg->layout == MOE_LAYOUT_PADDED && static_cast<long long>(cfg->E) * cfg->capacity > (1 << 30)))
    return MOE_ERR_UNSUPPORTED;
  if ((cfg->dtype == MOE_BF16 && cfg->d % 128 != 0) || (cfg->dtype == MOE_F32 && cfg->d % 4 != 0))
    return MOE_ERR_UNSUPPORTED;
  if (!x || !ids || !x_packed || !row_token || !route_row || !offsets || !demand)
    return MOE_ERR_INVALID;
  // The histogram must fit the fixed array.
  if (static_cast<long long>(num_tiles_for(cfg->T, cfg->E)) * cfg->E > kNoAllocHistEntries)
    return MOE_ERR_UNSUPPORTED;
  int32_t* hist = nullptr;
  if (hist_address(&hist) != cudaSuccess) return MOE_ERR_CUDA;
  // Nothing in the array has to start at zero: the histogram kernel writes every entry
  // that the scatter kernel reads.
  if (launch_dispatch_hist(*cfg, ids, hist, status, stream) != cudaSuccess) return MOE_ERR_CUDA;
  if (launch_dispatch_scatter(*cfg, x, ids, hist, x_packed, row_token, route_row, offsets,
                              demand, status, stream) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

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
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

// Largest histogram this entry point handles: num_tiles(T, E) * E int32 entries.  The
// array holds the histogram and, after it, the ticket counter of the dispatch prep; it
// lives in every device that loads the library, until the process exits.
constexpr int kNoAllocHistEntries = 16384;  // 64 KiB
constexpr int kNoAllocTicket = kNoAllocHistEntries;  // one more 256-byte-aligned slot
static __device__ __align__(256) int32_t g_noalloc_hist[kNoAllocHistEntries + 64];

// Device address of g_noalloc_hist in the current device's context.  In host code the
// symbol names a host-side stand-in, not device memory, so the address is looked up with
// the device current.  The lookup is a host-side query that enqueues no work; it is made
// on every call rather than cached, because the address belongs to the context that
// loaded the module: after cudaDeviceReset, or under another context on the same device,
// an address kept from an earlier call would point at memory that is no longer ours.
cudaError_t hist_address(int32_t** out) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_hist);
  if (e != cudaSuccess) return e;
  *out = static_cast<int32_t*>(p);
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
  // The checks every entry point applies, then the two limits of this one.
  const moe_status v = validate_config(cfg);
  if (v != MOE_OK) return v;
  // The reroute policy ranks with the router's logits, which live in a workspace.
  if (cfg->overflow == MOE_OVERFLOW_REROUTE) return MOE_ERR_UNSUPPORTED;
  if (!x || !ids || !x_packed || !row_token || !route_row || !offsets || !demand)
    return MOE_ERR_INVALID;
  // The histogram must fit the fixed array.
  if (static_cast<long long>(num_tiles_for(cfg->T, cfg->E)) * cfg->E > kNoAllocHistEntries)
    return MOE_ERR_UNSUPPORTED;
  int32_t* hist = nullptr;
  if (hist_address(&hist) != cudaSuccess) return MOE_ERR_CUDA;
  // The histogram kernel writes every histogram entry the pack reads; only the ticket has
  // to start at zero.  It is cleared here (the prep also leaves it zero), so a call never
  // depends on what an earlier one left behind.
  unsigned int* ticket = reinterpret_cast<unsigned int*>(hist + kNoAllocTicket);
  if (cudaMemsetAsync(ticket, 0, sizeof(unsigned int), stream) != cudaSuccess) return MOE_ERR_CUDA;
  const DispatchPrep prep = make_dispatch_prep(*cfg, hist, offsets, demand, ticket);
  if (launch_dispatch_hist(*cfg, ids, prep, status, stream) != cudaSuccess) return MOE_ERR_CUDA;
  if (launch_dispatch_pack(*cfg, x, ids, hist, offsets, x_packed, row_token, route_row, status,
                           stream) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

// Host-side declarations shared by the libmoe translation units.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "moe.h"

namespace moe {

// Host-side validation of a config: MOE_OK, MOE_ERR_INVALID or MOE_ERR_UNSUPPORTED (the
// same checks every entry point that takes a config applies before any launch).
moe_status validate_config(const moe_config* c);

// Token tile of the expert histogram that connects routing and packing: 128 tokens, the
// router's CTA tile (one TMEM lane per token).  The histogram is num_tiles x E int32.
constexpr int kHistTile = 128;
inline int tok_tile_for(int /*T*/, int /*E*/) { return kHistTile; }
inline int num_tiles_for(int T, int /*E*/) { return (T + kHistTile - 1) / kHistTile; }

// Optional router outputs (null: not written).
struct RouterExtras {
  float* tile_psum;  // [num_tiles, E] fp32: per token tile, the sum of every token's full
                     // softmax (routing statistics)
  float* zkeys;      // [T, E] fp32: the ranking keys (logit + bias, NaN as -inf) that
                     // top-k compared (the reroute policy ranks with them)
};

cudaError_t launch_router(const moe_config& c, const void* x, const void* w_router,
                          const float* bias, int32_t* ids, float* gates, int32_t* tile_hist,
                          const RouterExtras& extra, int32_t* status, cudaStream_t s);

// bf16 router on tensor cores (route_sm100.cu); the fp32 router runs on CUDA cores.
cudaError_t launch_router_sm100(const moe_config& c, const void* x, const void* w_router,
                                const float* bias, int32_t* ids, float* gates,
                                int32_t* tile_hist, const RouterExtras& extra,
                                int32_t* status, cudaStream_t s);

// Routing statistics from the per-tile probability sums and the dispatch counts.
// partial: [kStatsMaxBlocks, E] fp64 scratch; counter: zero before the call, left zero.
constexpr int kStatsMaxBlocks = 148;
// Kept routes: offsets[E] with the ragged layout, the sum of the filled-slot counts
// offsets[E+2 ..] with the padded one.
cudaError_t launch_routing_stats(const moe_config& c, const float* tile_psum,
                                 const int32_t* demand, const int32_t* offsets, float alpha,
                                 double* partial, unsigned int* counter, float* f, float* P,
                                 moe_routing_summary* out, cudaStream_t s);

// Reroute overflow policy on the padded buffer, after the arrival-order pack:
// places the overflowed routes (one CTA, in phases equivalent to the arrival-order walk),
// rewrites route_row, row_token, the filled-slot counts (offsets[E+2+e]) and the gates of
// tokens with a moved route, then copies the moved routes' token rows.
// scratch: [2 * E * C + 1 + 4 * T * k] int32.
cudaError_t launch_reroute(const moe_config& c, const void* x, const int32_t* ids,
                           const float* zkeys, float* gates, void* x_packed, int32_t* row_token,
                           int32_t* route_row, int32_t* offsets, int32_t* scratch,
                           int32_t* status, cudaStream_t s);

cudaError_t launch_dispatch_hist(const moe_config& c, const int32_t* ids, int32_t* tile_hist,
                                 int32_t* status, cudaStream_t s);

cudaError_t launch_dispatch_scatter(const moe_config& c, const void* x, const int32_t* ids,
                                    const int32_t* tile_hist, void* x_packed,
                                    int32_t* row_token, int32_t* route_row, int32_t* offsets,
                                    int32_t* demand, int32_t* status, cudaStream_t s);

cudaError_t launch_combine(const moe_config& c, const void* y_packed, const int32_t* route_row,
                           const float* gates, const int32_t* offsets, const void* residual,
                           void* y, cudaStream_t s);

struct FfnArgs {
  const void* x;          // [T, d] (shared expert's A operand)
  const void* x_packed;   // [Rmax, d]
  const int32_t* offsets; // [E + 2]
  const void* w_gate;     // [E, F, d]
  const void* w_up;       // [E, F, d]
  const void* w_down;     // [E, d, F]
  const void* s_gate;     // [F, d] or null
  const void* s_up;       // [F, d] or null
  const void* s_down;     // [d, F] or null
  void* h;                // [Rmax (+T), F]
  void* y_packed;         // [Rmax (+T), d]
  int64_t rmax;           // rows of x_packed
  int32_t* status;
  const int32_t* counts;  // [E] rows of each routed segment (padded layout), or null:
                          // rows = offsets[s + 1] - offsets[s]
};

// fp32 path: CUDA-core grouped GEMMs.  `mid` (may be null) is recorded between the
// gate/up and the down GEMM.
cudaError_t launch_ffn_simt(const moe_config& c, const FfnArgs& a, cudaStream_t s,
                            cudaEvent_t mid = nullptr);
// bf16 path: persistent tcgen05/TMEM grouped GEMMs fed by TMA.
cudaError_t launch_ffn_sm100(const moe_config& c, const FfnArgs& a, cudaStream_t s,
                             cudaEvent_t mid = nullptr);

cudaError_t launch_debug_wait(int32_t* status, int64_t limit_ns, cudaStream_t s);

// Default bound on every in-kernel wait (nanoseconds).
constexpr int64_t kWaitLimitNs = 2000000000LL;

}  // namespace moe

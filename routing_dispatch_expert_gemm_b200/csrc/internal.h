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

// What the CTA that writes the last tile of the expert histogram computes for the pack
// (dispatch_prep.cuh): per-tile exclusive prefixes in place of the counts, demand, the
// segment table (offsets, [E + 2] or [2E + 2] padded) and the filled-slot counts.
// `ticket` must be zero before the launch; it is left zero.  A null ticket: not computed.
struct DispatchPrep {
  int32_t* tile_hist;
  int32_t* offsets;
  int32_t* demand;
  unsigned int* ticket;
  int num_tiles, E, T, capacity, has_shared, padded;
};
DispatchPrep make_dispatch_prep(const moe_config& c, int32_t* tile_hist, int32_t* offsets,
                                int32_t* demand, unsigned int* ticket);

// Router: ids, gates and the per-tile expert histogram; with a non-null prep.ticket also
// the dispatch prep above (moe_forward passes one; moe_route does not).
cudaError_t launch_router(const moe_config& c, const void* x, const void* w_router,
                          const float* bias, int32_t* ids, float* gates, int32_t* tile_hist,
                          const RouterExtras& extra, const DispatchPrep& prep, int32_t* status,
                          cudaStream_t s);

// bf16 router on tensor cores (route_sm100.cu); the fp32 router runs on CUDA cores.
cudaError_t launch_router_sm100(const moe_config& c, const void* x, const void* w_router,
                                const float* bias, int32_t* ids, float* gates,
                                int32_t* tile_hist, const RouterExtras& extra,
                                const DispatchPrep& prep, int32_t* status, cudaStream_t s);

// Routing statistics from the per-tile probability sums and the dispatch counts.
// partial: [kStatsMaxBlocks, E] fp64 scratch; counter: zero before the call, left zero.
constexpr int kStatsMaxBlocks = 148;
// Kept routes: offsets[E] with the ragged layout, the sum of the filled-slot counts
// offsets[E+2 ..] with the padded one.
cudaError_t launch_routing_stats(const moe_config& c, const float* tile_psum,
                                 const int32_t* demand, const int32_t* offsets, float alpha,
                                 double* partial, unsigned int* counter, float* f, float* P,
                                 moe_routing_summary* out, cudaStream_t s);

// Reroute overflow policy on the padded buffer, after the arrival-order pack: ranks each
// overflowing token's experts (grid-wide), places the overflowed routes (one CTA, in phases
// equivalent to the arrival-order walk), rewrites route_row, row_token, the filled-slot
// counts (offsets[E+2+e]) and the gates of tokens with a moved route, then copies the moved
// routes' token rows.  scratch: reroute_scratch_bytes(c) bytes, 16-byte aligned.
size_t reroute_scratch_bytes(const moe_config& c);
cudaError_t launch_reroute(const moe_config& c, const void* x, const int32_t* ids,
                           const float* zkeys, float* gates, void* x_packed, int32_t* row_token,
                           int32_t* route_row, int32_t* offsets, int32_t* scratch,
                           int32_t* status, cudaStream_t s);

// Expert histogram of caller-given ids per 128-token tile (invalid ids are flagged and not
// counted), followed by the dispatch prep in the last CTA.
cudaError_t launch_dispatch_hist(const moe_config& c, const int32_t* ids,
                                 const DispatchPrep& prep, int32_t* status, cudaStream_t s);

// Pack: route_row, row_token and the packed rows, from the ids and the prep's prefixes and
// segment table (one warp per token).  With `fused` (moe_forward's fused steps): no row
// copy when the GEMM gathers (fused->copy == 0); with the fused combine, need[t] and the
// zeroed counters, and y[t] for tokens with no contribution at all.
struct PackFusion {
  int copy;               // 1: write x_packed
  int32_t* need;          // [T] or null
  int32_t* counters;      // [T, d / 32] or null
  const void* residual;   // x or null
  void* y;                // y (tokens with need 0) or null
  int has_shared;
};
cudaError_t launch_dispatch_pack(const moe_config& c, const void* x, const int32_t* ids,
                                 const int32_t* tile_prefix, const int32_t* offsets,
                                 void* x_packed, int32_t* row_token, int32_t* route_row,
                                 int32_t* status, cudaStream_t s,
                                 const PackFusion* fused = nullptr);

cudaError_t launch_combine(const moe_config& c, const void* y_packed, const int32_t* route_row,
                           const float* gates, const int32_t* offsets, const void* residual,
                           void* y, cudaStream_t s);

// The combine done in the down GEMM's epilogue (MOE_FUSE_COMBINE): every tile that writes
// 32 columns of a packed row counts itself on the token's counter for that column chunk;
// the one that brings it to need[t] (kept routes + shared expert) sums the token's rows
// of y_packed for those columns in slot order and writes them to y.
struct FusedCombine {
  const int32_t* route_row;  // [T, k]
  const float* gates;        // [T, k]
  const int32_t* row_token;  // [Rmax] token of each packed row
  const int32_t* need;       // [T] contributions per token (pack writes it)
  int32_t* counters;         // [T, d / 32], zeroed by the pack
  const void* residual;      // x [T, d] or null
  void* y;                   // [T, d]
  int k, has_shared;
};

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
  // Fused steps (column tiles only; null: not fused).
  const int32_t* gather_rows;  // row_token [Rmax]: the gate/up GEMM reads x[row_token[r]]
                               // instead of x_packed[r]
  const FusedCombine* combine; // the down GEMM's epilogue finishes the output rows
};

// fp32 path: CUDA-core grouped GEMMs.  `mid` (may be null) is recorded between the
// gate/up and the down GEMM.
cudaError_t launch_ffn_simt(const moe_config& c, const FfnArgs& a, cudaStream_t s,
                            cudaEvent_t mid = nullptr);
// bf16 path: persistent tcgen05/TMEM grouped GEMMs fed by TMA.  Chooses the tile shape:
// row tiles (tokens on the MMA's M side, gemm_sm100.cu) for large expert segments, column
// tiles (weights on M, tokens on N, gemm_cols_sm100.cu) for small ones.
cudaError_t launch_ffn_sm100(const moe_config& c, const FfnArgs& a, cudaStream_t s,
                             cudaEvent_t mid = nullptr);
// MOE_TILES_ROWS or MOE_TILES_COLUMNS: cfg.tiles, or the automatic choice.
int32_t ffn_tile_shape(const moe_config& c);
cudaError_t launch_ffn_cols_sm100(const moe_config& c, const FfnArgs& a, cudaStream_t s,
                                  cudaEvent_t mid = nullptr);
// Column tiles over SM pairs (gemm_pair_sm100.cu); d and d_ff multiples of 256.
cudaError_t launch_ffn_pair_sm100(const moe_config& c, const FfnArgs& a, cudaStream_t s,
                                  cudaEvent_t mid = nullptr);
// Row tiles over SM pairs (gemm_rowpair_sm100.cu); d a multiple of 256, d_ff of 128.
cudaError_t launch_ffn_rowpair_sm100(const moe_config& c, const FfnArgs& a, cudaStream_t s,
                                     cudaEvent_t mid = nullptr);
// One of its GEMMs over a subset of the segments: the routed ones and/or the shared expert's.
cudaError_t launch_rowpair_gate_up(const moe_config& c, const FfnArgs& a, cudaStream_t s,
                                   bool routed, bool shared);
cudaError_t launch_rowpair_down(const moe_config& c, const FfnArgs& a, cudaStream_t s,
                                bool routed, bool shared);
// Whether the automatic tile choice runs the shared expert's segment on row tiles over SM
// pairs, in launches of its own, next to row tiles for the routed segments.
bool ffn_shared_on_pairs(const moe_config& c);
// Kernel launches of the expert FFN for the config: 2, or 4 with ffn_shared_on_pairs.
int ffn_launches(const moe_config& c);

cudaError_t launch_debug_wait(int32_t* status, int64_t limit_ns, cudaStream_t s);

// Default bound on every in-kernel wait (nanoseconds).
constexpr int64_t kWaitLimitNs = 2000000000LL;

}  // namespace moe

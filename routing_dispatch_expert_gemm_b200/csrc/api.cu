// C ABI of libmoe.so: argument validation, workspace layout and launch sequencing.
// Every entry point is declared, with argument meaning, layout, ownership and error
// behaviour, in include/moe.h.
#include <algorithm>
#include <climits>
#include <cmath>

#include "common.cuh"
#include "internal.h"

using namespace moe;

namespace moe {

// Host-side checks shared by every entry point that takes a config (declared in
// internal.h).
moe_status validate_config(const moe_config* c) {
  if (c == nullptr) return MOE_ERR_INVALID;
  if (c->T < 1 || c->d < 1 || c->E < 1 || c->k < 1 || c->d_ff < 1) return MOE_ERR_INVALID;
  if (c->k > c->E) return MOE_ERR_INVALID;
  if (c->dtype != MOE_F32 && c->dtype != MOE_BF16) return MOE_ERR_INVALID;
  if (c->gate_mode < MOE_GATE_SOFTMAX_TOPK || c->gate_mode > MOE_GATE_TOPK_SOFTMAX)
    return MOE_ERR_INVALID;
  if ((c->has_shared != 0 && c->has_shared != 1) || (c->add_residual != 0 && c->add_residual != 1) ||
      (c->stats != 0 && c->stats != 1))
    return MOE_ERR_INVALID;
  if ((c->layout != MOE_LAYOUT_RAGGED && c->layout != MOE_LAYOUT_PADDED) ||
      (c->overflow != MOE_OVERFLOW_DROP && c->overflow != MOE_OVERFLOW_REROUTE))
    return MOE_ERR_INVALID;
  if (c->tiles < MOE_TILES_AUTO || c->tiles > MOE_TILES_ROW_PAIRS) return MOE_ERR_INVALID;
  if (c->fuse < 0 || c->fuse > (MOE_FUSE_GATHER | MOE_FUSE_COMBINE)) return MOE_ERR_INVALID;
  if (c->fuse != 0 && (c->tiles == MOE_TILES_ROWS || c->tiles == MOE_TILES_ROW_PAIRS))
    return MOE_ERR_INVALID;
  if (c->fuse != 0 && (c->dtype != MOE_BF16 || c->overflow != MOE_OVERFLOW_DROP))
    return MOE_ERR_UNSUPPORTED;
  if (c->layout == MOE_LAYOUT_PADDED && c->capacity < 0) return MOE_ERR_INVALID;  // C sizes it
  if (c->overflow == MOE_OVERFLOW_REROUTE && c->layout != MOE_LAYOUT_PADDED)
    return MOE_ERR_UNSUPPORTED;
  if (c->E > 256 || c->k > 32) return MOE_ERR_UNSUPPORTED;
  if (c->T > (1 << 24) || static_cast<int64_t>(c->T) * c->k > (INT_MAX / 2)) return MOE_ERR_UNSUPPORTED;
  if (c->layout == MOE_LAYOUT_PADDED && static_cast<int64_t>(c->E) * c->capacity > (INT_MAX / 2))
    return MOE_ERR_UNSUPPORTED;
  if (c->dtype == MOE_BF16) {
    if (c->d % 128 != 0 || c->d_ff % 128 != 0) return MOE_ERR_UNSUPPORTED;
  } else {
    if (c->d % 4 != 0 || c->d_ff % 4 != 0) return MOE_ERR_UNSUPPORTED;
  }
  return MOE_OK;
}

}  // namespace moe

namespace {

moe_status validate(const moe_config* c) { return validate_config(c); }

constexpr int32_t kAbiVersion = 5;

size_t align256(size_t v) { return (v + 255) & ~static_cast<size_t>(255); }

int64_t max_rows(const moe_config& c) {
  if (c.layout == MOE_LAYOUT_PADDED)
    return std::max<int64_t>(static_cast<int64_t>(c.E) * c.capacity, 1);
  int64_t r = static_cast<int64_t>(c.T) * c.k;
  if (c.capacity >= 0) r = std::min<int64_t>(r, static_cast<int64_t>(c.E) * c.capacity);
  return std::max<int64_t>(r, 1);
}

bool padded(const moe_config& c) { return c.layout == MOE_LAYOUT_PADDED; }
bool reroute(const moe_config& c) { return c.overflow == MOE_OVERFLOW_REROUTE; }
// Entries of the segment table (offsets): starts, plus the filled-slot counts when padded.
size_t offsets_len(const moe_config& c) { return c.E + 2 + (padded(c) ? c.E : 0); }

struct Layout {
  size_t tile_hist, tile_psum, stats_partial, zkeys, rlist, need, counters;
  size_t ids, gates, route_row, row_token, offsets, demand;
  size_t x_packed, h, y_packed;
  size_t scratch_end, total;
  int64_t rmax, rows_h;
};

Layout layout_of(const moe_config& c) {
  Layout L{};
  size_t off = kWsHeaderBytes;
  auto take = [&off](size_t bytes) {
    const size_t o = off;
    off = align256(off + bytes);
    return o;
  };
  const size_t esz = (c.dtype == MOE_BF16) ? 2 : 4;
  const size_t Tk = static_cast<size_t>(c.T) * c.k;
  L.rmax = max_rows(c);
  L.rows_h = L.rmax + (c.has_shared ? c.T : 0);
  L.tile_hist = take(static_cast<size_t>(num_tiles_for(c.T, c.E)) * c.E * 4);
  // Routing statistics (only with cfg.stats): per-tile probability sums and fp64 partials.
  L.tile_psum = c.stats ? take(static_cast<size_t>(num_tiles_for(c.T, c.E)) * c.E * 4) : 0;
  L.stats_partial = c.stats ? take(static_cast<size_t>(kStatsMaxBlocks) * c.E * 8) : 0;
  // Reroute policy (only with it): the router's ranking keys and the placement's scratch.
  L.zkeys = reroute(c) ? take(static_cast<size_t>(c.T) * c.E * 4) : 0;
  L.rlist = reroute(c) ? take(reroute_scratch_bytes(c)) : 0;
  // Fused combine (MOE_FUSE_COMBINE): contributions per token, counters per 32 columns.
  L.need = (c.fuse & MOE_FUSE_COMBINE) ? take(static_cast<size_t>(c.T) * 4) : 0;
  L.counters = (c.fuse & MOE_FUSE_COMBINE) ? take(static_cast<size_t>(c.T) * ((c.d + 31) / 32) * 4)
                                           : 0;
  L.scratch_end = off;
  L.ids = take(Tk * 4);
  L.gates = take(Tk * 4);
  L.route_row = take(Tk * 4);
  L.row_token = take(static_cast<size_t>(L.rmax) * 4);
  L.offsets = take(offsets_len(c) * 4);
  L.demand = take(static_cast<size_t>(c.E) * 4);
  L.x_packed = take(static_cast<size_t>(L.rmax) * c.d * esz);
  L.h = take(static_cast<size_t>(L.rows_h) * c.d_ff * esz);
  L.y_packed = take(static_cast<size_t>(L.rows_h) * c.d * esz);
  L.total = off;
  return L;
}

moe_status check_ws(const void* ws) {
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255) != 0) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

template <typename P>
uint8_t* at(P* base, size_t off) {
  return reinterpret_cast<uint8_t*>(const_cast<void*>(static_cast<const void*>(base))) + off;
}

moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

#define MOE_TRY(expr)                 \
  do {                                \
    const moe_status st_ = (expr);    \
    if (st_ != MOE_OK) return st_;    \
  } while (0)

moe_status ffn(const moe_config& c, const FfnArgs& f, cudaStream_t s, cudaEvent_t mid = nullptr) {
  return cuda_status(c.dtype == MOE_BF16 ? launch_ffn_sm100(c, f, s, mid)
                                         : launch_ffn_simt(c, f, s, mid));
}

moe_status record(void* const* events, int i, cudaStream_t s) {
  if (events == nullptr) return MOE_OK;
  return cuda_status(record_event(static_cast<cudaEvent_t>(events[i]), s));
}

moe_status forward_impl(const moe_config* cfg, const void* x, const void* w_router,
                        const float* logit_bias, const void* w_gate, const void* w_up,
                        const void* w_down, const void* shared_gate, const void* shared_up,
                        const void* shared_down, void* y, int32_t* ids_out, float* gates_out,
                        int32_t* demand_out, int32_t* offsets_out, void* const* ev, int n_ev,
                        void* ws,
                        cudaStream_t stream) {
  MOE_TRY(validate(cfg));
  MOE_TRY(check_ws(ws));
  if (!x || !w_router || !w_gate || !w_up || !w_down || !y) return MOE_ERR_INVALID;
  if (cfg->has_shared && (!shared_gate || !shared_up || !shared_down)) return MOE_ERR_INVALID;
  const moe_config& c = *cfg;
  const Layout L = layout_of(c);
  int32_t* status = static_cast<int32_t*>(ws);
  int32_t* hist = reinterpret_cast<int32_t*>(at(ws, L.tile_hist));
  const RouterExtras extra{c.stats ? reinterpret_cast<float*>(at(ws, L.tile_psum)) : nullptr,
                           reroute(c) ? reinterpret_cast<float*>(at(ws, L.zkeys)) : nullptr};
  int32_t* ids = ids_out ? ids_out : reinterpret_cast<int32_t*>(at(ws, L.ids));
  float* gates = gates_out ? gates_out : reinterpret_cast<float*>(at(ws, L.gates));
  int32_t* demand = demand_out ? demand_out : reinterpret_cast<int32_t*>(at(ws, L.demand));
  int32_t* offsets = offsets_out ? offsets_out : reinterpret_cast<int32_t*>(at(ws, L.offsets));
  int32_t* route_row = reinterpret_cast<int32_t*>(at(ws, L.route_row));
  int32_t* row_token = reinterpret_cast<int32_t*>(at(ws, L.row_token));
  void* x_packed = at(ws, L.x_packed);
  void* h = at(ws, L.h);
  void* y_packed = at(ws, L.y_packed);

  // The router's last tile also turns the histogram into prefixes and writes the segment
  // table, so the pack reads finished positions.
  const DispatchPrep prep = make_dispatch_prep(
      c, hist, offsets, demand, reinterpret_cast<unsigned int*>(at(ws, kWsPrepCounterOffset)));
  // events: 0 start, then after route, pack, [reroute, with 7 events], gate/up, down, combine
  const int rr_ev = (n_ev == 7) ? 1 : 0;
  MOE_TRY(record(ev, 0, stream));
  MOE_TRY(cuda_status(
      launch_router(c, x, w_router, logit_bias, ids, gates, hist, extra, prep, status, stream)));
  MOE_TRY(record(ev, 1, stream));
  const bool fuse_gather = (c.fuse & MOE_FUSE_GATHER) != 0;
  const bool fuse_combine = (c.fuse & MOE_FUSE_COMBINE) != 0;
  int32_t* need = fuse_combine ? reinterpret_cast<int32_t*>(at(ws, L.need)) : nullptr;
  int32_t* counters = fuse_combine ? reinterpret_cast<int32_t*>(at(ws, L.counters)) : nullptr;
  const void* resid = c.add_residual ? x : nullptr;
  const PackFusion pf{fuse_gather ? 0 : 1, need, counters, resid, fuse_combine ? y : nullptr,
                      c.has_shared};
  MOE_TRY(cuda_status(launch_dispatch_pack(c, x, ids, hist, offsets, x_packed, row_token,
                                           route_row, status, stream,
                                           c.fuse != 0 ? &pf : nullptr)));
  if (rr_ev) MOE_TRY(record(ev, 2, stream));
  if (reroute(c))
    MOE_TRY(cuda_status(launch_reroute(c, x, ids, extra.zkeys, gates, x_packed, row_token,
                                       route_row, offsets,
                                       reinterpret_cast<int32_t*>(at(ws, L.rlist)), status,
                                       stream)));
  MOE_TRY(record(ev, 2 + rr_ev, stream));
  const FusedCombine fc{route_row, gates, row_token, need, counters, resid, y, c.k, c.has_shared};
  FfnArgs f{x, x_packed, offsets, w_gate, w_up, w_down, shared_gate, shared_up, shared_down,
            h, y_packed, L.rmax, status, padded(c) ? offsets + c.E + 2 : nullptr,
            fuse_gather ? row_token : nullptr, fuse_combine ? &fc : nullptr};
  MOE_TRY(ffn(c, f, stream, ev ? static_cast<cudaEvent_t>(ev[3 + rr_ev]) : nullptr));
  MOE_TRY(record(ev, 4 + rr_ev, stream));
  if (!fuse_combine)
    MOE_TRY(cuda_status(launch_combine(c, y_packed, route_row, gates, offsets, x, y, stream)));
  return record(ev, 5 + rr_ev, stream);
}

}  // namespace

extern "C" {

int32_t moe_abi_version(void) { return kAbiVersion; }

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID: return "invalid argument";
    case MOE_ERR_UNSUPPORTED: return "unsupported configuration";
    case MOE_ERR_WORKSPACE: return "workspace missing or misaligned";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_BAD_EXPERT_ID: return "expert id out of range or repeated within a token";
    case MOE_ERR_TIMEOUT: return "a bounded device wait ran out";
  }
  return "unknown status";
}

int32_t moe_capacity(int32_t T, int32_t k, int32_t E, int32_t phi_num, int32_t phi_den) {
  if (T < 0 || k < 0 || E <= 0 || phi_num < 0 || phi_den <= 0) return -1;
  const int64_t num = static_cast<int64_t>(phi_num) * T * k;
  const int64_t den = static_cast<int64_t>(phi_den) * E;
  const int64_t c = (num + den - 1) / den;
  return c > INT32_MAX ? -1 : static_cast<int32_t>(c);
}

int32_t moe_ffn_tile_shape(const moe_config* cfg) {
  if (validate(cfg) != MOE_OK) return 0;
  return ffn_tile_shape(*cfg);
}

int32_t moe_ffn_launches(const moe_config* cfg) {
  if (validate(cfg) != MOE_OK) return 0;
  return ffn_launches(*cfg);
}

int64_t moe_max_rows(const moe_config* cfg) {
  if (validate(cfg) != MOE_OK) return 0;
  return max_rows(*cfg);
}

size_t moe_workspace_bytes(const moe_config* cfg) {
  if (validate(cfg) != MOE_OK) return 0;
  return layout_of(*cfg).total;
}

moe_status moe_workspace_init(void* ws, moe_stream_t stream) {
  MOE_TRY(check_ws(ws));
  return cuda_status(cudaMemsetAsync(ws, 0, kWsHeaderBytes, stream));
}

moe_status moe_route(const moe_config* cfg, const void* x, const void* w_router,
                     const float* logit_bias, int32_t* ids, float* gates, void* ws,
                     moe_stream_t stream) {
  MOE_TRY(validate(cfg));
  MOE_TRY(check_ws(ws));
  if (!x || !w_router || !ids || !gates) return MOE_ERR_INVALID;
  const Layout L = layout_of(*cfg);
  const RouterExtras extra{cfg->stats ? reinterpret_cast<float*>(at(ws, L.tile_psum)) : nullptr,
                           reroute(*cfg) ? reinterpret_cast<float*>(at(ws, L.zkeys)) : nullptr};
  const DispatchPrep no_prep{};  // moe_dispatch recounts from the ids it is given
  return cuda_status(launch_router(*cfg, x, w_router, logit_bias, ids, gates,
                                   reinterpret_cast<int32_t*>(at(ws, L.tile_hist)), extra,
                                   no_prep, static_cast<int32_t*>(ws), stream));
}

moe_status moe_dispatch(const moe_config* cfg, const void* x, const int32_t* ids,
                        float* gates, void* x_packed, int32_t* row_token, int32_t* route_row,
                        int32_t* offsets, int32_t* demand, void* ws, moe_stream_t stream) {
  MOE_TRY(validate(cfg));
  MOE_TRY(check_ws(ws));
  if (!x || !ids || !x_packed || !row_token || !route_row || !offsets || !demand)
    return MOE_ERR_INVALID;
  if (reroute(*cfg) && !gates) return MOE_ERR_INVALID;
  const Layout L = layout_of(*cfg);
  int32_t* hist = reinterpret_cast<int32_t*>(at(ws, L.tile_hist));
  int32_t* status = static_cast<int32_t*>(ws);
  const DispatchPrep prep = make_dispatch_prep(
      *cfg, hist, offsets, demand, reinterpret_cast<unsigned int*>(at(ws, kWsPrepCounterOffset)));
  MOE_TRY(cuda_status(launch_dispatch_hist(*cfg, ids, prep, status, stream)));
  MOE_TRY(cuda_status(launch_dispatch_pack(*cfg, x, ids, hist, offsets, x_packed, row_token,
                                           route_row, status, stream)));
  if (!reroute(*cfg)) return MOE_OK;
  return cuda_status(launch_reroute(*cfg, x, ids, reinterpret_cast<const float*>(at(ws, L.zkeys)),
                                    gates, x_packed, row_token, route_row, offsets,
                                    reinterpret_cast<int32_t*>(at(ws, L.rlist)), status, stream));
}

moe_status moe_expert_ffn(const moe_config* cfg, const void* x, const void* x_packed,
                          const int32_t* offsets, const void* w_gate, const void* w_up,
                          const void* w_down, const void* shared_gate, const void* shared_up,
                          const void* shared_down, void* h, void* y_packed, void* ws,
                          moe_stream_t stream) {
  MOE_TRY(validate(cfg));
  MOE_TRY(check_ws(ws));
  if (!x_packed || !offsets || !w_gate || !w_up || !w_down || !h || !y_packed)
    return MOE_ERR_INVALID;
  if (cfg->has_shared && (!x || !shared_gate || !shared_up || !shared_down)) return MOE_ERR_INVALID;
  FfnArgs f{x, x_packed, offsets, w_gate, w_up, w_down, shared_gate, shared_up, shared_down,
            h, y_packed, max_rows(*cfg), static_cast<int32_t*>(ws),
            padded(*cfg) ? offsets + cfg->E + 2 : nullptr};
  return ffn(*cfg, f, stream);
}

moe_status moe_combine(const moe_config* cfg, const void* y_packed, const int32_t* route_row,
                       const float* gates, const int32_t* offsets, const void* residual,
                       void* y, moe_stream_t stream) {
  MOE_TRY(validate(cfg));
  if (!y_packed || !route_row || !gates || !y) return MOE_ERR_INVALID;
  if (cfg->has_shared && !offsets) return MOE_ERR_INVALID;
  if (cfg->add_residual && !residual) return MOE_ERR_INVALID;
  return cuda_status(launch_combine(*cfg, y_packed, route_row, gates, offsets, residual, y, stream));
}

moe_status moe_forward(const moe_config* cfg, const void* x, const void* w_router,
                       const float* logit_bias, const void* w_gate, const void* w_up,
                       const void* w_down, const void* shared_gate, const void* shared_up,
                       const void* shared_down, void* y, int32_t* ids_out, float* gates_out,
                       int32_t* demand_out, int32_t* offsets_out, void* ws,
                       moe_stream_t stream) {
  return forward_impl(cfg, x, w_router, logit_bias, w_gate, w_up, w_down, shared_gate, shared_up,
                      shared_down, y, ids_out, gates_out, demand_out, offsets_out, nullptr, 0,
                      ws, stream);
}

moe_status moe_forward_profiled(const moe_config* cfg, const void* x, const void* w_router,
                                const float* logit_bias, const void* w_gate, const void* w_up,
                                const void* w_down, const void* shared_gate,
                                const void* shared_up, const void* shared_down, void* y,
                                int32_t* ids_out, float* gates_out, int32_t* demand_out,
                                int32_t* offsets_out, void* const* events, int32_t n_events,
                                void* ws, moe_stream_t stream) {
  if (events == nullptr || (n_events != 6 && n_events != 7)) return MOE_ERR_INVALID;
  for (int i = 0; i < n_events; ++i)
    if (events[i] == nullptr) return MOE_ERR_INVALID;
  return forward_impl(cfg, x, w_router, logit_bias, w_gate, w_up, w_down, shared_gate, shared_up,
                      shared_down, y, ids_out, gates_out, demand_out, offsets_out, events,
                      n_events, ws, stream);
}

moe_status moe_routing_stats(const moe_config* cfg, const int32_t* demand,
                             const int32_t* offsets, float alpha, float* f, float* P,
                             moe_routing_summary* summary, void* ws, moe_stream_t stream) {
  MOE_TRY(validate(cfg));
  MOE_TRY(check_ws(ws));
  if (!cfg->stats || summary == nullptr || !std::isfinite(alpha)) return MOE_ERR_INVALID;
  const Layout L = layout_of(*cfg);
  const int32_t* dem = demand ? demand : reinterpret_cast<const int32_t*>(at(ws, L.demand));
  const int32_t* off = offsets ? offsets : reinterpret_cast<const int32_t*>(at(ws, L.offsets));
  return cuda_status(launch_routing_stats(
      *cfg, reinterpret_cast<const float*>(at(ws, L.tile_psum)), dem, off, alpha,
      reinterpret_cast<double*>(at(ws, L.stats_partial)),
      reinterpret_cast<unsigned int*>(at(ws, kWsStatsCounterOffset)), f, P, summary, stream));
}

moe_status moe_get_device_status(void* ws, moe_stream_t stream, int32_t clear,
                                 int32_t* status_out) {
  MOE_TRY(check_ws(ws));
  if (status_out == nullptr) return MOE_ERR_INVALID;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return MOE_ERR_CUDA;
  int32_t v = 0;
  if (cudaMemcpy(&v, ws, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return MOE_ERR_CUDA;
  if (clear && cudaMemset(ws, 0, sizeof(int32_t)) != cudaSuccess) return MOE_ERR_CUDA;
  *status_out = v;
  return MOE_OK;
}

moe_status moe_debug_bounded_wait(void* ws, int64_t limit_ns, moe_stream_t stream) {
  MOE_TRY(check_ws(ws));
  if (limit_ns < 1000 || limit_ns > 10000000000LL) return MOE_ERR_INVALID;
  return cuda_status(launch_debug_wait(static_cast<int32_t*>(ws), limit_ns, stream));
}

}  // extern "C"

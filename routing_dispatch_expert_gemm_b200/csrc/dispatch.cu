// Pack: per-expert demand, arrival-order positions, capacity mask, expert-major offsets,
// and the copy of duplicated token rows into expert batches.
//
// Sources: "271,104 Routes: What I Missed About Mixture-of-Experts", section 3 Dispatch
// (route table of token, expert, position, gate; group by expert; bincount + cumsum
// segment ends) and its subsection on expert capacity; "Mixture-of-Experts: routing and
// capacity", Capacity and Worked case (arrival order decides which route is dropped);
// "Mixture-of-experts routing", Capacity (C = ceil(phi T k / E)).
//
// Positions are deterministic without ordered atomics: the position of route (t, j) in
// expert e is the number of earlier tokens that chose e, i.e.
//   (routes to e in earlier 128-token tiles)  +  (earlier tokens of t's tile that chose e).
// The first term is the exclusive prefix that the dispatch prep leaves in place of the
// tile histogram (dispatch_prep.cuh: computed once, by the CTA that writes the histogram's
// last tile, in the router for moe_forward or in hist_kernel for caller-given ids); the
// second is counted by the token's warp with ballots over the tile's ids.  Each warp owns
// one token: it loads the token row while it works out the positions, then writes the row
// to each kept route's row with 16-byte stores.  With the padded [E, C, d] buffer expert
// e's rows start at e*C and empty slots are marked -1.
#include "common.cuh"
#include "dispatch_prep.cuh"
#include "internal.h"

namespace moe {

DispatchPrep make_dispatch_prep(const moe_config& c, int32_t* tile_hist, int32_t* offsets,
                                int32_t* demand, unsigned int* ticket) {
  return DispatchPrep{tile_hist, offsets, demand, ticket, num_tiles_for(c.T, c.E), c.E, c.T,
                      c.capacity, c.has_shared, c.layout == MOE_LAYOUT_PADDED ? 1 : 0};
}

namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads)
    hist_kernel(const int32_t* __restrict__ ids, int T, int k, int E, DispatchPrep prep,
                int32_t* status) {
  __shared__ int s_hist[256];
  __shared__ int s_scratch[kPrepScratchInts];
  const int tile = blockIdx.x;
  const int tok0 = tile * kHistTile;
  const int ntok = min(kHistTile, T - tok0);
  for (int e = threadIdx.x; e < E; e += kThreads) s_hist[e] = 0;
  pdl_trigger();
  pdl_wait();
  __syncthreads();
  for (int r = threadIdx.x; r < ntok * k; r += kThreads) {
    const int t = tok0 + r / k, j = r % k;
    const int32_t* row = ids + static_cast<size_t>(t) * k;
    const int e = row[j];
    if (route_id_valid(row, j, e, E))
      atomicAdd(&s_hist[e], 1);
    else
      record_status(status, MOE_ERR_BAD_EXPERT_ID);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kThreads)
    prep.tile_hist[static_cast<size_t>(tile) * E + e] = s_hist[e];
  dispatch_prep_arrive(prep, s_scratch);
}

struct PackArgs {
  const void* x;
  const int32_t* ids;
  const int32_t* tile_prefix;  // [num_tiles, E]: routes to e in earlier tiles
  const int32_t* offsets;      // segment table ([E+2], or [2E+2] padded)
  int T, d, k, E, capacity, padded;
  void* x_packed;
  int32_t* row_token;
  int32_t* route_row;
  int32_t* status;
  // fused steps of moe_forward (see PackFusion)
  int copy;
  int32_t* need;
  int32_t* counters;
  int counter_cols;
  const void* residual;
  void* y;
  int has_shared;
};

constexpr int kWarpsPerCta = kThreads / 32;
constexpr int kNV = 8;  // 16-byte vectors per lane per pass over a token row (4 KB per warp)

template <typename T, int KMAX>
__global__ void __launch_bounds__(kThreads) pack_kernel(PackArgs a) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_trigger();
  pdl_wait();
  const int E = a.E, k = a.k;
  if (a.padded) {  // padding slots of the buffer: row_token = -1 (every CTA takes a share)
    const long long slots = static_cast<long long>(E) * a.capacity;
    for (long long i = static_cast<long long>(blockIdx.x) * kThreads + threadIdx.x; i < slots;
         i += static_cast<long long>(gridDim.x) * kThreads) {
      const int e = static_cast<int>(i / a.capacity);
      const int p = static_cast<int>(i - static_cast<long long>(e) * a.capacity);
      if (p >= __ldg(a.offsets + E + 2 + e)) a.row_token[i] = -1;
    }
  }
  const int t = blockIdx.x * kWarpsPerCta + warp;
  if (t >= a.T) return;

  // 1. The first pass of the token row goes out first: it does not depend on the routing.
  const int nvec = a.d * static_cast<int>(sizeof(T)) / 16;
  const uint4* __restrict__ xrow = reinterpret_cast<const uint4*>(static_cast<const T*>(a.x) +
                                                                   static_cast<size_t>(t) * a.d);
  uint4 v[kNV];
#pragma unroll
  for (int i = 0; i < kNV; ++i) {
    const int idx = i * 32 + lane;
    v[i] = idx < nvec ? __ldg(xrow + idx) : make_uint4(0, 0, 0, 0);
  }

  // 2. The token's routes: lane j holds slot j.  A route is valid if its id is in range
  //    and not repeated earlier in the token's row.
  int e = -1;
  if (lane < k) e = __ldg(a.ids + static_cast<size_t>(t) * k + lane);
  bool valid = lane < k && e >= 0 && e < E;
#pragma unroll
  for (int q = 0; q < KMAX; ++q) {
    if (q >= k) break;
    const int eq = __shfl_sync(0xffffffffu, e, q);
    if (q < lane && eq == e) valid = false;
  }
  if (lane < k && !valid) record_status(a.status, MOE_ERR_BAD_EXPERT_ID);
  // rank among the earlier tokens of the tile: lane l looks at token c + l; for each slot j
  // a ballot counts the earlier tokens that hold slot j's expert (once per token, as the
  // histogram counts it)
  const int tile = t / kHistTile;
  int rank = 0;
  for (int c = tile * kHistTile; c < t; c += 32) {
    const int tok = c + lane;
    int row[KMAX];
#pragma unroll
    for (int q = 0; q < KMAX; ++q)
      row[q] = (q < k && tok < t) ? __ldg(a.ids + static_cast<size_t>(tok) * k + q) : -1;
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      if (j >= k) break;
      const int ej = __shfl_sync(0xffffffffu, e, j);
      const bool vj = __shfl_sync(0xffffffffu, valid ? 1 : 0, j) != 0;
      bool m = false;
#pragma unroll
      for (int q = 0; q < KMAX; ++q) m |= (row[q] == ej);
      const int cnt = __popc(__ballot_sync(0xffffffffu, vj && m));
      if (lane == j) rank += cnt;
    }
  }
  int out = -1;
  if (valid) {
    const int pos = __ldg(a.tile_prefix + static_cast<size_t>(tile) * E + e) + rank;
    if (a.capacity < 0 || pos < a.capacity) {
      out = a.padded ? e * a.capacity + pos : __ldg(a.offsets + e) + pos;
      a.row_token[out] = t;
    }
  }
  if (lane < k) a.route_row[static_cast<size_t>(t) * k + lane] = out;

  // Fused combine: the token's number of contributions and its zeroed counters; a token
  // with none (every route dropped, no shared expert) gets its output row here:
  // x[t] with the residual, else zeros (what the combine's fp32 sum would round to).
  bool write_y = false;
  if (a.need != nullptr) {
    const int cnt = __popc(__ballot_sync(0xffffffffu, lane < k && out >= 0)) + a.has_shared;
    if (lane == 0) a.need[t] = cnt;
    for (int i = lane; i < a.counter_cols; i += 32)
      a.counters[static_cast<size_t>(t) * a.counter_cols + i] = 0;
    write_y = (cnt == 0);
  }
  if (!a.copy && !write_y) return;

  // 3. Copy: each pass of the row is written to every kept route's row.
  T* __restrict__ XP = static_cast<T*>(a.x_packed);
  uint4* __restrict__ yrow = write_y ? reinterpret_cast<uint4*>(static_cast<T*>(a.y) +
                                                                 static_cast<size_t>(t) * a.d)
                                     : nullptr;
  for (int base = 0; base < nvec; base += 32 * kNV) {
    if (base > 0) {
#pragma unroll
      for (int i = 0; i < kNV; ++i) {
        const int idx = base + i * 32 + lane;
        v[i] = idx < nvec ? __ldg(xrow + idx) : make_uint4(0, 0, 0, 0);
      }
    }
    if (write_y) {
#pragma unroll
      for (int i = 0; i < kNV; ++i) {
        const int idx = base + i * 32 + lane;
        if (idx < nvec) yrow[idx] = a.residual != nullptr ? v[i] : make_uint4(0, 0, 0, 0);
      }
    }
    if (!a.copy) continue;
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      if (j >= k) break;
      const int r = __shfl_sync(0xffffffffu, out, j);
      if (r < 0) continue;
      uint4* dst = reinterpret_cast<uint4*>(XP + static_cast<size_t>(r) * a.d);
#pragma unroll
      for (int i = 0; i < kNV; ++i) {
        const int idx = base + i * 32 + lane;
        if (idx < nvec) dst[idx] = v[i];
      }
    }
  }
}

template <typename T>
cudaError_t launch_pack_typed(const PackArgs& a, cudaStream_t s) {
  const int grid = (a.T + kWarpsPerCta - 1) / kWarpsPerCta;
  const dim3 g(grid), b(kThreads);
  if (a.k <= 1) return launch_pdl(pack_kernel<T, 1>, g, b, 0, s, a);
  if (a.k <= 2) return launch_pdl(pack_kernel<T, 2>, g, b, 0, s, a);
  if (a.k <= 4) return launch_pdl(pack_kernel<T, 4>, g, b, 0, s, a);
  if (a.k <= 8) return launch_pdl(pack_kernel<T, 8>, g, b, 0, s, a);
  if (a.k <= 16) return launch_pdl(pack_kernel<T, 16>, g, b, 0, s, a);
  return launch_pdl(pack_kernel<T, 32>, g, b, 0, s, a);
}

}  // namespace

cudaError_t launch_dispatch_hist(const moe_config& c, const int32_t* ids,
                                 const DispatchPrep& prep, int32_t* status, cudaStream_t s) {
  const int grid = num_tiles_for(c.T, c.E);
  static DeviceOnce once;
  cudaError_t e = once.run([] { return prefer_max_shared(hist_kernel); });
  if (e != cudaSuccess) return e;
  return launch_pdl(hist_kernel, dim3(grid), dim3(kThreads), 0, s, ids, c.T, c.k, c.E, prep,
                    status);
}

cudaError_t launch_dispatch_pack(const moe_config& c, const void* x, const int32_t* ids,
                                 const int32_t* tile_prefix, const int32_t* offsets,
                                 void* x_packed, int32_t* row_token, int32_t* route_row,
                                 int32_t* status, cudaStream_t s, const PackFusion* fused) {
  PackArgs a{x, ids, tile_prefix, offsets, c.T, c.d, c.k, c.E, c.capacity,
             c.layout == MOE_LAYOUT_PADDED ? 1 : 0, x_packed, row_token, route_row, status,
             1, nullptr, nullptr, (c.d + 31) / 32, nullptr, nullptr, c.has_shared};
  if (fused != nullptr) {
    a.copy = fused->copy;
    a.need = fused->need;
    a.counters = fused->counters;
    a.residual = fused->residual;
    a.y = fused->y;
  }
  if (c.dtype == MOE_BF16) return launch_pack_typed<__nv_bfloat16>(a, s);
  return launch_pack_typed<float>(a, s);
}

}  // namespace moe

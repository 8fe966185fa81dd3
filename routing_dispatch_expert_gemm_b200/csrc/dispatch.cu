// Pack: per-expert demand, arrival-order positions, capacity mask, expert-major offsets,
// and the scatter of duplicated token rows into expert batches.
//
// Sources: "271,104 Routes: What I Missed About Mixture-of-Experts", section 3 Dispatch
// (route table of token, expert, position, gate; group by expert; bincount + cumsum
// segment ends) and its subsection on expert capacity; "Mixture-of-Experts: routing and
// capacity", Capacity and Worked case (arrival order decides which route is dropped);
// "Mixture-of-experts routing", Capacity (C = ceil(phi T k / E)).
//
// Positions are deterministic without ordered atomics: the position of route (t, j) in
// expert e is the number of earlier tokens that chose e, i.e.
//   (routes to e in earlier token tiles)  +  popcount(bitmask of earlier tokens of this
//   tile that chose e).
// The first term is an exclusive prefix over the per-128-token-tile histogram; every CTA
// computes the prefix it needs directly from the histogram (ceil(T/128) x E entries), so
// no separate scan launch and no inter-CTA waiting is needed.  Pack CTAs cover 8-token
// sub-tiles of a histogram tile, so the copy work spreads over many SMs.  A CTA starts the
// bulk loads of its token rows first (they do not depend on the routing), works out the
// positions meanwhile, then all its warps write each row to its kept routes' rows.  With
// the padded [E, C, d] buffer expert e's rows start at e*C and empty slots are marked -1.
#include "common.cuh"
#include "internal.h"

namespace moe {

namespace {

constexpr int kThreads = 256;

__global__ void __launch_bounds__(kThreads)
    hist_kernel(const int32_t* __restrict__ ids, int T, int k, int E, int tok_tile,
                int32_t* __restrict__ tile_hist, int32_t* status) {
  __shared__ int s_hist[256];
  const int tile = blockIdx.x;
  const int tok0 = tile * tok_tile;
  const int ntok = min(tok_tile, T - tok0);
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
    tile_hist[static_cast<size_t>(tile) * E + e] = s_hist[e];
}

struct ScatterArgs {
  const void* x;
  const int32_t* ids;
  const int32_t* tile_hist;
  int T, d, k, E, tok_tile, num_tiles, capacity, has_shared, copy_round, padded;
  void* x_packed;
  int32_t* row_token;
  int32_t* route_row;
  int32_t* offsets;
  int32_t* demand;
  int32_t* status;
};

constexpr int kSubTok = 8;  // tokens packed per CTA
constexpr size_t kStageBudget = 64 * 1024;  // shared memory staging token rows for the copy

template <typename T>
__global__ void __launch_bounds__(kThreads) scatter_kernel(ScatterArgs a) {
  constexpr int kBatch = 8;    // histogram loads in flight per thread
  constexpr int kWords = kHistTile / 32;
  __shared__ int s_pre[256];   // routes to e in earlier tiles
  __shared__ int s_tot[256];   // routes to e in all tiles (demand)
  __shared__ int s_off[257];   // segment starts over kept routes
  __shared__ int s_rows[kSubTok][32];
  __shared__ uint32_t s_mask[256 * kWords];  // [E][words]: bit = token of the tile chose e
  __shared__ int s_ids[kHistTile * 32];      // the histogram tile's expert ids [128][k]
  __shared__ __align__(8) uint64_t s_bar;
  extern __shared__ __align__(128) uint8_t s_stage[];  // copy_round token rows

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t_begin = blockIdx.x * kSubTok;
  const int nsub = min(kSubTok, a.T - t_begin);
  const int tile = t_begin / kHistTile;
  const int tile0 = tile * kHistTile;
  const int ntile = min(kHistTile, a.T - tile0);
  const int E = a.E, k = a.k;

  for (int e = tid; e < E; e += kThreads) { s_pre[e] = 0; s_tot[e] = 0; }
  for (int w = tid; w < E * kWords; w += kThreads) s_mask[w] = 0;
  pdl_trigger();
  pdl_wait();

  // 0. The token rows do not depend on the routing: start the first round of their bulk
  //    loads now, so that they arrive while the positions are being worked out.
  const uint32_t row_bytes = static_cast<uint32_t>(a.d) * sizeof(T);
  const int round = a.copy_round;  // token rows staged at a time
  const T* __restrict__ X = static_cast<const T*>(a.x);
  T* __restrict__ XP = static_cast<T*>(a.x_packed);
  if (tid == 0) {
    mbar_init(&s_bar, 1);
    fence_mbar_init();
    const int nr = min(round, nsub);
    mbar_arrive_expect_tx(&s_bar, nr * row_bytes);
    for (int i = 0; i < nr; ++i)
      bulk_load(s_stage + i * row_bytes, X + static_cast<size_t>(t_begin + i) * a.d, row_bytes,
                &s_bar);
  }
  // The tile's expert ids, one coalesced pass (its loads overlap the histogram's below).
  for (int r = tid; r < ntile * k; r += kThreads)
    s_ids[r] = __ldg(a.ids + static_cast<size_t>(tile0) * k + r);
  __syncthreads();

  // 1. prefix (tiles < this one) and total per expert, split over all threads with
  //    kBatch independent loads in flight per thread
  {
    const int nparts = kThreads / E;  // >= 1 since E <= 256
    if (tid < nparts * E) {
      const int e = tid % E, part = tid / E;
      int pre = 0, tot = 0;
      for (int i0 = part; i0 < a.num_tiles; i0 += nparts * kBatch) {
        int h[kBatch];
#pragma unroll
        for (int q = 0; q < kBatch; ++q) {
          const int i = i0 + q * nparts;
          h[q] = (i < a.num_tiles) ? __ldg(a.tile_hist + static_cast<size_t>(i) * E + e) : 0;
        }
#pragma unroll
        for (int q = 0; q < kBatch; ++q) {
          tot += h[q];
          pre += (i0 + q * nparts < tile) ? h[q] : 0;
        }
      }
      atomicAdd(&s_pre[e], pre);
      atomicAdd(&s_tot[e], tot);
    }
  }
  // 2. bitmask of the histogram tile's tokens per expert
  for (int r = tid; r < ntile * k; r += kThreads) {
    const int tl = r / k, j = r % k;
    const int32_t* row = s_ids + tl * k;
    const int e = row[j];
    if (route_id_valid(row, j, e, E)) atomicOr(&s_mask[e * kWords + (tl >> 5)], 1u << (tl & 31));
  }
  __syncthreads();

  // 3. kept counts -> exclusive scan -> offsets (warp 0, 32 experts per step); the padded
  //    buffer gives expert e the fixed rows e*C ..
  if (a.padded) {
    for (int e = tid; e <= E; e += kThreads) s_off[e] = e * a.capacity;
  } else if (warp == 0) {
    int carry = 0;
    for (int base = 0; base < E; base += 32) {
      const int e = base + lane;
      int kept = 0;
      if (e < E) kept = (a.capacity < 0) ? s_tot[e] : min(s_tot[e], a.capacity);
      int incl = kept;
#pragma unroll
      for (int s = 1; s < 32; s <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, s);
        if (lane >= s) incl += o;
      }
      if (e < E) s_off[e] = carry + incl - kept;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) s_off[E] = carry;
  }
  __syncthreads();
  if (blockIdx.x == 0) {
    for (int e = tid; e <= E; e += kThreads) a.offsets[e] = s_off[e];
    if (tid == 0) a.offsets[E + 1] = s_off[E] + (a.has_shared ? a.T : 0);
    for (int e = tid; e < E; e += kThreads) a.demand[e] = s_tot[e];
    if (a.padded)  // filled slots
      for (int e = tid; e < E; e += kThreads) a.offsets[E + 2 + e] = min(s_tot[e], a.capacity);
  }
  if (a.padded) {  // padding slots of the buffer: row_token = -1 (the CTAs share the sweep)
    const long long slots = static_cast<long long>(E) * a.capacity;
    for (long long i = static_cast<long long>(blockIdx.x) * kThreads + tid; i < slots;
         i += static_cast<long long>(gridDim.x) * kThreads) {
      const int e = static_cast<int>(i / a.capacity);
      const int p = static_cast<int>(i - static_cast<long long>(e) * a.capacity);
      if (p >= s_tot[e]) a.row_token[i] = -1;
    }
  }

  // 4. rows of this CTA's tokens' routes
  for (int r = tid; r < nsub * k; r += kThreads) {
    const int ts = r / k, j = r - ts * k;
    const int t = t_begin + ts, tl = t - tile0;
    const int32_t* row = s_ids + tl * k;
    const int e = row[j];
    int out = -1;
    if (route_id_valid(row, j, e, E)) {
      const uint32_t* m = s_mask + e * kWords;
      int rank = __popc(m[tl >> 5] & ((1u << (tl & 31)) - 1u));
      for (int w = 0; w < (tl >> 5); ++w) rank += __popc(m[w]);
      const int pos = s_pre[e] + rank;
      if (a.capacity < 0 || pos < a.capacity) {
        out = s_off[e] + pos;
        a.row_token[out] = t;
      }
    }
    a.route_row[static_cast<size_t>(t) * k + j] = out;
    s_rows[ts][j] = out;
  }
  __syncthreads();

  // 5. copy: each token row is loaded once into shared memory by the bulk-copy engine
  //    (the first round was issued at the start) and written to each of its kept routes'
  //    rows by all warps with 16-byte stores, one warp per destination row.
  __shared__ int s_ok;
  uint32_t phase = 0;
  const int nvec = static_cast<int>(row_bytes / 16);
  for (int r0 = 0; r0 < nsub; r0 += round) {
    const int nr = min(round, nsub - r0);
    if (r0 > 0) {
      __syncthreads();  // every warp has finished reading the previous round's rows
      if (tid == 0) {
        mbar_arrive_expect_tx(&s_bar, nr * row_bytes);
        for (int i = 0; i < nr; ++i)
          bulk_load(s_stage + i * row_bytes, X + static_cast<size_t>(t_begin + r0 + i) * a.d,
                    row_bytes, &s_bar);
      }
    }
    if (tid == 0) {
      int ok = mbar_wait_bounded(&s_bar, phase, nullptr, kWaitLimitNs, a.status);
      if (!ok) mbar_wait_bounded(&s_bar, phase, nullptr, kWaitLimitNs, a.status);  // drain
      s_ok = ok;
    }
    __syncthreads();  // the rows have landed (thread 0 saw the transaction count complete)
    if (!s_ok) return;
    phase ^= 1u;
    for (int ij = warp; ij < nr * k; ij += kThreads / 32) {
      const int i = ij / k, j = ij - i * k;
      const int r = s_rows[r0 + i][j];
      if (r < 0) continue;
      const uint4* src = reinterpret_cast<const uint4*>(s_stage + i * row_bytes);
      uint4* dst = reinterpret_cast<uint4*>(XP + static_cast<size_t>(r) * a.d);
      for (int v = lane; v < nvec; v += 32) dst[v] = src[v];
    }
  }
}

}  // namespace

cudaError_t launch_dispatch_hist(const moe_config& c, const int32_t* ids, int32_t* tile_hist,
                                 int32_t* status, cudaStream_t s) {
  const int tt = tok_tile_for(c.T, c.E);
  const int grid = (c.T + tt - 1) / tt;
  static DeviceOnce once;
  cudaError_t e = once.run([] { return prefer_max_shared(hist_kernel); });
  if (e != cudaSuccess) return e;
  return launch_pdl(hist_kernel, dim3(grid), dim3(kThreads), 0, s, ids, c.T, c.k, c.E, tt,
                    tile_hist, status);
}

cudaError_t launch_dispatch_scatter(const moe_config& c, const void* x, const int32_t* ids,
                                    const int32_t* tile_hist, void* x_packed,
                                    int32_t* row_token, int32_t* route_row, int32_t* offsets,
                                    int32_t* demand, int32_t* status, cudaStream_t s) {
  const int grid = (c.T + kSubTok - 1) / kSubTok;
  const size_t row_bytes = static_cast<size_t>(c.d) * (c.dtype == MOE_BF16 ? 2 : 4);
  int round = static_cast<int>(kStageBudget / row_bytes);
  round = round < 1 ? 1 : (round > kSubTok ? kSubTok : round);
  ScatterArgs a{x, ids, tile_hist, c.T, c.d, c.k, c.E, kHistTile, num_tiles_for(c.T, c.E),
                c.capacity, c.has_shared, round, c.layout == MOE_LAYOUT_PADDED ? 1 : 0, x_packed,
                row_token, route_row, offsets, demand, status};
  const size_t smem = static_cast<size_t>(round) * row_bytes;
  static DeviceOnce once;
  cudaError_t e = once.run([] {
    prefer_max_shared(scatter_kernel<__nv_bfloat16>);
    prefer_max_shared(scatter_kernel<float>);
    cudaError_t r = cudaFuncSetAttribute(scatter_kernel<__nv_bfloat16>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(kStageBudget));
    if (r != cudaSuccess) return r;
    return cudaFuncSetAttribute(scatter_kernel<float>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                static_cast<int>(kStageBudget));
  });
  if (e != cudaSuccess) return e;
  if (c.dtype == MOE_BF16)
    return launch_pdl(scatter_kernel<__nv_bfloat16>, dim3(grid), dim3(kThreads), smem, s, a);
  return launch_pdl(scatter_kernel<float>, dim3(grid), dim3(kThreads), smem, s, a);
}

}  // namespace moe

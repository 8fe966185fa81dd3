// Reroute overflow policy on the padded dispatch buffer [E, C, d].
//
// Sources: "Mixture-of-Experts: routing and capacity", Capacity (the buffer has C slots
// per expert; empty slots are padding) and Overflow policies (reroute: the overflowing
// route is handled by the next-best expert by score, the router's decision overridden).
//
// Runs after the arrival-order pack, which has already placed every route that fit and
// left route_row = -1 on the ones that overflowed.  The reroute is sequential by definition
// (whether a route finds a free slot depends on every earlier reroute): reroute_walk_kernel
// walks the overflowed routes in arrival order with one warp, while the other warps of its
// CTA precompute each route's preference order.  A second, grid-wide kernel copies each
// moved route's token row and re-evaluates that token's gates by the gate mode over its
// final experts.
#include <climits>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kThreads = 256;  // copy kernel
constexpr int kWarps = kThreads / 32;


__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, s));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) v += __shfl_xor_sync(0xffffffffu, v, s);
  return v;
}

// Gates of token t over its final experts (warp-wide; lane j < k writes slot j).  Slot j's
// expert is the one whose block holds its row, or its original expert when it was dropped.
__device__ void regate(const int32_t* ids, const float* zkeys, const int32_t* route_row,
                       float* gates, int t, int k, int E, int C, int gate_mode, int lane) {
  const float* zrow = zkeys + static_cast<size_t>(t) * E;
  int e = -1;
  if (lane < k) {
    const int r = route_row[static_cast<size_t>(t) * k + lane];
    e = (r >= 0) ? r / C : ids[static_cast<size_t>(t) * k + lane];
  }
  const bool valid = e >= 0 && e < E;
  const float zf = valid ? zrow[e] : -INFINITY;
  float g;
  if (gate_mode != MOE_GATE_SOFTMAX_TOPK) {
    // softmax over the final experts' logits.  For the renormalised mode this is
    // p_i / sum_j p_j with the full softmax's normaliser cancelled; shifting by the
    // final experts' own max keeps it finite when the token no longer holds its top
    // expert and every selected p would underflow.
    const float m = warp_max(zf);
    const float ex = valid ? expf(zf - m) : 0.f;
    g = ex / warp_sum(ex);
  } else {  // the full-softmax probability of each final expert
    float m = -INFINITY;
    for (int q = lane; q < E; q += 32) m = fmaxf(m, zrow[q]);
    m = warp_max(m);
    float den = 0.f;
    for (int q = lane; q < E; q += 32) den += expf(zrow[q] - m);
    den = warp_sum(den);
    g = valid ? expf(zf - m) / den : 0.f;
  }
  if (lane < k) gates[static_cast<size_t>(t) * k + lane] = g;
}

// ---------------------------------------------------------------------------------
// Placement: the arrival-order walk itself, by one warp, fed by 31 helper warps.
//  * All 1024 threads first list the overflowed routes in arrival order.
//  * Helper warps take the listed routes in order and, for each, write into a ring of
//    chunks in shared memory the token's expert preference order (logit descending, ties
//    to the lower index: each expert's rank is counted against the whole row of keys) and
//    the set of experts the token already holds (its ids).
//  * Warp 0 walks the routes in arrival order: a route takes the first expert of its
//    preference order that its token does not hold (its ids plus the experts its earlier
//    routes moved to in this walk) and that has a free slot, found 32 candidates at a time
//    with a ballot; its slot is the expert's next free one.  With none it stays dropped.
// Every wait is bounded; on a timeout the kernel records MOE_ERR_TIMEOUT and stops.
// ---------------------------------------------------------------------------------
constexpr int kWalkThreads = 1024;
constexpr int kWalkWarps = kWalkThreads / 32;
constexpr int kHelpers = kWalkWarps - 1;  // warps 1 .. 31
constexpr int kChunk = 32;                // routes per ring chunk
constexpr int kRing = 4;                  // chunks in the ring

struct WalkArgs {
  const int32_t* ids;      // [T, k]
  const float* zkeys;      // [T, E] ranking keys (NaN as -inf)
  int32_t* row_token;      // [E * C]
  int32_t* route_row;      // [T, k]
  int32_t* offsets;        // filled-slot counts at offsets[E + 2 + e]
  int32_t* list;           // [0]: moved routes m, then (token, row) pairs
  int32_t* ag_r;           // [T * k] overflowed routes (flat index), arrival order
  int32_t* status;
  int T, k, E, C;
  int64_t limit_ns;
};

struct RingEntry {
  uint8_t pref[256];   // experts in the token's preference order
  uint32_t held[8];    // experts the token holds (its ids)
  int r;               // flat route index t * k + j; -1: padding past the last route
  int pad[3];
};

__global__ void __launch_bounds__(kWalkThreads, 1) reroute_walk_kernel(WalkArgs a) {
  __shared__ int s_cnt[256];
  __shared__ int s_wtot[kWalkWarps];
  __shared__ int s_n;
  __shared__ __align__(16) RingEntry s_ring[kRing][kChunk];
  __shared__ __align__(8) uint64_t s_full[kRing], s_empty[kRing];
  __shared__ volatile int s_abort;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int E = a.E, k = a.k, C = a.C;
  pdl_wait();  // route_row, counts and the keys come from the router and the pack

  for (int e = tid; e < 256; e += kWalkThreads) s_cnt[e] = (e < E) ? a.offsets[E + 2 + e] : C;
  if (tid == 0) {
    s_n = 0;
    s_abort = 0;
    for (int q = 0; q < kRing; ++q) {
      mbar_init(&s_full[q], kChunk);  // one arrival per route of the chunk
      mbar_init(&s_empty[q], 1);      // the walker, once it is done with the chunk
    }
    fence_mbar_init();
  }
  __syncthreads();

  // 1. overflowed routes, arrival order (block scan of per-warp ballots)
  const int total = a.T * k;  // <= INT_MAX / 2 (validated on the host)
  for (int base = 0; base < total; base += kWalkThreads) {
    const int r = base + tid;
    bool flag = false;
    if (r < total) {
      const int t = r / k, j = r - t * k;
      const int32_t* row = a.ids + static_cast<size_t>(t) * k;
      flag = a.route_row[r] < 0 && route_id_valid(row, j, row[j], E);
    }
    const uint32_t bal = __ballot_sync(0xffffffffu, flag);
    if (lane == 0) s_wtot[warp] = __popc(bal);
    __syncthreads();
    int before = 0, n = 0;
    for (int w = 0; w < kWalkWarps; ++w) {
      before += (w < warp) ? s_wtot[w] : 0;
      n += s_wtot[w];
    }
    if (flag) a.ag_r[s_n + before + __popc(bal & ((1u << lane) - 1u))] = r;
    __syncthreads();
    if (tid == 0) s_n += n;
    __syncthreads();
  }
  const int n = s_n;
  const int nchunks = (n + kChunk - 1) / kChunk;
  __threadfence_block();  // ag_r (global) written by other threads of this CTA above

  if (warp > 0) {
    // ------------------------------------------------------------ helpers
    for (int i = warp - 1; i < nchunks * kChunk; i += kHelpers) {
      const int c = i / kChunk, slot = c % kRing, pos = i % kChunk;
      int ok = 1;
      if (lane == 0)
        ok = mbar_wait_bounded(&s_empty[slot], ((c / kRing) & 1) ^ 1, &s_abort, a.limit_ns,
                               a.status);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      RingEntry& en = s_ring[slot][pos];
      if (i < n) {
        const int r = a.ag_r[i];
        const int t = r / k;
        const float* zrow = a.zkeys + static_cast<size_t>(t) * E;
        float key[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) key[q] = (q * 32 + lane < E) ? zrow[q * 32 + lane] : -INFINITY;
        int rank[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) rank[q] = 0;
        for (int e2 = 0; e2 < E; ++e2) {
          float z2 = key[0];
#pragma unroll
          for (int q = 1; q < 8; ++q) z2 = (q == (e2 >> 5)) ? key[q] : z2;
          z2 = __shfl_sync(0xffffffffu, z2, e2 & 31);
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const int e = q * 32 + lane;
            rank[q] += (z2 > key[q] || (z2 == key[q] && e2 < e)) ? 1 : 0;
          }
        }
#pragma unroll
        for (int q = 0; q < 8; ++q)
          if (q * 32 + lane < E) en.pref[rank[q]] = static_cast<uint8_t>(q * 32 + lane);
        int e = (lane < k) ? a.ids[static_cast<size_t>(t) * k + lane] : -1;
        if (e < 0 || e >= E) e = -1;
#pragma unroll
        for (int w = 0; w < 8; ++w) {
          const uint32_t bit = (e >= 0 && (e >> 5) == w) ? (1u << (e & 31)) : 0u;
          const uint32_t word = __reduce_or_sync(0xffffffffu, bit);
          if (lane == 0) en.held[w] = word;
        }
        if (lane == 0) en.r = r;
      } else if (lane == 0) {
        en.r = -1;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_full[slot]);  // release: the entry is written
    }
  } else {
    // ------------------------------------------------------------ the walk (warp 0)
    int moved = 0;
    int cur_t = -1;
    uint32_t extra[8] = {0, 0, 0, 0, 0, 0, 0, 0};  // experts the current token moved to
    for (int c = 0; c < nchunks; ++c) {
      const int slot = c % kRing;
      int ok = 1;
      if (lane == 0)
        ok = mbar_wait_bounded(&s_full[slot], (c / kRing) & 1, &s_abort, a.limit_ns, a.status);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) {
        if (lane == 0) s_abort = 1;
        break;
      }
      for (int pos = 0; pos < kChunk; ++pos) {
        const RingEntry& en = s_ring[slot][pos];
        const int r = en.r;
        if (r < 0) break;
        const int t = r / k;
        if (t != cur_t) {
          cur_t = t;
#pragma unroll
          for (int w = 0; w < 8; ++w) extra[w] = 0;
        }
        int pick = -1;
        for (int base = 0; base < E && pick < 0; base += 32) {
          const int idx = base + lane;
          int e = -1;
          bool avail = false;
          if (idx < E) {
            e = en.pref[idx];
            uint32_t hw = en.held[e >> 5];
#pragma unroll
            for (int w = 0; w < 8; ++w) hw |= (w == (e >> 5)) ? extra[w] : 0u;
            avail = !((hw >> (e & 31)) & 1u) && s_cnt[e] < C;
          }
          const uint32_t b = __ballot_sync(0xffffffffu, avail);
          if (b != 0) pick = __shfl_sync(0xffffffffu, e, __ffs(b) - 1);
        }
        if (pick >= 0) {
          if (lane == 0) {
            const int slot_in_e = s_cnt[pick];
            s_cnt[pick] = slot_in_e + 1;
            const int row = pick * C + slot_in_e;
            a.route_row[r] = row;
            a.row_token[row] = t;
            a.list[1 + 2 * moved] = t;
            a.list[2 + 2 * moved] = row;
          }
          ++moved;
#pragma unroll
          for (int w = 0; w < 8; ++w)
            if (w == (pick >> 5)) extra[w] |= 1u << (pick & 31);
        }
        __syncwarp();  // lane 0's count update is seen by the next route's checks
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_empty[slot]);  // the chunk's entries may be rewritten
    }
    if (lane == 0) a.list[0] = moved;
  }
  __syncthreads();
  for (int e = tid; e < E; e += kWalkThreads) a.offsets[E + 2 + e] = s_cnt[e];
  pdl_trigger();
}

struct CopyArgs {
  const void* x;
  void* x_packed;
  const int32_t* list;
  const int32_t* ids;
  const float* zkeys;
  const int32_t* route_row;
  float* gates;
  int d, k, E, C, gate_mode;
};

// One warp per moved route: copy x[t] to its new row of the padded buffer and re-evaluate
// token t's gates (a token with two moved routes is evaluated twice, to the same values).
template <typename T>
__global__ void __launch_bounds__(kThreads) reroute_copy_kernel(CopyArgs a) {
  constexpr int VEC = Vec<T>::N;
  pdl_trigger();
  pdl_wait();
  const int n = a.list[0];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nvec = a.d / VEC;
  for (int i = blockIdx.x * kWarps + warp; i < n; i += gridDim.x * kWarps) {
    const int t = a.list[1 + 2 * i], row = a.list[2 + 2 * i];
    const T* src = static_cast<const T*>(a.x) + static_cast<size_t>(t) * a.d;
    T* dst = static_cast<T*>(a.x_packed) + static_cast<size_t>(row) * a.d;
    for (int v = lane; v < nvec; v += 32) st_vec(dst + v * VEC, ld_vec(src + v * VEC));
    regate(a.ids, a.zkeys, a.route_row, a.gates, t, a.k, a.E, a.C, a.gate_mode, lane);
  }
}

}  // namespace

cudaError_t launch_reroute(const moe_config& c, const void* x, const int32_t* ids,
                           const float* zkeys, float* gates, void* x_packed, int32_t* row_token,
                           int32_t* route_row, int32_t* offsets, int32_t* scratch, int32_t* status,
                           cudaStream_t s) {
  const size_t slots = static_cast<size_t>(c.E) * c.capacity;
  const size_t routes = static_cast<size_t>(c.T) * c.k;
  int32_t* list = scratch;
  int32_t* ag = scratch + 2 * slots + 1;
  (void)routes;
  WalkArgs a{ids, zkeys, row_token, route_row, offsets, list, ag, status, c.T, c.k, c.E,
             c.capacity, kWaitLimitNs};
  cudaError_t e = launch_pdl(reroute_walk_kernel, dim3(1), dim3(kWalkThreads), 0, s, a);
  if (e != cudaSuccess) return e;
  int grid = static_cast<int>((slots + kWarps - 1) / kWarps);
  if (grid > 4 * 148) grid = 4 * 148;
  if (grid < 1) grid = 1;
  const CopyArgs ca{x, x_packed, list, ids, zkeys, route_row, gates, c.d, c.k, c.E, c.capacity,
                    c.gate_mode};
  if (c.dtype == MOE_BF16)
    return launch_pdl(reroute_copy_kernel<__nv_bfloat16>, dim3(grid), dim3(kThreads), 0, s, ca);
  return launch_pdl(reroute_copy_kernel<float>, dim3(grid), dim3(kThreads), 0, s, ca);
}

}  // namespace moe

// Reroute overflow policy on the padded dispatch buffer [E, C, d].
//
// Sources: "Mixture-of-Experts: routing and capacity", Capacity (the buffer has C slots
// per expert; empty slots are padding) and Overflow policies (reroute: the overflowing
// route is handled by the next-best expert by score, the router's decision overridden).
//
// Runs after the arrival-order pack, which has already placed every route that fit and
// left route_row = -1 on the ones that overflowed.  The reroute is sequential by
// definition: whether a route finds a free slot depends on every earlier reroute.  One CTA
// walks the routes in chunks: all threads compact a chunk's overflowed routes (arrival
// order) and stage their tokens' ranking keys and expert ids in shared memory; then one
// warp places them one at a time.  In that warp lane l owns experts l, l+32, ..: it keeps
// their filled-slot counts and the current token's "already held" flags in registers, so a
// placement is a warp max over an order-preserving integer code of the key (free, not held
// experts only) and a warp min of the expert index among the maxima -- the router's order
// and tie rule on the router's own keys -- with no memory round trip on the critical path.
// The walk stops as soon as no slot is free; the loop keeps all its state in registers and
// only issues stores.  A second, grid-wide kernel copies each moved route's token row and
// re-evaluates that token's gates by the gate mode over its final experts.
#include <climits>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kThreads = 256;  // copy kernel
constexpr int kWarps = kThreads / 32;
constexpr int kAssignThreads = 512;
constexpr int kAssignWarps = kAssignThreads / 32;
constexpr int kStageFloats = 16384;  // staged keys per chunk (64 KB)
constexpr int kStageIds = 16384;     // staged expert ids per chunk (64 KB)

struct AssignArgs {
  const int32_t* ids;    // [T, k]
  const float* zkeys;    // [T, E]
  int32_t* row_token;    // [E * C]
  int32_t* route_row;    // [T, k]
  int32_t* offsets;      // segment table; filled-slot counts at offsets[E + 2 + e]
  int32_t* list;         // [0]: moved routes n, then n (token, row) pairs
  int T, k, E, C, chunk;
};

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

// Order-preserving map of a ranking key (never NaN) to a nonzero unsigned code: a larger
// key gives a larger code, -0 and +0 the same one, and -inf the smallest (still > 0).
__device__ __forceinline__ uint32_t key_code(float z) {
  if (z == 0.f) z = 0.f;
  const uint32_t u = __float_as_uint(z);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
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

// QE: experts per lane of the placing warp, ceil(E / 32) rounded up to a power of two.
template <int QE>
__global__ void __launch_bounds__(kAssignThreads, 1) reroute_assign_kernel(AssignArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  float* s_z = reinterpret_cast<float*>(smem);                                  // [chunk][E]
  int* s_ids = reinterpret_cast<int*>(smem + static_cast<size_t>(a.chunk) * a.E * 4);  // [chunk][k]
  __shared__ int s_list[kAssignThreads];
  __shared__ int s_row[kAssignThreads];  // placed row of each listed route, -1 if none
  __shared__ int s_mv[kAssignThreads];   // its index in the list of moved routes
  __shared__ int s_wtot[kAssignWarps];
  __shared__ int s_n, s_done;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int E = a.E, k = a.k, C = a.C;
  // The dependent launch is released only at the end (below): a dependent grid made
  // resident early would share this CTA's SM while the placing warp runs.
  pdl_wait();  // route_row, counts and the keys come from the router and the pack

  // placing warp's state: counts and held flags of experts lane + 32 q
  int cnt[QE];
  bool held[QE];
  int free_total = 0;
  if (warp == 0) {
    int f = 0;
#pragma unroll
    for (int q = 0; q < QE; ++q) {
      const int e = lane + 32 * q;
      cnt[q] = (e < E) ? a.offsets[E + 2 + e] : C;
      held[q] = false;
      f += C - cnt[q];
    }
    free_total = static_cast<int>(__reduce_add_sync(0xffffffffu, static_cast<unsigned>(f)));
    if (lane == 0) s_done = free_total <= 0 ? 1 : 0;
  }
  __syncthreads();

  const int total = a.T * k;  // <= INT_MAX / 2 (validated on the host)
  int cur_t = -1, moved = 0;
  for (int base = 0; base < total && !s_done; base += a.chunk) {
    // 1. overflowed routes of this chunk, in arrival order
    const int r = base + tid;
    bool flag = false;
    if (tid < a.chunk && r < total) {
      const int t = r / k, j = r - t * k;
      const int32_t* row = a.ids + static_cast<size_t>(t) * k;
      flag = a.route_row[r] < 0 && route_id_valid(row, j, row[j], E);
    }
    const uint32_t bal = __ballot_sync(0xffffffffu, flag);
    if (lane == 0) s_wtot[warp] = __popc(bal);
    __syncthreads();
    int before = 0, n = 0;
#pragma unroll
    for (int w = 0; w < kAssignWarps; ++w) {
      before += (w < warp) ? s_wtot[w] : 0;
      n += s_wtot[w];
    }
    if (flag) s_list[before + __popc(bal & ((1u << lane) - 1u))] = r;
    if (tid == 0) s_n = n;
    __syncthreads();

    // 2. stage their tokens' ranking keys and expert ids
    for (int idx = tid; idx < n * E; idx += kAssignThreads) {
      const int i = idx / E, e = idx - i * E;
      s_z[idx] = a.zkeys[static_cast<size_t>(s_list[i] / k) * E + e];
    }
    for (int idx = tid; idx < n * k; idx += kAssignThreads) {
      const int i = idx / k, jj = idx - i * k;
      s_ids[idx] = a.ids[static_cast<size_t>(s_list[i] / k) * k + jj];
    }
    if (tid < n) s_row[tid] = -1;
    __syncthreads();

    // 3. one warp places them in order
    if (warp == 0) {
      for (int i = 0; i < n; ++i) {
        const int rr = s_list[i];
        const int t = rr / k;
        if (t != cur_t) {  // a new token: it holds its own top-k experts
          cur_t = t;
#pragma unroll
          for (int q = 0; q < QE; ++q) held[q] = false;
          for (int jj = 0; jj < k; ++jj) {
            const int e0 = s_ids[i * k + jj];
#pragma unroll
            for (int q = 0; q < QE; ++q) held[q] = held[q] || (e0 == lane + 32 * q);
          }
        }
        uint32_t best = 0u;
        unsigned best_e = 0xffffffffu;
#pragma unroll
        for (int q = 0; q < QE; ++q) {
          const int e = lane + 32 * q;
          if (e < E && !held[q] && cnt[q] < C) {
            const uint32_t code = key_code(s_z[i * E + e]);
            if (code > best) { best = code; best_e = static_cast<unsigned>(e); }
          }
        }
        const uint32_t m = __reduce_max_sync(0xffffffffu, best);
        if (m == 0u) continue;  // no free expert the token does not hold: stays dropped
        const int es = static_cast<int>(__reduce_min_sync(0xffffffffu, best == m ? best_e : 0xffffffffu));
        const int owner = es & 31, qs = es >> 5;
        int slot = 0;
#pragma unroll
        for (int q = 0; q < QE; ++q)
          if (q == qs && lane == owner) { slot = cnt[q]; cnt[q] = slot + 1; held[q] = true; }
        slot = __shfl_sync(0xffffffffu, slot, owner);
        if (lane == 0) {  // results go out after the walk, written by the whole CTA
          s_row[i] = es * C + slot;
          s_mv[i] = moved;
        }
        ++moved;
        if (--free_total == 0) break;
      }
      if (lane == 0) s_done = free_total == 0 ? 1 : 0;
    }
    __syncthreads();
    // 4. write this chunk's placements
    if (tid < n && s_row[tid] >= 0) {
      const int rr = s_list[tid], row = s_row[tid], m = s_mv[tid];
      const int t = rr / k;
      a.route_row[rr] = row;
      a.row_token[row] = t;
      a.list[1 + 2 * m] = t;
      a.list[2 + 2 * m] = row;
    }
  }
  if (warp == 0) {
#pragma unroll
    for (int q = 0; q < QE; ++q)
      if (lane + 32 * q < E) a.offsets[E + 2 + lane + 32 * q] = cnt[q];
    if (lane == 0) a.list[0] = moved;
  }
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
                           int32_t* route_row, int32_t* offsets, int32_t* list, int32_t* status,
                           cudaStream_t s) {
  (void)status;
  int chunk = kAssignThreads;
  if (chunk > kStageFloats / c.E) chunk = kStageFloats / c.E;
  if (chunk > kStageIds / c.k) chunk = kStageIds / c.k;
  AssignArgs a{ids, zkeys, row_token, route_row, offsets, list, c.T, c.k, c.E, c.capacity, chunk};
  const size_t smem = static_cast<size_t>(chunk) * (c.E + c.k) * 4;
  static bool configured = false;
  if (!configured) {
    const int lim = (kStageFloats + kStageIds) * 4;
    cudaFuncSetAttribute(reroute_assign_kernel<1>, cudaFuncAttributeMaxDynamicSharedMemorySize, lim);
    cudaFuncSetAttribute(reroute_assign_kernel<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, lim);
    cudaFuncSetAttribute(reroute_assign_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, lim);
    cudaFuncSetAttribute(reroute_assign_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, lim);
    configured = true;
  }
  cudaError_t e;
  if (c.E <= 32)
    e = launch_pdl(reroute_assign_kernel<1>, dim3(1), dim3(kAssignThreads), smem, s, a);
  else if (c.E <= 64)
    e = launch_pdl(reroute_assign_kernel<2>, dim3(1), dim3(kAssignThreads), smem, s, a);
  else if (c.E <= 128)
    e = launch_pdl(reroute_assign_kernel<4>, dim3(1), dim3(kAssignThreads), smem, s, a);
  else
    e = launch_pdl(reroute_assign_kernel<8>, dim3(1), dim3(kAssignThreads), smem, s, a);
  if (e != cudaSuccess) return e;
  long long slots = static_cast<long long>(c.E) * c.capacity;
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

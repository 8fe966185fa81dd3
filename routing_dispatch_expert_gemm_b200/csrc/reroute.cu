// Reroute overflow policy on the padded dispatch buffer [E, C, d].
//
// Sources: "Mixture-of-Experts: routing and capacity", Capacity (the buffer has C slots
// per expert; empty slots are padding) and Overflow policies (reroute: the overflowing
// route is handled by the next-best expert by score, the router's decision overridden).
//
// Runs after the arrival-order pack, which has already placed every route that fit and
// left route_row = -1 on the ones that overflowed.  The reroute itself is sequential by
// definition: whether a route finds a free slot depends on every earlier reroute.  One CTA
// therefore walks the overflowed routes in arrival order (t, then j): each chunk of 256
// routes is compacted with a block-wide scan, then warp 0 places the chunk's overflowed
// routes one at a time.  For each, the 32 lanes take an arg-max over the experts the token
// does not hold and that still have a free slot, ordered by (ranking key descending, expert
// index ascending), the router's own order and tie rule on the router's own keys.  The walk
// stops as soon as no slot is free.  A token with a moved route gets its gates recomputed by
// the gate mode over its final experts.  A second kernel copies the moved routes' rows.
#include <climits>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

struct AssignArgs {
  const int32_t* ids;    // [T, k]
  const float* zkeys;    // [T, E]
  float* gates;          // [T, k]
  int32_t* row_token;    // [E * C]
  int32_t* route_row;    // [T, k]
  int32_t* offsets;      // segment table; filled-slot counts at offsets[E + 2 + e]
  int32_t* list;         // [0]: moved routes n, then n (token, row) pairs
  int T, k, E, C, gate_mode;
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

// Gates of token t over its final experts fin[0..k) (warp-wide; lane j < k owns slot j).
__device__ void regate(const AssignArgs& a, int t, const int* fin, int lane) {
  const float* zrow = a.zkeys + static_cast<size_t>(t) * a.E;
  const int e = (lane < a.k) ? fin[lane] : -1;
  const bool valid = e >= 0 && e < a.E;
  const float zf = valid ? zrow[e] : -INFINITY;
  float g;
  if (a.gate_mode != MOE_GATE_SOFTMAX_TOPK) {
    // softmax over the final experts' logits.  For the renormalised mode this is
    // p_i / sum_j p_j with the full softmax's normaliser cancelled; shifting by the
    // final experts' own max keeps it finite when the token no longer holds its top
    // expert and every selected p would underflow.
    const float m = warp_max(zf);
    const float ex = valid ? expf(zf - m) : 0.f;
    g = ex / warp_sum(ex);
  } else {  // the full-softmax probability of each final expert
    float m = -INFINITY;
    for (int q = lane; q < a.E; q += 32) m = fmaxf(m, zrow[q]);
    m = warp_max(m);
    float den = 0.f;
    for (int q = lane; q < a.E; q += 32) den += expf(zrow[q] - m);
    den = warp_sum(den);
    g = valid ? expf(zf - m) / den : 0.f;
  }
  if (lane < a.k) a.gates[static_cast<size_t>(t) * a.k + lane] = g;
}

__global__ void __launch_bounds__(kThreads, 1) reroute_assign_kernel(AssignArgs a) {
  __shared__ int s_cnt[256];
  __shared__ int s_list[kThreads];
  __shared__ int s_wtot[kWarps];
  __shared__ uint32_t s_held[8];   // 256-bit set: experts the current token holds
  __shared__ int s_fin[32];        // the current token's expert per slot
  __shared__ int s_n, s_free, s_moved;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int E = a.E, k = a.k, C = a.C;
  pdl_trigger();
  pdl_wait();  // route_row, counts and the keys come from the router and the pack

  for (int e = tid; e < E; e += kThreads) s_cnt[e] = a.offsets[E + 2 + e];
  __syncthreads();
  if (warp == 0) {
    int f = 0;
    for (int e = lane; e < E; e += 32) f += C - s_cnt[e];
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1) f += __shfl_xor_sync(0xffffffffu, f, s);
    if (lane == 0) { s_free = f; s_moved = 0; }
  }
  __syncthreads();

  const int total = a.T * k;  // <= INT_MAX / 2 (validated on the host)
  int cur_t = -1;             // warp 0: token whose routes are being placed
  bool cur_moved = false;
  for (int base = 0; base < total && s_free > 0; base += kThreads) {
    // 1. overflowed routes of this chunk, in arrival order
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
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      before += (w < warp) ? s_wtot[w] : 0;
      n += s_wtot[w];
    }
    if (flag) s_list[before + __popc(bal & ((1u << lane) - 1u))] = r;
    if (tid == 0) s_n = n;
    __syncthreads();

    // 2. warp 0 places them one at a time
    if (warp == 0) {
      for (int i = 0; i < s_n; ++i) {
        __syncwarp();
        if (s_free <= 0) break;
        const int rr = s_list[i];
        const int t = rr / k, j = rr - t * k;
        if (t != cur_t) {
          if (cur_moved) regate(a, cur_t, s_fin, lane);
          cur_t = t;
          cur_moved = false;
          if (lane < 8) s_held[lane] = 0u;
          __syncwarp();
          if (lane < k) {
            const int e = a.ids[static_cast<size_t>(t) * k + lane];
            s_fin[lane] = e;
            if (e >= 0 && e < E) atomicOr(&s_held[e >> 5], 1u << (e & 31));
          }
          __syncwarp();
        }
        const float* zrow = a.zkeys + static_cast<size_t>(t) * E;
        float bv = -INFINITY;
        int be = INT_MAX;  // INT_MAX: no candidate
        for (int e = lane; e < E; e += 32) {
          if (((s_held[e >> 5] >> (e & 31)) & 1u) == 0u && s_cnt[e] < C) {
            const float v = zrow[e];
            if (be == INT_MAX || v > bv || (v == bv && e < be)) { bv = v; be = e; }
          }
        }
#pragma unroll
        for (int s = 16; s >= 1; s >>= 1) {
          const float ov = __shfl_xor_sync(0xffffffffu, bv, s);
          const int oe = __shfl_xor_sync(0xffffffffu, be, s);
          if (oe != INT_MAX && (be == INT_MAX || ov > bv || (ov == bv && oe < be))) {
            bv = ov;
            be = oe;
          }
        }
        if (be != INT_MAX) {  // the same on every lane
          if (lane == 0) {
            const int slot = s_cnt[be];
            s_cnt[be] = slot + 1;
            const int row = be * C + slot;
            a.route_row[rr] = row;
            a.row_token[row] = t;
            const int m = s_moved;
            a.list[1 + 2 * m] = t;
            a.list[2 + 2 * m] = row;
            s_moved = m + 1;
            s_free = s_free - 1;
            s_fin[j] = be;
            s_held[be >> 5] |= 1u << (be & 31);
          }
          cur_moved = true;
        }
      }
      __syncwarp();
    }
    __syncthreads();
  }
  if (warp == 0 && cur_moved) regate(a, cur_t, s_fin, lane);
  __syncthreads();
  for (int e = tid; e < E; e += kThreads) a.offsets[E + 2 + e] = s_cnt[e];
  if (tid == 0) a.list[0] = s_moved;
}

// One warp per moved route: copy x[t] to its new row of the padded buffer.
template <typename T>
__global__ void __launch_bounds__(kThreads) reroute_copy_kernel(const T* __restrict__ x,
                                                                T* __restrict__ xp,
                                                                const int32_t* list, int d) {
  constexpr int VEC = Vec<T>::N;
  pdl_trigger();
  pdl_wait();
  const int n = list[0];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nvec = d / VEC;
  for (int i = blockIdx.x * kWarps + warp; i < n; i += gridDim.x * kWarps) {
    const int t = list[1 + 2 * i], row = list[2 + 2 * i];
    const T* src = x + static_cast<size_t>(t) * d;
    T* dst = xp + static_cast<size_t>(row) * d;
    for (int v = lane; v < nvec; v += 32) st_vec(dst + v * VEC, ld_vec(src + v * VEC));
  }
}

}  // namespace

cudaError_t launch_reroute(const moe_config& c, const void* x, const int32_t* ids,
                           const float* zkeys, float* gates, void* x_packed, int32_t* row_token,
                           int32_t* route_row, int32_t* offsets, int32_t* list, int32_t* status,
                           cudaStream_t s) {
  (void)status;
  AssignArgs a{ids, zkeys, gates, row_token, route_row, offsets, list,
               c.T, c.k, c.E, c.capacity, c.gate_mode};
  cudaError_t e = launch_pdl(reroute_assign_kernel, dim3(1), dim3(kThreads), 0, s, a);
  if (e != cudaSuccess) return e;
  long long slots = static_cast<long long>(c.E) * c.capacity;
  int grid = static_cast<int>((slots + kWarps - 1) / kWarps);
  if (grid > 4 * 148) grid = 4 * 148;
  if (grid < 1) grid = 1;
  if (c.dtype == MOE_BF16)
    return launch_pdl(reroute_copy_kernel<__nv_bfloat16>, dim3(grid), dim3(kThreads), 0, s,
                      static_cast<const __nv_bfloat16*>(x), static_cast<__nv_bfloat16*>(x_packed),
                      static_cast<const int32_t*>(list), c.d);
  return launch_pdl(reroute_copy_kernel<float>, dim3(grid), dim3(kThreads), 0, s,
                    static_cast<const float*>(x), static_cast<float*>(x_packed),
                    static_cast<const int32_t*>(list), c.d);
}

}  // namespace moe

// Reroute overflow policy on the padded dispatch buffer [E, C, d].
//
// Sources: "Mixture-of-Experts: routing and capacity", Capacity (the buffer has C slots
// per expert; empty slots are padding) and Overflow policies (reroute: the overflowing
// route is handled by the next-best expert by score, the router's decision overridden).
//
// Runs after the arrival-order pack, which has already placed every route that fit and
// left route_row = -1 on the ones that overflowed.  The reroute is sequential by definition
// (whether a route finds a free slot depends on every earlier reroute), but because every
// expert ranks routes by arrival order the result can be built in phases (see
// reroute_phase_kernel), one CTA, at most E + 1 phases.  A second, grid-wide kernel copies
// each moved route's token row and re-evaluates that token's gates by the gate mode over its
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
// Phased placement.  Every expert ranks the overflowed routes by arrival order, so the
// sequential walk is reproduced exactly in phases: each pending route proposes the expert
// it would take if the experts full at the phase start were the only full ones (its
// token's best-ranked expert that it does not hold and that is not full, or the next-best
// one after the token's earlier routes of the same phase); a scan in arrival order counts
// each expert's proposals and finds the first route whose expert has run out of slots.
// Every route before it is placed exactly as the walk would place it.  The phase then
// restarts at that route with at least one more expert full, so there are at most E + 1
// phases.  Only routes whose proposal became full (and the later routes of the same
// token) re-choose.
// ---------------------------------------------------------------------------------
constexpr int kPhThreads = 1024;
constexpr int kPhWarps = kPhThreads / 32;

struct PhaseArgs {
  const int32_t* ids;      // [T, k]
  const float* zkeys;      // [T, E]
  int32_t* row_token;      // [E * C]
  int32_t* route_row;      // [T, k]
  int32_t* offsets;        // filled-slot counts at offsets[E + 2 + e]
  int32_t* list;           // [0]: moved routes n, then (token, row) pairs
  int32_t* ag_r;           // [T * k] overflowed routes (flat index), arrival order
  int32_t* ag_c;           // [T * k] proposed / final expert, -1: none
  int32_t* ag_rank;        // [T * k] rank among the phase's proposals to the same expert
  int32_t* ag_st;          // [T * k] proposal went stale at the end of the phase
  int T, k, E, C;
};

__device__ __forceinline__ bool bit_of(const uint32_t (&w)[8], int e) {
  uint32_t v = 0;
#pragma unroll
  for (int q = 0; q < 8; ++q) v = (q == (e >> 5)) ? w[q] : v;
  return (v >> (e & 31)) & 1u;
}
__device__ __forceinline__ void set_bit(uint32_t (&w)[8], int e) {
#pragma unroll
  for (int q = 0; q < 8; ++q)
    if (q == (e >> 5)) w[q] |= 1u << (e & 31);
}

// The expert route i proposes when the phase starts at `pos` and s_full marks full experts.
__device__ int propose(const PhaseArgs& a, int i, int pos, const uint32_t* s_full) {
  const int t = a.ag_r[i] / a.k;
  uint32_t held[8];
#pragma unroll
  for (int q = 0; q < 8; ++q) held[q] = s_full[q];
  for (int jj = 0; jj < a.k; ++jj) {
    const int e = a.ids[static_cast<size_t>(t) * a.k + jj];
    if (e >= 0 && e < a.E) set_bit(held, e);
  }
  int m = 0;  // the token's earlier routes still pending in this phase
  for (int q = i - 1; q >= 0 && a.ag_r[q] / a.k == t; --q) {
    if (q >= pos) {
      ++m;
    } else {
      const int cq = a.ag_c[q];
      if (cq >= 0) set_bit(held, cq);
    }
  }
  const float* zrow = a.zkeys + static_cast<size_t>(t) * a.E;
  int pick = -1;
  for (int round = 0; round <= m; ++round) {
    float bv = -INFINITY;
    int be = -1;
    for (int e = 0; e < a.E; ++e) {
      if (bit_of(held, e)) continue;
      const float v = zrow[e];
      if (be < 0 || v > bv) { bv = v; be = e; }  // strict: equal keys keep the lower index
    }
    if (be < 0) return -1;
    set_bit(held, be);
    pick = be;
  }
  return pick;
}

__global__ void __launch_bounds__(kPhThreads, 1) reroute_phase_kernel(PhaseArgs a) {
  __shared__ int s_cnt[256], s_carry[256], s_inc[256];
  __shared__ int s_wc[kPhWarps][256];  // per-warp proposal counts per expert, then bases
  __shared__ uint32_t s_full[8];
  __shared__ int s_wtot[kPhWarps];
  __shared__ int s_n, s_istar, s_moved;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int E = a.E, k = a.k, C = a.C;
  pdl_wait();  // route_row, counts and the keys come from the router and the pack

  for (int e = tid; e < 256; e += kPhThreads) {
    s_cnt[e] = (e < E) ? a.offsets[E + 2 + e] : C;
    s_inc[e] = 0;
  }
  if (tid == 0) { s_n = 0; s_moved = 0; }
  __syncthreads();

  // 1. overflowed routes, arrival order
  const int total = a.T * k;  // <= INT_MAX / 2 (validated on the host)
  for (int base = 0; base < total; base += kPhThreads) {
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
    for (int w = 0; w < kPhWarps; ++w) {
      before += (w < warp) ? s_wtot[w] : 0;
      n += s_wtot[w];
    }
    if (flag) a.ag_r[s_n + before + __popc(bal & ((1u << lane) - 1u))] = r;
    __syncthreads();
    if (tid == 0) s_n += n;
    __syncthreads();
  }
  const int n = s_n;
  if (tid < 8) {
    uint32_t w = 0;
    for (int b = 0; b < 32; ++b) {
      const int e = tid * 32 + b;
      if (e >= E || s_cnt[e] >= C) w |= 1u << b;
    }
    s_full[tid] = w;
  }
  __syncthreads();

  // 2. first proposals (a token's routes are consecutive, each counts its earlier ones)
  for (int i = tid; i < n; i += kPhThreads) a.ag_c[i] = propose(a, i, 0, s_full);
  __syncthreads();

  // 3. phases
  int pos = 0;
  while (pos < n) {
    for (int e = tid; e < 256; e += kPhThreads) s_carry[e] = 0;
    if (tid == 0) s_istar = n;
    __syncthreads();
    for (int base = pos; base < n; base += kPhThreads) {
      for (int x = tid; x < kPhWarps * 256; x += kPhThreads) (&s_wc[0][0])[x] = 0;
      __syncthreads();
      const int i = base + tid;
      const int c = (i < n) ? a.ag_c[i] : -1;
      const uint32_t peers = __match_any_sync(0xffffffffu, c);
      const int wrank = __popc(peers & ((1u << lane) - 1u));
      if (c >= 0 && wrank == 0) s_wc[warp][c] = __popc(peers);
      __syncthreads();
      for (int e = tid; e < E; e += kPhThreads) {  // exclusive prefix over warps
        int run = s_carry[e];
        for (int w = 0; w < kPhWarps; ++w) {
          const int v = s_wc[w][e];
          s_wc[w][e] = run;
          run += v;
        }
        s_carry[e] = run;
      }
      __syncthreads();
      if (c >= 0) {
        const int rank = s_wc[warp][c] + wrank;
        a.ag_rank[i] = rank;
        if (s_cnt[c] + rank >= C) atomicMin(&s_istar, i);
      }
      __syncthreads();
      if (s_istar < n) break;
    }
    const int istar = s_istar;
    // commit the routes before istar
    for (int i = pos + tid; i < istar; i += kPhThreads) {
      const int c = a.ag_c[i];
      if (c < 0) continue;
      const int r = a.ag_r[i], t = r / k;
      const int row = c * C + s_cnt[c] + a.ag_rank[i];
      a.route_row[r] = row;
      a.row_token[row] = t;
      const int m = atomicAdd(&s_moved, 1);
      a.list[1 + 2 * m] = t;
      a.list[2 + 2 * m] = row;
      atomicAdd(&s_inc[c], 1);
    }
    __syncthreads();
    for (int e = tid; e < E; e += kPhThreads) {
      s_cnt[e] += s_inc[e];
      s_inc[e] = 0;
    }
    __syncthreads();
    if (tid < 8) {
      uint32_t w = 0;
      for (int b = 0; b < 32; ++b) {
        const int e = tid * 32 + b;
        if (e >= E || s_cnt[e] >= C) w |= 1u << b;
      }
      s_full[tid] = w;
    }
    __syncthreads();
    pos = istar;
    if (pos >= n) break;
    // stale proposals: their expert filled up; later routes of the same token follow them
    for (int i = pos + tid; i < n; i += kPhThreads) {
      const int c = a.ag_c[i];
      a.ag_st[i] = (c >= 0 && ((s_full[c >> 5] >> (c & 31)) & 1u)) ? 1 : 0;
    }
    __syncthreads();
    for (int i = pos + tid; i < n; i += kPhThreads) {
      const int t = a.ag_r[i] / k;
      bool redo = a.ag_st[i] != 0;
      for (int q = i - 1; !redo && q >= pos && a.ag_r[q] / k == t; --q) redo = a.ag_st[q] != 0;
      if (redo) a.ag_c[i] = propose(a, i, pos, s_full);
    }
    __syncthreads();
  }
  for (int e = tid; e < E; e += kPhThreads) a.offsets[E + 2 + e] = s_cnt[e];
  if (tid == 0) a.list[0] = s_moved;
  __syncthreads();
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
  (void)status;
  const size_t slots = static_cast<size_t>(c.E) * c.capacity;
  const size_t routes = static_cast<size_t>(c.T) * c.k;
  int32_t* list = scratch;
  int32_t* ag = scratch + 2 * slots + 1;
  PhaseArgs a{ids, zkeys, row_token, route_row, offsets, list, ag, ag + routes, ag + 2 * routes,
              ag + 3 * routes, c.T, c.k, c.E, c.capacity};
  cudaError_t e = launch_pdl(reroute_phase_kernel, dim3(1), dim3(kPhThreads), 0, s, a);
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

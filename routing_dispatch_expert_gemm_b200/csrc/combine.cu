// Combine: y[t] = sum_j g[t,j] * Y[route_row[t,j]] (+ shared expert row) (+ residual x[t]).
//
// Sources: "271,104 Routes: What I Missed About Mixture-of-Experts", section 1 (y = sum
// over selected experts of p_i E_i(x)) and section 3 (apply the gate weights, add, and
// restore the original token order); "MoE Inference Visualized", Expert Execution
// (scale by the router weight, scatter back to sequence positions); "Mixture-of-Experts:
// routing and capacity", Top-k and mixture (output = weighted sum + shared + residual).
//
// Each output element gathers its token's k expert rows by route_row (the inverse of the
// packing permutation), so the sum needs no atomics and its order is fixed: fp32, slots
// j = 0..k-1, then the shared expert, then the residual; one rounding to the output type.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kWarpTokensMin = 2048;  // below this many tokens, one thread per 16-byte vector

struct CombineArgs {
  const void* y_packed;
  const int32_t* route_row;
  const float* gates;
  const int32_t* offsets;
  const void* residual;
  void* y;
  int T, d, k, E, has_shared, tpc;
  int32_t* status;
};

// Few tokens, k <= 8: one thread per (token, 16-byte vector) with the token's k rows and
// gates in registers, loaded straight from global memory (the threads of a warp share a
// token, so the loads are broadcasts), and the shared-expert and residual rows requested
// before the gathers since they do not depend on the route table.  Same arithmetic and
// order as combine_warp_kernel.
template <typename T, int KMAX>
__global__ void __launch_bounds__(kThreads) combine_reg_kernel(CombineArgs a) {
  constexpr int VEC = Vec<T>::N;
  pdl_trigger();
  pdl_wait();
  const int nvec = a.d / VEC;
  const long long idx = static_cast<long long>(blockIdx.x) * kThreads + threadIdx.x;
  if (idx >= static_cast<long long>(a.T) * nvec) return;
  const int t = static_cast<int>(idx / nvec), c = static_cast<int>(idx - static_cast<long long>(t) * nvec);
  const T* __restrict__ Y = static_cast<const T*>(a.y_packed);
  const T* __restrict__ R = static_cast<const T*>(a.residual);
  int rows[KMAX];
  float g[KMAX];
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    rows[j] = (j < a.k) ? __ldg(a.route_row + static_cast<size_t>(t) * a.k + j) : -1;
    g[j] = (j < a.k) ? __ldg(a.gates + static_cast<size_t>(t) * a.k + j) : 0.f;
  }
  const uint4 rv = (R != nullptr) ? ld_vec(R + static_cast<size_t>(t) * a.d + c * VEC) : make_uint4(0, 0, 0, 0);
  uint4 sv = make_uint4(0, 0, 0, 0);
  if (a.has_shared) {
    const int shared_base = __ldg(a.offsets + a.E);
    sv = ld_vec(Y + static_cast<size_t>(shared_base + t) * a.d + c * VEC);
  }
  uint4 v[KMAX];
#pragma unroll
  for (int j = 0; j < KMAX; ++j)
    v[j] = (rows[j] >= 0) ? ld_vec(Y + static_cast<size_t>(rows[j]) * a.d + c * VEC) : make_uint4(0, 0, 0, 0);
  float acc[VEC];
#pragma unroll
  for (int q = 0; q < VEC; ++q) acc[q] = 0.f;
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    if (rows[j] >= 0) {  // a dropped route contributes nothing
      float f[VEC];
      Vec<T>::to_f32(v[j], f);
#pragma unroll
      for (int q = 0; q < VEC; ++q) acc[q] = fmaf(g[j], f[q], acc[q]);
    }
  }
  if (a.has_shared) {
    float f[VEC];
    Vec<T>::to_f32(sv, f);
#pragma unroll
    for (int q = 0; q < VEC; ++q) acc[q] += f[q];
  }
  if (R != nullptr) {
    float f[VEC];
    Vec<T>::to_f32(rv, f);
#pragma unroll
    for (int q = 0; q < VEC; ++q) acc[q] += f[q];
  }
  st_vec(static_cast<T*>(a.y) + static_cast<size_t>(t) * a.d + c * VEC, Vec<T>::from_f32(acc));
}

// One warp per token (k <= 32): the token's route rows and gates sit in lanes 0..k-1 and
// are broadcast with shuffles; each pass over the row gathers NV 16-byte vectors per lane
// from each kept route row, the shared-expert row and the residual row (all requested
// before any is used), then sums them in the fixed order: fp32, slots j = 0..k-1, then the
// shared expert, then the residual; one rounding.  A warp's loads of one row are 512
// contiguous bytes, and every warp of the grid runs at once, so the gathers keep many
// bytes in flight per SM.
template <typename T, int KMAX>
__global__ void __launch_bounds__(kThreads) combine_warp_kernel(CombineArgs a) {
  constexpr int VEC = Vec<T>::N;
  constexpr int NV = KMAX <= 4 ? 4 : (KMAX <= 8 ? 2 : 1);  // vectors per lane per pass
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  pdl_trigger();
  pdl_wait();
  const int t = blockIdx.x * (kThreads / 32) + warp;
  if (t >= a.T) return;
  const int k = a.k;
  int my_row = -1;
  float my_g = 0.f;
  if (lane < k) {
    my_row = __ldg(a.route_row + static_cast<size_t>(t) * k + lane);
    my_g = __ldg(a.gates + static_cast<size_t>(t) * k + lane);
  }
  const int shared_base = a.has_shared ? __ldg(a.offsets + a.E) : -1;
  int rows[KMAX];
  float g[KMAX];
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    rows[j] = __shfl_sync(0xffffffffu, my_row, j);
    g[j] = __shfl_sync(0xffffffffu, my_g, j);
    if (j >= k) rows[j] = -1;
  }
  const uint4* __restrict__ Y = static_cast<const uint4*>(a.y_packed);
  const uint4* __restrict__ R = static_cast<const uint4*>(a.residual);
  uint4* __restrict__ out = static_cast<uint4*>(a.y);
  const int nvec = a.d / VEC;  // 16-byte vectors per row
  for (int base = 0; base < nvec; base += 32 * NV) {
    uint4 rv[NV], sv[NV], v[KMAX][NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int idx = base + i * 32 + lane;
      const bool in = idx < nvec;
      rv[i] = (in && R != nullptr) ? ld_vec(R + static_cast<size_t>(t) * nvec + idx) : make_uint4(0, 0, 0, 0);
      sv[i] = (in && shared_base >= 0) ? ld_vec(Y + static_cast<size_t>(shared_base + t) * nvec + idx)
                                       : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int j = 0; j < KMAX; ++j)
        v[j][i] = (in && rows[j] >= 0) ? ld_vec(Y + static_cast<size_t>(rows[j]) * nvec + idx)
                                       : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const int idx = base + i * 32 + lane;
      if (idx >= nvec) continue;
      float acc[VEC];
#pragma unroll
      for (int q = 0; q < VEC; ++q) acc[q] = 0.f;
#pragma unroll
      for (int j = 0; j < KMAX; ++j) {
        if (rows[j] >= 0) {  // a dropped route contributes nothing
          float f[VEC];
          Vec<T>::to_f32(v[j][i], f);
#pragma unroll
          for (int q = 0; q < VEC; ++q) acc[q] = fmaf(g[j], f[q], acc[q]);
        }
      }
      if (shared_base >= 0) {
        float f[VEC];
        Vec<T>::to_f32(sv[i], f);
#pragma unroll
        for (int q = 0; q < VEC; ++q) acc[q] += f[q];
      }
      if (R != nullptr) {
        float f[VEC];
        Vec<T>::to_f32(rv[i], f);
#pragma unroll
        for (int q = 0; q < VEC; ++q) acc[q] += f[q];
      }
      out[static_cast<size_t>(t) * nvec + idx] = Vec<T>::from_f32(acc);
    }
  }
}

template <typename T>
cudaError_t launch_warp(const CombineArgs& a, cudaStream_t s) {
  const int grid = (a.T + kThreads / 32 - 1) / (kThreads / 32);
  const dim3 g(grid), b(kThreads);
  if (a.k <= 1) return launch_pdl(combine_warp_kernel<T, 1>, g, b, 0, s, a);
  if (a.k <= 2) return launch_pdl(combine_warp_kernel<T, 2>, g, b, 0, s, a);
  if (a.k <= 4) return launch_pdl(combine_warp_kernel<T, 4>, g, b, 0, s, a);
  if (a.k <= 8) return launch_pdl(combine_warp_kernel<T, 8>, g, b, 0, s, a);
  if (a.k <= 16) return launch_pdl(combine_warp_kernel<T, 16>, g, b, 0, s, a);
  return launch_pdl(combine_warp_kernel<T, 32>, g, b, 0, s, a);
}

template <typename T>
cudaError_t launch_reg(const CombineArgs& a, int nvec, cudaStream_t s) {
  const long long threads = static_cast<long long>(a.T) * nvec;
  const int grid = static_cast<int>((threads + kThreads - 1) / kThreads);
  if (a.k <= 1) return launch_pdl(combine_reg_kernel<T, 1>, dim3(grid), dim3(kThreads), 0, s, a);
  if (a.k <= 2) return launch_pdl(combine_reg_kernel<T, 2>, dim3(grid), dim3(kThreads), 0, s, a);
  if (a.k <= 4) return launch_pdl(combine_reg_kernel<T, 4>, dim3(grid), dim3(kThreads), 0, s, a);
  return launch_pdl(combine_reg_kernel<T, 8>, dim3(grid), dim3(kThreads), 0, s, a);
}

}  // namespace

cudaError_t launch_combine(const moe_config& c, const void* y_packed, const int32_t* route_row,
                           const float* gates, const int32_t* offsets, const void* residual,
                           void* y, cudaStream_t s) {
  CombineArgs a{y_packed, route_row, gates, offsets, c.add_residual ? residual : nullptr,
                y, c.T, c.d, c.k, c.E, c.has_shared, 1, nullptr};
  // Few tokens (decode): a warp per token leaves most SMs idle, so each thread takes one
  // 16-byte vector of one token instead (T * d / 8 threads).  Otherwise a warp per token.
  if (c.T < kWarpTokensMin && c.k <= 8) {
    const int nvec = c.d / (c.dtype == MOE_BF16 ? 8 : 4);
    if (c.dtype == MOE_BF16) return launch_reg<__nv_bfloat16>(a, nvec, s);
    return launch_reg<float>(a, nvec, s);
  }
  if (c.dtype == MOE_BF16) return launch_warp<__nv_bfloat16>(a, s);
  return launch_warp<float>(a, s);
}

}  // namespace moe

// Combine: y[t] = sum_j g[t,j] * Y[route_row[t,j]] (+ shared expert row) (+ residual x[t]).
//
// Sources: "271,104 Routes: What I Missed About Mixture-of-Experts", section 1 (y = sum
// over selected experts of p_i E_i(x)) and section 3 (apply the gate weights, add, and
// restore the original token order); "MoE Inference Visualized", Expert Execution
// (scale by the router weight, scatter back to sequence positions); "Mixture-of-Experts:
// routing and capacity", Top-k and mixture (output = weighted sum + shared + residual).
//
// One warp per token gathers its k expert rows by route_row (the inverse of the packing
// permutation), so the sum needs no atomics and its order is fixed: fp32, slots
// j = 0..k-1, then the shared expert, then the residual; one rounding to the output type.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

struct CombineArgs {
  const void* y_packed;
  const int32_t* route_row;
  const float* gates;
  const int32_t* offsets;
  const void* residual;
  void* y;
  int T, d, k, E, has_shared;
};

template <typename T>
__global__ void __launch_bounds__(kThreads) combine_kernel(CombineArgs a) {
  constexpr int VEC = Vec<T>::N;
  __shared__ int s_row[kWarps][32];
  __shared__ float s_g[kWarps][32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * kWarps + warp;
  if (t >= a.T) return;  // warp-uniform; no block-level sync below

  if (lane < a.k) {
    s_row[warp][lane] = __ldg(a.route_row + static_cast<size_t>(t) * a.k + lane);
    s_g[warp][lane] = __ldg(a.gates + static_cast<size_t>(t) * a.k + lane);
  }
  __syncwarp();
  const T* __restrict__ Y = static_cast<const T*>(a.y_packed);
  const T* __restrict__ R = static_cast<const T*>(a.residual);
  T* __restrict__ out = static_cast<T*>(a.y);
  const int shared_row = a.has_shared ? __ldg(a.offsets + a.E) + t : -1;
  const int nvec = a.d / VEC;

  for (int c = lane; c < nvec; c += 32) {
    float acc[VEC];
#pragma unroll
    for (int q = 0; q < VEC; ++q) acc[q] = 0.f;
    for (int j = 0; j < a.k; ++j) {
      const int r = s_row[warp][j];
      if (r < 0) continue;  // dropped route contributes nothing
      const float g = s_g[warp][j];
      float f[VEC];
      Vec<T>::to_f32(ld_vec(Y + static_cast<size_t>(r) * a.d + c * VEC), f);
#pragma unroll
      for (int q = 0; q < VEC; ++q) acc[q] = fmaf(g, f[q], acc[q]);
    }
    if (shared_row >= 0) {
      float f[VEC];
      Vec<T>::to_f32(ld_vec(Y + static_cast<size_t>(shared_row) * a.d + c * VEC), f);
#pragma unroll
      for (int q = 0; q < VEC; ++q) acc[q] += f[q];
    }
    if (R != nullptr) {
      float f[VEC];
      Vec<T>::to_f32(ld_vec(R + static_cast<size_t>(t) * a.d + c * VEC), f);
#pragma unroll
      for (int q = 0; q < VEC; ++q) acc[q] += f[q];
    }
    st_vec(out + static_cast<size_t>(t) * a.d + c * VEC, Vec<T>::from_f32(acc));
  }
}

}  // namespace

cudaError_t launch_combine(const moe_config& c, const void* y_packed, const int32_t* route_row,
                           const float* gates, const int32_t* offsets, const void* residual,
                           void* y, cudaStream_t s) {
  CombineArgs a{y_packed, route_row, gates, offsets, c.add_residual ? residual : nullptr,
                y, c.T, c.d, c.k, c.E, c.has_shared};
  const int grid = (c.T + kWarps - 1) / kWarps;
  if (c.dtype == MOE_BF16)
    combine_kernel<__nv_bfloat16><<<grid, kThreads, 0, s>>>(a);
  else
    combine_kernel<float><<<grid, kThreads, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace moe

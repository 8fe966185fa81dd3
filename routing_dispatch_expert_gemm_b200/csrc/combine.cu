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
constexpr int kMaxTok = 32;   // tokens per CTA (upper bound)
constexpr int kBatch = 8;     // gathers issued together per thread

struct CombineArgs {
  const void* y_packed;
  const int32_t* route_row;
  const float* gates;
  const int32_t* offsets;
  const void* residual;
  void* y;
  int T, d, k, E, has_shared, tpc;
};

// A CTA handles `tpc` tokens; each thread owns one 16-byte vector of one token's output
// and issues the gathers of kBatch routes at once, so up to kBatch loads are in flight
// per thread (the pass is bound by memory latency otherwise).
template <typename T>
__global__ void __launch_bounds__(kThreads) combine_kernel(CombineArgs a) {
  constexpr int VEC = Vec<T>::N;
  __shared__ int s_row[kMaxTok][32];
  __shared__ float s_g[kMaxTok][32];
  const int t0 = blockIdx.x * a.tpc;
  const int ntok = min(a.tpc, a.T - t0);
  pdl_trigger();
  pdl_wait();
  for (int i = threadIdx.x; i < ntok * a.k; i += kThreads) {
    const int tl = i / a.k, j = i - tl * a.k;
    s_row[tl][j] = __ldg(a.route_row + static_cast<size_t>(t0) * a.k + i);
    s_g[tl][j] = __ldg(a.gates + static_cast<size_t>(t0) * a.k + i);
  }
  const int shared_base = a.has_shared ? __ldg(a.offsets + a.E) : -1;
  __syncthreads();

  const T* __restrict__ Y = static_cast<const T*>(a.y_packed);
  const T* __restrict__ R = static_cast<const T*>(a.residual);
  T* __restrict__ out = static_cast<T*>(a.y);
  const int nvec = a.d / VEC;
  for (int idx = threadIdx.x; idx < ntok * nvec; idx += kThreads) {
    const int tl = idx / nvec, c = idx - tl * nvec;
    const int t = t0 + tl;
    float acc[VEC];
#pragma unroll
    for (int q = 0; q < VEC; ++q) acc[q] = 0.f;
    for (int j0 = 0; j0 < a.k; j0 += kBatch) {
      uint4 v[kBatch];
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int j = j0 + u;
        const int r = (j < a.k) ? s_row[tl][j] : -1;
        v[u] = (r >= 0) ? ld_vec(Y + static_cast<size_t>(r) * a.d + c * VEC) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < kBatch; ++u) {
        const int j = j0 + u;
        if (j < a.k && s_row[tl][j] >= 0) {  // a dropped route contributes nothing
          const float g = s_g[tl][j];
          float f[VEC];
          Vec<T>::to_f32(v[u], f);
#pragma unroll
          for (int q = 0; q < VEC; ++q) acc[q] = fmaf(g, f[q], acc[q]);
        }
      }
    }
    if (shared_base >= 0) {
      float f[VEC];
      Vec<T>::to_f32(ld_vec(Y + static_cast<size_t>(shared_base + t) * a.d + c * VEC), f);
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
  const int vec = (c.dtype == MOE_BF16) ? 8 : 4;
  const int nvec = c.d / vec;
  int tpc = kThreads / nvec;
  tpc = tpc < 1 ? 1 : (tpc > kMaxTok ? kMaxTok : tpc);
  CombineArgs a{y_packed, route_row, gates, offsets, c.add_residual ? residual : nullptr,
                y, c.T, c.d, c.k, c.E, c.has_shared, tpc};
  const int grid = (c.T + tpc - 1) / tpc;
  static bool configured = false;
  if (!configured) {
    prefer_max_shared(combine_kernel<__nv_bfloat16>);
    prefer_max_shared(combine_kernel<float>);
    configured = true;
  }
  if (c.dtype == MOE_BF16)
    return launch_pdl(combine_kernel<__nv_bfloat16>, dim3(grid), dim3(kThreads), 0, s, a);
  return launch_pdl(combine_kernel<float>, dim3(grid), dim3(kThreads), 0, s, a);
}

}  // namespace moe

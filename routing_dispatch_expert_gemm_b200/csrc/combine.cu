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
constexpr size_t kBulkSmemMax = 192 * 1024;  // double buffer of a token's rows
constexpr int kBatch = 8;     // gathers issued together per thread

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

// Combine on the bulk-copy engine.  A CTA handles `tpc` tokens one after another with a
// two-buffer pipeline: while the threads reduce token i from shared memory, the rows of
// token i+1 (its kept routes' expert outputs, the shared-expert row and the residual row)
// are already streaming in as whole-row bulk copies.  Same arithmetic and order as
// combine_kernel: fp32, slots j = 0..k-1, then shared, then residual, one rounding.
constexpr int kMaxTokBulk = 16;

template <typename T>
__global__ void __launch_bounds__(256) combine_bulk_kernel(CombineArgs a) {
  constexpr int VEC = Vec<T>::N;
  __shared__ int s_row[kMaxTokBulk][32];
  __shared__ float s_g[kMaxTokBulk][32];
  __shared__ __align__(8) uint64_t s_full[2];
  extern __shared__ __align__(128) uint8_t s_buf[];  // 2 x (k + 2) rows
  const int tid = threadIdx.x;
  const int t0 = blockIdx.x * a.tpc;
  const int ntok = min(a.tpc, a.T - t0);
  const int slots = a.k + 2;  // k routed rows, shared row, residual row
  const uint32_t row_bytes = static_cast<uint32_t>(a.d) * sizeof(T);
  if (tid == 0) {
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    fence_mbar_init();
  }
  pdl_trigger();
  pdl_wait();
  for (int i = tid; i < ntok * a.k; i += blockDim.x) {
    const int tl = i / a.k, j = i - tl * a.k;
    s_row[tl][j] = __ldg(a.route_row + static_cast<size_t>(t0) * a.k + i);
    s_g[tl][j] = __ldg(a.gates + static_cast<size_t>(t0) * a.k + i);
  }
  const int shared_base = a.has_shared ? __ldg(a.offsets + a.E) : -1;
  __syncthreads();

  const T* __restrict__ Y = static_cast<const T*>(a.y_packed);
  const T* __restrict__ R = static_cast<const T*>(a.residual);
  T* __restrict__ out = static_cast<T*>(a.y);
  auto issue = [&](int tl, int b) {  // thread 0: bulk loads of token tl's rows into buffer b
    uint8_t* buf = s_buf + static_cast<size_t>(b) * slots * row_bytes;
    const int t = t0 + tl;
    uint32_t bytes = 0;
    for (int j = 0; j < a.k; ++j) bytes += (s_row[tl][j] >= 0) ? row_bytes : 0;
    if (shared_base >= 0) bytes += row_bytes;
    if (R != nullptr) bytes += row_bytes;
    mbar_arrive_expect_tx(&s_full[b], bytes);
    for (int j = 0; j < a.k; ++j) {
      const int r = s_row[tl][j];
      if (r >= 0) bulk_load(buf + j * row_bytes, Y + static_cast<size_t>(r) * a.d, row_bytes, &s_full[b]);
    }
    if (shared_base >= 0)
      bulk_load(buf + a.k * row_bytes, Y + static_cast<size_t>(shared_base + t) * a.d, row_bytes,
                &s_full[b]);
    if (R != nullptr)
      bulk_load(buf + (a.k + 1) * row_bytes, R + static_cast<size_t>(t) * a.d, row_bytes, &s_full[b]);
  };
  if (tid == 0) {
    issue(0, 0);
    if (ntok > 1) issue(1, 1);
  }
  const int nvec = a.d / VEC;
  for (int tl = 0; tl < ntok; ++tl) {
    const int b = tl & 1;
    if (!mbar_wait_bounded(&s_full[b], (tl >> 1) & 1, nullptr, kWaitLimitNs, nullptr)) {
      // unreachable in practice (bounded by the copy engine); leave the token unwritten
      if (tid == 0) record_status(a.status, MOE_ERR_TIMEOUT);
    }
    const uint8_t* buf = s_buf + static_cast<size_t>(b) * slots * row_bytes;
    const int t = t0 + tl;
    for (int c = tid; c < nvec; c += blockDim.x) {
      float acc[VEC];
#pragma unroll
      for (int q = 0; q < VEC; ++q) acc[q] = 0.f;
      for (int j = 0; j < a.k; ++j) {
        if (s_row[tl][j] < 0) continue;  // a dropped route contributes nothing
        const float g = s_g[tl][j];
        float f[VEC];
        Vec<T>::to_f32(*reinterpret_cast<const uint4*>(buf + j * row_bytes + c * 16), f);
#pragma unroll
        for (int q = 0; q < VEC; ++q) acc[q] = fmaf(g, f[q], acc[q]);
      }
      if (shared_base >= 0) {
        float f[VEC];
        Vec<T>::to_f32(*reinterpret_cast<const uint4*>(buf + a.k * row_bytes + c * 16), f);
#pragma unroll
        for (int q = 0; q < VEC; ++q) acc[q] += f[q];
      }
      if (R != nullptr) {
        float f[VEC];
        Vec<T>::to_f32(*reinterpret_cast<const uint4*>(buf + (a.k + 1) * row_bytes + c * 16), f);
#pragma unroll
        for (int q = 0; q < VEC; ++q) acc[q] += f[q];
      }
      st_vec(out + static_cast<size_t>(t) * a.d + c * VEC, Vec<T>::from_f32(acc));
    }
    __syncthreads();  // everyone is done with buffer b
    if (tid == 0 && tl + 2 < ntok) {
      fence_proxy_async_smem();  // the reads above happen before the copy engine rewrites b
      issue(tl + 2, b);
    }
  }
}

// Small k (<= 8): one thread per (token, 16-byte vector) with the token's k rows and gates
// in registers, loaded straight from global memory (the threads of a warp share a token, so
// the loads are broadcasts), and the shared-expert and residual rows requested before the
// gathers since they do not depend on the route table.  Same arithmetic and order as
// combine_kernel.
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
  const int vec = (c.dtype == MOE_BF16) ? 8 : 4;
  const int nvec = c.d / vec;
  const size_t row_bytes = static_cast<size_t>(c.d) * (c.dtype == MOE_BF16 ? 2 : 4);
  const size_t bulk_smem = 2 * static_cast<size_t>(c.k + 2) * row_bytes;
  // Whole-row bulk copies pay off for long rows (measured: d = 4096 bf16 faster, d <= 1024
  // slower than the thread-level gather); they also need the double buffer to fit.
  if (row_bytes >= 4096 && bulk_smem <= kBulkSmemMax) {
    // about two CTAs per SM worth of tokens, at most kMaxTokBulk per CTA
    int tpc = c.T / 296;
    tpc = tpc < 1 ? 1 : (tpc > kMaxTokBulk ? kMaxTokBulk : tpc);
    const int threads = nvec <= 128 ? 128 : 256;
    CombineArgs a{y_packed, route_row, gates, offsets, c.add_residual ? residual : nullptr,
                  y, c.T, c.d, c.k, c.E, c.has_shared, tpc, nullptr};
    const int grid = (c.T + tpc - 1) / tpc;
    static DeviceOnce once;
    cudaError_t e = once.run([] {
      prefer_max_shared(combine_bulk_kernel<__nv_bfloat16>);
      prefer_max_shared(combine_bulk_kernel<float>);
      cudaError_t r = cudaFuncSetAttribute(combine_bulk_kernel<__nv_bfloat16>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(kBulkSmemMax));
      if (r != cudaSuccess) return r;
      return cudaFuncSetAttribute(combine_bulk_kernel<float>,
                                  cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  static_cast<int>(kBulkSmemMax));
    });
    if (e != cudaSuccess) return e;
    if (c.dtype == MOE_BF16)
      return launch_pdl(combine_bulk_kernel<__nv_bfloat16>, dim3(grid), dim3(threads), bulk_smem, s, a);
    return launch_pdl(combine_bulk_kernel<float>, dim3(grid), dim3(threads), bulk_smem, s, a);
  }
  if (c.k <= 8) {
    CombineArgs a{y_packed, route_row, gates, offsets, c.add_residual ? residual : nullptr,
                  y, c.T, c.d, c.k, c.E, c.has_shared, 1, nullptr};
    if (c.dtype == MOE_BF16) return launch_reg<__nv_bfloat16>(a, nvec, s);
    return launch_reg<float>(a, nvec, s);
  }
  int tpc = kThreads / nvec;
  tpc = tpc < 1 ? 1 : (tpc > kMaxTok ? kMaxTok : tpc);
  CombineArgs a{y_packed, route_row, gates, offsets, c.add_residual ? residual : nullptr,
                y, c.T, c.d, c.k, c.E, c.has_shared, tpc, nullptr};
  const int grid = (c.T + tpc - 1) / tpc;
  static DeviceOnce once;
  cudaError_t e = once.run([] {
    prefer_max_shared(combine_kernel<__nv_bfloat16>);
    return prefer_max_shared(combine_kernel<float>);
  });
  if (e != cudaSuccess) return e;
  if (c.dtype == MOE_BF16)
    return launch_pdl(combine_kernel<__nv_bfloat16>, dim3(grid), dim3(kThreads), 0, s, a);
  return launch_pdl(combine_kernel<float>, dim3(grid), dim3(kThreads), 0, s, a);
}

}  // namespace moe

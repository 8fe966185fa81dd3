// fp32 expert FFN: grouped GEMMs on CUDA cores over the ragged expert segments.
//
// The fp32 configuration asks for 1e-4 relative agreement, which tf32 tensor-core
// arithmetic cannot give, so fp32 layers run here in full fp32 FMA.  The bf16 layers use
// the tcgen05 kernel in gemm_sm100.cu.
//
// Source: "MoE Inference Visualized", Expert Execution: expert(x) = down(SiLU(gate(x)) *
// up(x)); "271,104 Routes: What I Missed About Mixture-of-Experts", section 3: one dense
// matmul per expert batch.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int BM = 32, BN = 32, BK = 32, kThreads = 256;

struct SimtArgs {
  const float* a_routed;   // [Rmax, K]   packed rows (mode gate/up) or H (mode down)
  const float* a_shared;   // [T, K]      x for the shared expert in mode gate/up, else = a_routed
  const int32_t* offsets;  // [E + 2] segment starts
  const int32_t* counts;   // [E] routed segment rows (padded layout) or null
  const float* w0;         // [E, N, K]   gate (mode 0) or down (mode 1)
  const float* w1;         // [E, N, K]   up (mode 0)
  const float* w0s;        // [N, K]      shared expert
  const float* w1s;
  float* out;              // [rows, N]
  int E, nseg, K, N;
};

__device__ __forceinline__ int seg_rows(const SimtArgs& a, int s) {
  return (a.counts != nullptr && s < a.E) ? a.counts[s] : a.offsets[s + 1] - a.offsets[s];
}

// Map a linear m-tile index to (segment, m-tile within segment); -1 when past the end.
__device__ int find_segment(const SimtArgs& a, int nseg, int mt, int* m_local) {
  int acc = 0;
  for (int s = 0; s < nseg; ++s) {
    const int rows = seg_rows(a, s);
    const int n = (rows + BM - 1) / BM;
    if (mt < acc + n) { *m_local = mt - acc; return s; }
    acc += n;
  }
  return -1;
}

__device__ __forceinline__ float silu(float g) { return g / (1.f + expf(-g)); }

// MODE 0: out = SiLU(A W0^T) * (A W1^T).  MODE 1: out = A W0^T.
template <int MODE>
__global__ void __launch_bounds__(kThreads) simt_kernel(SimtArgs a) {
  __shared__ float sA[BK][BM + 1];
  __shared__ float sB0[BK][BN + 1];
  __shared__ float sB1[MODE == 0 ? BK : 1][BN + 1];
  __shared__ int s_seg, s_m;
  pdl_trigger();
  pdl_wait();
  if (threadIdx.x == 0) s_seg = find_segment(a, a.nseg, blockIdx.x, &s_m);
  __syncthreads();
  const int seg = s_seg;
  if (seg < 0) return;
  const int row0 = __ldg(a.offsets + seg);
  const int rows = seg_rows(a, seg);
  const int m0 = s_m * BM, n0 = blockIdx.y * BN;
  const bool shared = seg == a.E;
  // A rows: packed segment for routed experts; for the shared expert in mode 0 the
  // rows are x[0..T) themselves, in mode 1 they are H rows of the shared segment.
  const float* A = (shared && MODE == 0) ? a.a_shared : a.a_routed + static_cast<size_t>(row0) * a.K;
  const float* W0 = shared ? a.w0s : a.w0 + static_cast<size_t>(seg) * a.N * a.K;
  const float* W1 = (MODE == 0) ? (shared ? a.w1s : a.w1 + static_cast<size_t>(seg) * a.N * a.K) : nullptr;

  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;  // 2x2 outputs per thread
  float c0[2][2] = {}, c1[2][2] = {};
  for (int k0 = 0; k0 < a.K; k0 += BK) {
    for (int i = threadIdx.x; i < BM * BK; i += kThreads) {
      const int r = i / BK, kk = i % BK;
      const int gr = m0 + r, gk = k0 + kk;
      sA[kk][r] = (gr < rows && gk < a.K) ? A[static_cast<size_t>(gr) * a.K + gk] : 0.f;
      const int gn = n0 + r;
      sB0[kk][r] = (gn < a.N && gk < a.K) ? W0[static_cast<size_t>(gn) * a.K + gk] : 0.f;
      if (MODE == 0) sB1[kk][r] = (gn < a.N && gk < a.K) ? W1[static_cast<size_t>(gn) * a.K + gk] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < BK; ++kk) {
      const float a0 = sA[kk][ty * 2], a1 = sA[kk][ty * 2 + 1];
      const float b0 = sB0[kk][tx * 2], b1 = sB0[kk][tx * 2 + 1];
      c0[0][0] = fmaf(a0, b0, c0[0][0]); c0[0][1] = fmaf(a0, b1, c0[0][1]);
      c0[1][0] = fmaf(a1, b0, c0[1][0]); c0[1][1] = fmaf(a1, b1, c0[1][1]);
      if (MODE == 0) {
        const float u0 = sB1[kk][tx * 2], u1 = sB1[kk][tx * 2 + 1];
        c1[0][0] = fmaf(a0, u0, c1[0][0]); c1[0][1] = fmaf(a0, u1, c1[0][1]);
        c1[1][0] = fmaf(a1, u0, c1[1][0]); c1[1][1] = fmaf(a1, u1, c1[1][1]);
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 2; ++i)
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int gr = m0 + ty * 2 + i, gn = n0 + tx * 2 + j;
      if (gr < rows && gn < a.N) {
        const float v = (MODE == 0) ? silu(c0[i][j]) * c1[i][j] : c0[i][j];
        a.out[static_cast<size_t>(row0 + gr) * a.N + gn] = v;
      }
    }
}

}  // namespace

cudaError_t launch_ffn_simt(const moe_config& c, const FfnArgs& f, cudaStream_t s,
                            cudaEvent_t mid) {
  const int nseg = c.E + (c.has_shared ? 1 : 0);
  // Upper bound on m-tiles: every segment may end in a partial tile.
  const long long rows_bound = f.rmax + (c.has_shared ? c.T : 0);
  const int mtiles = static_cast<int>((rows_bound + BM - 1) / BM + nseg);
  SimtArgs g{static_cast<const float*>(f.x_packed), static_cast<const float*>(f.x), f.offsets,
             f.counts, static_cast<const float*>(f.w_gate), static_cast<const float*>(f.w_up),
             static_cast<const float*>(f.s_gate), static_cast<const float*>(f.s_up),
             static_cast<float*>(f.h), c.E, nseg, c.d, c.d_ff};
  dim3 grid1(mtiles, (c.d_ff + BN - 1) / BN);
  cudaError_t e = launch_pdl(simt_kernel<0>, grid1, dim3(kThreads), 0, s, g);
  if (e != cudaSuccess) return e;
  if (mid != nullptr && (e = record_event(mid, s)) != cudaSuccess) return e;
  SimtArgs g2{static_cast<const float*>(f.h), static_cast<const float*>(f.h), f.offsets,
              f.counts, static_cast<const float*>(f.w_down), nullptr, static_cast<const float*>(f.s_down),
              nullptr, static_cast<float*>(f.y_packed), c.E, nseg, c.d_ff, c.d};
  dim3 grid2(mtiles, (c.d + BN - 1) / BN);
  return launch_pdl(simt_kernel<1>, grid2, dim3(kThreads), 0, s, g2);
}

}  // namespace moe

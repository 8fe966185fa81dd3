// Router on CUDA cores (fp32 layers; bf16 layers use route_sm100.cu): logits
// z = x W_r^T + bias, softmax and warp-level top-k with lowest-index ties, gate weights in
// one of three modes, and the per-token-tile expert histogram for dispatch.
//
// Sources: "271,104 Routes: What I Missed About Mixture-of-Experts", section 2 The Router;
// "Mixture of Experts: Routing, Dispatch, and Load Balancing", section 1 and section 3
// (softmax, topk, normalised weighted sum); "MoE Inference Visualized", The Router;
// "Mixture-of-experts routing", The gate.
//
// Design: one warp per token (8 tokens per CTA round).  A block of EP experts' router
// rows is staged in shared memory (cp.async) in d-chunks and shared by the CTA's tokens;
// each lane accumulates fp32 partial dot products for all EP experts over its slice of d
// (16-byte loads of x), then a reduce-scatter across the warp leaves the logit of expert
// (lane mod EP) on each lane.  Top-k is k rounds of a warp arg-max ordered by (logit
// descending, expert index ascending), so ties go to the lower index deterministically.
#include <cfloat>

#include "common.cuh"
#include "dispatch_prep.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kThreads = 256;       // 8 warps
constexpr int kTokPerWarp = 1;      // tokens per warp per sub-batch
constexpr int kSubTokens = 8 * kTokPerWarp;
// x vectors loaded together per lane: fewer for 32 experts per pass so that two CTAs
// (16 warps) fit on an SM without spilling the 32 partial sums.
template <int EP> constexpr int kXBatch = (EP >= 32) ? 2 : 4;
constexpr int kWChunkBytes = 64 * 1024;

struct RouterArgs {
  const void* x;
  const void* w;
  const float* bias;
  int T, d, E, k, gate_mode, tok_tile, dc;
  int32_t* ids;
  float* gates;
  int32_t* tile_hist;
  float* tile_psum;  // null: no routing statistics
  float* zkeys;      // null: ranking keys not stored
  DispatchPrep prep; // null ticket: no dispatch prep
};

// NaN logits rank as -inf so that k valid experts are always selected.
__device__ __forceinline__ float rank_key(float z) { return isnan(z) ? -INFINITY : z; }

// Reduce EP per-lane partial sums over the warp.  Afterwards every lane holds the full
// sum for expert (lane % EP).  Reduce-scatter over the low log2(EP) lane bits, then a
// butterfly over the remaining bits.
template <int EP>
__device__ __forceinline__ float warp_reduce_experts(float (&v)[EP], int lane) {
#pragma unroll
  for (int s = EP / 2; s >= 1; s >>= 1) {
    const bool upper = (lane & s) != 0;
#pragma unroll
    for (int i = 0; i < s; ++i) {
      const float send = upper ? v[i] : v[i + s];
      const float keep = upper ? v[i + s] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, s);
    }
  }
  float r = v[0];
#pragma unroll
  for (int s = 16; s >= EP; s >>= 1) r += __shfl_xor_sync(0xffffffffu, r, s);
  return r;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) v += __shfl_xor_sync(0xffffffffu, v, s);
  return v;
}

template <typename Tin, int EP>
__global__ void __launch_bounds__(kThreads, 1) router_kernel(RouterArgs a) {
  constexpr int VEC = Vec<Tin>::N;
  constexpr int NP = (EP == 32) ? 8 : 1;  // passes over experts (E <= 256)
  extern __shared__ uint4 s_w[];          // [EP][dc / VEC] vectors
  __shared__ int s_hist[256];
  __shared__ float s_psum[8][256];  // per-warp running sums of full-softmax probabilities

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile = blockIdx.x;
  const int tok0 = tile * a.tok_tile;
  const int tok_end = min(a.T, tok0 + a.tok_tile);
  const int npass = (a.E + EP - 1) / EP;
  const int dcv = a.dc / VEC;  // vectors per chunk row
  const Tin* __restrict__ X = static_cast<const Tin*>(a.x);
  const Tin* __restrict__ W = static_cast<const Tin*>(a.w);

  for (int e = tid; e < a.E; e += kThreads) s_hist[e] = 0;
  if (a.tile_psum != nullptr)
    for (int i = tid; i < 8 * 256; i += kThreads) s_psum[i >> 8][i & 255] = 0.f;
  pdl_trigger();
  pdl_wait();

  for (int sub = tok0; sub < tok_end; sub += kSubTokens) {
    int tok[kTokPerWarp];
#pragma unroll
    for (int i = 0; i < kTokPerWarp; ++i) tok[i] = sub + warp * kTokPerWarp + i;

    float zl[kTokPerWarp][NP];
#pragma unroll
    for (int i = 0; i < kTokPerWarp; ++i)
#pragma unroll
      for (int p = 0; p < NP; ++p) zl[i][p] = -INFINITY;

    for (int p = 0; p < npass; ++p) {
      float acc[kTokPerWarp][EP];
#pragma unroll
      for (int i = 0; i < kTokPerWarp; ++i)
#pragma unroll
        for (int e = 0; e < EP; ++e) acc[i][e] = 0.f;

      for (int d0 = 0; d0 < a.d; d0 += a.dc) {
        const int ncv = min(a.dc, a.d - d0) / VEC;
        __syncthreads();  // previous chunk fully consumed
        for (int v = tid; v < EP * ncv; v += kThreads) {
          const int e = v / ncv, c = v - e * ncv;
          const int ge = p * EP + e;
          if (ge < a.E)
            cp_async_16(&s_w[e * dcv + c], W + static_cast<size_t>(ge) * a.d + d0 + c * VEC);
          else
            s_w[e * dcv + c] = make_uint4(0, 0, 0, 0);
        }
        cp_async_wait_all();
        __syncthreads();
#pragma unroll
        for (int i = 0; i < kTokPerWarp; ++i) {
          if (tok[i] >= tok_end) continue;
          const Tin* xr = X + static_cast<size_t>(tok[i]) * a.d + d0;
          for (int c0 = lane; c0 < ncv; c0 += 32 * kXBatch<EP>) {
            uint4 xv[kXBatch<EP>];
#pragma unroll
            for (int u = 0; u < kXBatch<EP>; ++u) {
              const int c = c0 + 32 * u;
              xv[u] = (c < ncv) ? ld_vec(xr + c * VEC) : make_uint4(0, 0, 0, 0);
            }
#pragma unroll
            for (int u = 0; u < kXBatch<EP>; ++u) {
              const int c = c0 + 32 * u;
              if (c >= ncv) break;
              float xf[VEC];
              Vec<Tin>::to_f32(xv[u], xf);
#pragma unroll
              for (int e = 0; e < EP; ++e) {
                float wf[VEC];
                Vec<Tin>::to_f32(s_w[e * dcv + c], wf);
                float s = acc[i][e];
#pragma unroll
                for (int q = 0; q < VEC; ++q) s = fmaf(xf[q], wf[q], s);
                acc[i][e] = s;
              }
            }
          }
        }
      }
#pragma unroll
      for (int i = 0; i < kTokPerWarp; ++i) {
        const float z = warp_reduce_experts<EP>(acc[i], lane);
        const int ge = p * EP + (lane % EP);
        const float zb = (ge < a.E && a.bias != nullptr) ? z + __ldg(a.bias + ge) : z;
        if (a.zkeys != nullptr && tok[i] < tok_end && lane < EP && ge < a.E)
          a.zkeys[static_cast<size_t>(tok[i]) * a.E + ge] = rank_key(zb);
#pragma unroll
        for (int q = 0; q < NP; ++q)
          if (q == p) zl[i][q] = zb;
      }
    }

    // ---- top-k, gates, histogram: one token at a time per warp ----
#pragma unroll
    for (int i = 0; i < kTokPerWarp; ++i) {
      const int t = tok[i];
      if (t >= tok_end) continue;  // warp-uniform
      uint32_t taken = 0;
      float sel_z = -INFINITY;
      int sel_e = 0;
      for (int j = 0; j < a.k; ++j) {
        float bv = -INFINITY;
        int be = 0x7fffffff;
#pragma unroll
        for (int p = 0; p < NP; ++p) {
          const int ge = p * EP + lane;
          if (p < npass && lane < EP && ge < a.E && !(taken & (1u << p))) {
            const float v = rank_key(zl[i][p]);
            if (v > bv || (v == bv && ge < be)) { bv = v; be = ge; }
          }
        }
#pragma unroll
        for (int s = 16; s >= 1; s >>= 1) {
          const float ov = __shfl_xor_sync(0xffffffffu, bv, s);
          const int oe = __shfl_xor_sync(0xffffffffu, be, s);
          if (ov > bv || (ov == bv && oe < be)) { bv = ov; be = oe; }
        }
        if (lane == be % EP && be / EP < NP) taken |= 1u << (be / EP);
        if (lane == j) { sel_z = bv; sel_e = be; }
      }
      const float m = __shfl_sync(0xffffffffu, sel_z, 0);  // largest selected logit
      const float ej = (lane < a.k) ? expf(sel_z - m) : 0.f;
      float g;
      float denom_all = 0.f;
      if (a.gate_mode != MOE_GATE_TOPK_SOFTMAX || a.tile_psum != nullptr) {
        float local = 0.f;
#pragma unroll
        for (int p = 0; p < NP; ++p) {
          const int ge = p * EP + lane;
          if (p < npass && lane < EP && ge < a.E) local += expf(rank_key(zl[i][p]) - m);
        }
        denom_all = warp_sum(local);
      }
      if (a.gate_mode == MOE_GATE_TOPK_SOFTMAX) {
        g = ej / warp_sum(ej);
      } else {
        const float pj = ej / denom_all;
        g = (a.gate_mode == MOE_GATE_SOFTMAX_TOPK) ? pj : pj / warp_sum(pj);
      }
      if (a.tile_psum != nullptr) {
        // Routing statistics: this warp adds its tokens' full softmax in token order;
        // expert ge belongs to exactly one lane, so the per-warp sums are race-free.
        const float inv = 1.f / denom_all;
#pragma unroll
        for (int p = 0; p < NP; ++p) {
          const int ge = p * EP + lane;
          if (p < npass && lane < EP && ge < a.E)
            s_psum[warp][ge] += expf(rank_key(zl[i][p]) - m) * inv;
        }
      }
      if (lane < a.k) {
        a.ids[static_cast<size_t>(t) * a.k + lane] = sel_e;
        a.gates[static_cast<size_t>(t) * a.k + lane] = g;
        atomicAdd(&s_hist[sel_e], 1);
      }
    }
  }
  __syncthreads();
  if (a.tile_hist != nullptr)
    for (int e = tid; e < a.E; e += kThreads)
      a.tile_hist[static_cast<size_t>(tile) * a.E + e] = s_hist[e];
  if (a.tile_psum != nullptr)
    for (int e = tid; e < a.E; e += kThreads) {
      float v = 0.f;
#pragma unroll
      for (int w = 0; w < 8; ++w) v += s_psum[w][e];
      a.tile_psum[static_cast<size_t>(tile) * a.E + e] = v;
    }
  // the probability sums' shared memory is free now: scratch for the dispatch prep
  if (a.prep.ticket != nullptr) dispatch_prep_arrive(a.prep, reinterpret_cast<int*>(&s_psum[0][0]));
}

template <typename Tin, int EP>
cudaError_t launch_ep(const RouterArgs& a, int grid, cudaStream_t s) {
  const int smem = EP * a.dc * static_cast<int>(sizeof(Tin));
  static DeviceOnce once;  // attribute set once per instantiation and device
  cudaError_t e = once.run([] {
    return cudaFuncSetAttribute(router_kernel<Tin, EP>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, kWChunkBytes);
  });
  if (e != cudaSuccess) return e;
  return launch_pdl(router_kernel<Tin, EP>, dim3(grid), dim3(kThreads), smem, s, a);
}

template <typename Tin>
cudaError_t launch_typed(RouterArgs a, cudaStream_t s) {
  constexpr int VEC = Vec<Tin>::N;
  int EP = 1;
  while (EP < a.E && EP < 32) EP *= 2;
  int dc = kWChunkBytes / (EP * static_cast<int>(sizeof(Tin)));
  dc = (dc / (32 * VEC)) * (32 * VEC);  // whole warp sweeps
  if (dc > a.d) dc = a.d;
  a.dc = dc;
  const int grid = (a.T + a.tok_tile - 1) / a.tok_tile;
  switch (EP) {
    case 1: return launch_ep<Tin, 1>(a, grid, s);
    case 2: return launch_ep<Tin, 2>(a, grid, s);
    case 4: return launch_ep<Tin, 4>(a, grid, s);
    case 8: return launch_ep<Tin, 8>(a, grid, s);
    case 16: return launch_ep<Tin, 16>(a, grid, s);
    default: return launch_ep<Tin, 32>(a, grid, s);
  }
}

}  // namespace

cudaError_t launch_router(const moe_config& c, const void* x, const void* w_router,
                          const float* bias, int32_t* ids, float* gates, int32_t* tile_hist,
                          const RouterExtras& extra, const DispatchPrep& prep, int32_t* status,
                          cudaStream_t s) {
  if (c.dtype == MOE_BF16)
    return launch_router_sm100(c, x, w_router, bias, ids, gates, tile_hist, extra, prep, status,
                               s);
  RouterArgs a{x, w_router, bias, c.T, c.d, c.E, c.k, c.gate_mode, kHistTile, 0,
               ids, gates, tile_hist, extra.tile_psum, extra.zkeys, prep};
  return launch_typed<float>(a, s);
}

}  // namespace moe

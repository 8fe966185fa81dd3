// Router for bf16 layers on the 5th-generation tensor cores: logits z = x W_r^T + bias,
// top-k (largest first, ties to the lower expert index), gates in one of three modes, and
// the expert histogram of the 128-token tile, in one kernel.
//
// Sources: "271,104 Routes: What I Missed About Mixture-of-Experts", section 2 The Router
// (a projection, topk, softmax of the selected logits); "Mixture of Experts: Routing,
// Dispatch, and Load Balancing", section 1 (linear projection + softmax, weight stored
// [N, d]) and section 3 (topk of the probabilities, division by the selected total);
// "MoE Inference Visualized", The Router (the top-1 weight is the softmax probability);
// "Mixture-of-experts routing", The gate (softmax over only the top-k).
//
// The logit contraction [128 tokens x d] x [d x E] runs as tcgen05.mma with M = 128 tokens
// and N = E rounded up to 16 experts, fp32 accumulation in tensor memory, x streaming
// through a TMA ring.  Two kernels:
//  * router_cluster_kernel (E <= 64, d >= 512): a cluster of 8 CTAs shares a 128-token tile,
//    each contracting 1/8 of d; the partial logits are summed in distributed shared memory
//    in rank order, and top-k is a rank count with 8 lanes per token (see the kernel).
//  * router_tc_kernel (otherwise): one CTA per tile; each thread owns one token (one TMEM
//    lane).  For E <= 64 its logits stay in registers and top-k is a tournament (see
//    topk_tournament); above that it reads 16-column chunks into a sorted top-KMAX list
//    (insertion in expert order, so an equal logit never displaces an earlier expert).
// Both form the gates and the tile's expert histogram, and optionally the per-tile sums of
// the full softmax (routing statistics) and the ranking keys (reroute policy).
#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "dispatch_prep.cuh"
#include "internal.h"

namespace moe {

bool encode_2d_box(CUtensorMap* m, const void* ptr, uint64_t cols, uint64_t rows,
                   uint32_t box_rows);

namespace {

constexpr int kTokens = 128;           // tokens per CTA = MMA M = TMEM lanes
constexpr int BK = 64;                 // 128-byte swizzle rows of bf16
constexpr int kThreads = 192;          // warps 0-3 epilogue, 4 TMA producer, 5 MMA
constexpr int kMaxStages = 12;         // deepest TMA ring (the router-weight tile is small)
constexpr int A_BYTES = kTokens * BK * 2;
constexpr int kRingBudget = 192 * 1024;

struct RouteMaps {
  CUtensorMap x;  // [T, d] bf16, box 64 x 128
  CUtensorMap w;  // [E, d] bf16, box 64 x EN (rows >= E read as zero)
};

struct RouteParams {
  const float* bias;
  int T, d, E, k, EN, gate_mode, stages, tmem_cols;
  int32_t* ids;
  float* gates;
  int32_t* tile_hist;
  float* tile_psum;  // null: no routing statistics
  float* zkeys;      // null: ranking keys not stored
  int32_t* status;
  int64_t limit_ns;
  DispatchPrep prep; // null ticket: no dispatch prep
};

__device__ __forceinline__ float rank_key(float z) { return isnan(z) ? -INFINITY : z; }

// (v, e) ranks before (v2, e2): larger logit first, then lower expert index.
__device__ __forceinline__ bool ranks_before(float v, int e, float v2, int e2) {
  return v > v2 || (v == v2 && e < e2);
}

__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void epilogue_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// Sum over the warp's 32 lanes.  The butterfly pairs the same two partial sums on both
// lanes of each exchange, so every lane ends with identical bits.
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) v += __shfl_xor_sync(0xffffffffu, v, s);
  return v;
}

// Top-k of one token's logits z[0..NV) held in registers: k rounds of a tournament
// (binary-tree arg-max).  At every node the left child covers lower expert indices, so
// taking the left child on equality breaks ties towards the lower index exactly; taken
// experts are masked out.  Each round has depth log2(NV) and NV-1 independent-per-level
// comparisons, which keeps the per-thread dependency chains short.
template <int NV, int KMAX>
__device__ __forceinline__ void topk_tournament(const float (&z)[NV], int E, int k, float (&tv)[KMAX],
                                                int (&te)[KMAX]) {
  uint64_t taken = 0;
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    if (j >= k) break;
    float bv[NV];
    int bi[NV];
    bool ok[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      bv[i] = z[i];
      bi[i] = i;
      ok[i] = (i < E) && !((taken >> i) & 1u);
    }
#pragma unroll
    for (int w = NV / 2; w >= 1; w /= 2) {
#pragma unroll
      for (int i = 0; i < w; ++i) {
        const bool left = ok[2 * i] && (!ok[2 * i + 1] || bv[2 * i] >= bv[2 * i + 1]);
        bv[i] = left ? bv[2 * i] : bv[2 * i + 1];
        bi[i] = left ? bi[2 * i] : bi[2 * i + 1];
        ok[i] = ok[2 * i] || ok[2 * i + 1];
      }
    }
    tv[j] = bv[0];
    te[j] = bi[0];
    taken |= 1ull << bi[0];
  }
}

// EN_T: compile-time logit count for E <= 64 (16, 32 or 64, whole token in registers);
// 0 selects the general path (any E <= 256) that streams 16-logit chunks through an
// insertion into a sorted top-KMAX list.
template <int EN_T, int KMAX>
__global__ void __launch_bounds__(kThreads, 1)
    router_tc_kernel(const __grid_constant__ RouteMaps maps, const RouteParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int b_bytes = p.EN * BK * 2;
  const int stage_bytes = A_BYTES + b_bytes;  // multiple of 1024 (EN multiple of 8)
  uint8_t* ctl = base + p.stages * stage_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(ctl);
  uint64_t* empty = full + kMaxStages;
  uint64_t* tfull = empty + kMaxStages;
  uint64_t* drain = tfull + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctl + 8 * (2 * kMaxStages + 2));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* s_bias = reinterpret_cast<float*>(ctl + 256);
  int* s_hist = reinterpret_cast<int*>(ctl + 256 + 256 * 4);
  float* s_psum = reinterpret_cast<float*>(ctl + 256 + 2 * 256 * 4);  // [4 warps][256]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x;
  const int k_blocks = p.d / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    mbar_init(tfull, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&maps.x);
    tma_prefetch_desc(&maps.w);
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, p.tmem_cols);
    tmem_relinquish();
  }
  pdl_trigger();
  pdl_wait();  // x comes from the previous layer; ids/gates/hist are read by earlier kernels
  for (int e = threadIdx.x; e < 256; e += kThreads) s_hist[e] = 0;
  if (p.tile_psum != nullptr)
    for (int i = threadIdx.x; i < 4 * 256; i += kThreads) s_psum[i] = 0.f;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 4 && lane == 0) {
    // ---------------------------------------------------------------- TMA producer
    int stage = 0;
    uint32_t phase = 0;
    bool wrapped = false, ok = true;
    for (int kb = 0; kb < k_blocks; ++kb) {
      if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, p.limit_ns, p.status)) {
        ok = false;
        break;
      }
      mbar_arrive_expect_tx(&full[stage], stage_bytes);
      uint8_t* dst = base + stage * stage_bytes;
      tma_load_2d(dst, &maps.x, &full[stage], kb * BK, tile * kTokens);
      tma_load_2d(dst + A_BYTES, &maps.w, &full[stage], kb * BK, 0);
      if (++stage == p.stages) { stage = 0; phase ^= 1u; wrapped = true; }
    }
    if (!ok) {
      for (int s = 0; s < p.stages; ++s) {
        if (!wrapped && s >= stage) continue;
        mbar_wait_bounded(&full[s], (s < stage) ? phase : (phase ^ 1u), nullptr, p.limit_ns, p.status);
      }
    }
  } else if (warp == 5 && lane == 0) {
    // ---------------------------------------------------------------- MMA issuer
    const uint32_t idesc = idesc_bf16_f32(kTokens, p.EN);
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int kb = 0; kb < k_blocks; ++kb) {
      if (!mbar_wait_bounded(&full[stage], phase, abort_flag, p.limit_ns, p.status)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint8_t* src = base + stage * stage_bytes;
      const uint64_t ad = smem_desc_k_sw128(src);
      const uint64_t bd = smem_desc_k_sw128(src + A_BYTES);
#pragma unroll
      for (int kk = 0; kk < BK / 16; ++kk)
        tc_mma_bf16(tmem_base, ad + 2 * kk, bd + 2 * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
      tc_commit(&empty[stage]);
      if (++stage == p.stages) { stage = 0; phase ^= 1u; }
    }
    if (ok) {
      tc_commit(tfull);
    } else {
      tc_commit(drain);
      mbar_wait_bounded(drain, 0, nullptr, p.limit_ns, p.status);
    }
  } else if (warp < 4) {
    // ---------------------------------------------------------------- epilogue
    // The bias is read while the contraction runs (epilogue threads only).
    for (int e = threadIdx.x; e < 256; e += 128)
      s_bias[e] = (e < p.E && p.bias != nullptr) ? __ldg(p.bias + e) : 0.f;
    epilogue_bar();
    int ok = 1;
    if (lane == 0) ok = mbar_wait_bounded(tfull, 0, abort_flag, p.limit_ns, p.status);
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (ok) {
      tc_fence_after();
      const uint32_t trow = tmem_base + (static_cast<uint32_t>(warp * 32) << 16);
      const int t = tile * kTokens + warp * 32 + lane;
      float tv[KMAX];
      int te[KMAX];
#pragma unroll
      for (int j = 0; j < KMAX; ++j) { tv[j] = -INFINITY; te[j] = 0x7fffffff; }
      float zr[EN_T > 0 ? EN_T : 1];
      if constexpr (EN_T > 0) {
#pragma unroll
        for (int c0 = 0; c0 < EN_T; c0 += 16) {
          uint32_t r[16];
          tmem_ld_32x32b_x16(trow + c0, r);
#pragma unroll
          for (int j = 0; j < 16; ++j) zr[c0 + j] = __uint_as_float(r[j]);
        }
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < EN_T; ++e) zr[e] = (e < p.E) ? rank_key(zr[e] + s_bias[e]) : -INFINITY;
        if (p.zkeys != nullptr && t < p.T) {
          float* zrow = p.zkeys + static_cast<size_t>(t) * p.E;
#pragma unroll
          for (int e = 0; e < EN_T; ++e)
            if (e < p.E) zrow[e] = zr[e];
        }
        topk_tournament<EN_T, KMAX>(zr, p.E, p.k, tv, te);
      } else {
        for (int c0 = 0; c0 < p.EN; c0 += 16) {
          uint32_t r[16];
          tmem_ld_32x32b_x16(trow + c0, r);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int e = c0 + j;
            if (e < p.E) {
              const float v = rank_key(__uint_as_float(r[j]) + s_bias[e]);
              if (p.zkeys != nullptr && t < p.T) p.zkeys[static_cast<size_t>(t) * p.E + e] = v;
              if (ranks_before(v, e, tv[KMAX - 1], te[KMAX - 1])) {
                tv[KMAX - 1] = v;
                te[KMAX - 1] = e;
#pragma unroll
                for (int q = KMAX - 1; q > 0; --q) {
                  if (ranks_before(tv[q], te[q], tv[q - 1], te[q - 1])) {
                    const float fv = tv[q]; tv[q] = tv[q - 1]; tv[q - 1] = fv;
                    const int fe = te[q]; te[q] = te[q - 1]; te[q - 1] = fe;
                  }
                }
              }
            }
          }
        }
      }
      const float m = tv[0];  // largest logit
      const bool want_all = p.gate_mode != MOE_GATE_TOPK_SOFTMAX || p.tile_psum != nullptr;
      float denom_all = 0.f;
      if (EN_T > 0 && want_all) {
#pragma unroll
        for (int e = 0; e < (EN_T > 0 ? EN_T : 1); ++e)
          if (e < p.E) denom_all += expf(zr[e] - m);
      } else if (want_all) {  // softmax over all E: a second pass
        for (int c0 = 0; c0 < p.EN; c0 += 16) {
          uint32_t r[16];
          tmem_ld_32x32b_x16(trow + c0, r);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int e = c0 + j;
            if (e < p.E) denom_all += expf(rank_key(__uint_as_float(r[j]) + s_bias[e]) - m);
          }
        }
      }
      float g[KMAX];
      float sel = 0.f;
#pragma unroll
      for (int j = 0; j < KMAX; ++j) {
        g[j] = (j < p.k) ? expf(tv[j] - m) : 0.f;
        if (p.gate_mode != MOE_GATE_TOPK_SOFTMAX) g[j] = g[j] / denom_all;  // probability
        sel += g[j];
      }
      if (t < p.T) {
#pragma unroll
        for (int j = 0; j < KMAX; ++j) {
          if (j < p.k) {
            const float gj = (p.gate_mode == MOE_GATE_SOFTMAX_TOPK) ? g[j] : g[j] / sel;
            p.ids[static_cast<size_t>(t) * p.k + j] = te[j];
            p.gates[static_cast<size_t>(t) * p.k + j] = gj;
            atomicAdd(&s_hist[te[j]], 1);
          }
        }
      }
      if (p.tile_psum != nullptr) {
        // Routing statistics: every token's full softmax, summed over the warp's 32
        // tokens one expert at a time (tokens past T contribute zero).
        const float inv = (t < p.T) ? 1.f / denom_all : 0.f;
        if constexpr (EN_T > 0) {
#pragma unroll
          for (int e = 0; e < EN_T; ++e) {
            const float v = warp_sum(expf(zr[e] - m) * inv);  // zr = -inf past E
            if (lane == (e & 31) && e < p.E) s_psum[warp * 256 + e] = v;
          }
        } else {
          for (int c0 = 0; c0 < p.EN; c0 += 16) {
            uint32_t r[16];
            tmem_ld_32x32b_x16(trow + c0, r);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int e = c0 + j;
              const float z = (e < p.E) ? rank_key(__uint_as_float(r[j]) + s_bias[e]) : -INFINITY;
              const float v = warp_sum(expf(z - m) * inv);
              if (lane == (e & 31) && e < p.E) s_psum[warp * 256 + e] = v;
            }
          }
        }
      }
    }
    epilogue_bar();
    if (p.tile_hist != nullptr)
      for (int e = threadIdx.x; e < p.E; e += 128)
        p.tile_hist[static_cast<size_t>(tile) * p.E + e] = s_hist[e];
    if (p.tile_psum != nullptr)
      for (int e = threadIdx.x; e < p.E; e += 128)
        p.tile_psum[static_cast<size_t>(tile) * p.E + e] =
            ((s_psum[e] + s_psum[256 + e]) + s_psum[512 + e]) + s_psum[768 + e];
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5) tmem_dealloc(tmem_base, p.tmem_cols);
  // the TMA ring is idle now: scratch for the dispatch prep
  if (p.prep.ticket != nullptr) dispatch_prep_arrive(p.prep, reinterpret_cast<int*>(base));
}

// ---------------------------------------------------------------------------------
// Cluster variant (E <= 64, d >= 8 * 64): the 128-token tile is shared by a cluster of 8
// CTAs.  CTA r contracts d-blocks [r KB / 8, (r+1) KB / 8) for all 128 tokens, so the tile's
// x streams through 8 SMs instead of one.  The 8 partial logit tiles meet in distributed
// shared memory: CTA r adds up the rows of its 16 tokens from all 8 CTAs in rank order
// (the same order every run), adds the bias, and runs the epilogue with 8 lanes per token:
// each lane counts the rank of its experts against the token's row (larger logit first, then
// lower expert index) and writes the ones ranked below k to their slots.  CTA 0 adds up the
// 8 per-CTA histograms (and probability sums) in rank order.
// ---------------------------------------------------------------------------------
constexpr int kCluster = 8;
constexpr int kMaxSmemPerCta = 227 * 1024;
constexpr int kSmemPerSm = 228 * 1024;      // shared memory of one SM
constexpr int kSmemReservedPerCta = 1024;   // taken by the system from each resident CTA
constexpr int kTokPerCta = kTokens / kCluster;  // 16
constexpr int kLanesPerTok = 128 / kTokPerCta;  // 8

template <int EN_T>
__global__ void __launch_bounds__(kThreads, 1)
    router_cluster_kernel(const __grid_constant__ RouteMaps maps, const RouteParams p) {
  constexpr int V = EN_T / kLanesPerTok;  // logits per lane
  static_assert(V >= 1 && V <= 32, "logits per lane");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int stage_bytes = A_BYTES + EN_T * BK * 2;
  float* s_part = reinterpret_cast<float*>(base + p.stages * stage_bytes);  // [128][EN_T]
  float* s_red = s_part + kTokens * EN_T;                                   // [16][EN_T]
  float* s_p = s_red + kTokPerCta * EN_T;                                   // [16][EN_T]
  uint8_t* ctl = reinterpret_cast<uint8_t*>(s_p + kTokPerCta * EN_T);
  uint64_t* full = reinterpret_cast<uint64_t*>(ctl);
  uint64_t* empty = full + kMaxStages;
  uint64_t* tfull = empty + kMaxStages;
  uint64_t* drain = tfull + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctl + 8 * (2 * kMaxStages + 2));
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* s_bias = reinterpret_cast<float*>(ctl + 256);
  int* s_hist = reinterpret_cast<int*>(ctl + 256 + 256 * 4);
  float* s_psum = reinterpret_cast<float*>(ctl + 256 + 2 * 256 * 4);
  float* s_gsel = reinterpret_cast<float*>(ctl + 256 + 3 * 256 * 4);  // [16][32] top-k exps
  float* s_gden = s_gsel + kTokPerCta * 32;                           // [16][8] partial sums

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int tile = blockIdx.x / kCluster;
  const int KB = p.d / BK;
  const int kb0 = static_cast<int>(rank) * KB / kCluster;
  const int kb1 = (static_cast<int>(rank) + 1) * KB / kCluster;

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    mbar_init(tfull, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&maps.x);
    tma_prefetch_desc(&maps.w);
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, p.tmem_cols);
    tmem_relinquish();
  }
  pdl_trigger();
  pdl_wait();  // x comes from the previous layer; ids/gates/hist are read by earlier kernels
  for (int e = threadIdx.x; e < 256; e += kThreads) {
    s_hist[e] = 0;
    s_psum[e] = 0.f;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 4 && lane == 0) {
    // ---------------------------------------------------------------- TMA producer
    int stage = 0;
    uint32_t phase = 0;
    bool wrapped = false, ok = true;
    for (int kb = kb0; kb < kb1; ++kb) {
      if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, p.limit_ns, p.status)) {
        ok = false;
        break;
      }
      mbar_arrive_expect_tx(&full[stage], stage_bytes);
      uint8_t* dst = base + stage * stage_bytes;
      tma_load_2d(dst, &maps.x, &full[stage], kb * BK, tile * kTokens);
      tma_load_2d(dst + A_BYTES, &maps.w, &full[stage], kb * BK, 0);
      if (++stage == p.stages) { stage = 0; phase ^= 1u; wrapped = true; }
    }
    if (!ok) {
      for (int s = 0; s < p.stages; ++s) {
        if (!wrapped && s >= stage) continue;
        mbar_wait_bounded(&full[s], (s < stage) ? phase : (phase ^ 1u), nullptr, p.limit_ns, p.status);
      }
    }
  } else if (warp == 5 && lane == 0) {
    // ---------------------------------------------------------------- MMA issuer
    const uint32_t idesc = idesc_bf16_f32(kTokens, EN_T);
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int kb = kb0; kb < kb1; ++kb) {
      if (!mbar_wait_bounded(&full[stage], phase, abort_flag, p.limit_ns, p.status)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint8_t* src = base + stage * stage_bytes;
      const uint64_t ad = smem_desc_k_sw128(src);
      const uint64_t bd = smem_desc_k_sw128(src + A_BYTES);
#pragma unroll
      for (int kk = 0; kk < BK / 16; ++kk)
        tc_mma_bf16(tmem_base, ad + 2 * kk, bd + 2 * kk, idesc, (kb != kb0 || kk != 0) ? 1u : 0u);
      tc_commit(&empty[stage]);
      if (++stage == p.stages) { stage = 0; phase ^= 1u; }
    }
    if (ok) {
      tc_commit(tfull);
    } else {
      tc_commit(drain);
      mbar_wait_bounded(drain, 0, nullptr, p.limit_ns, p.status);
    }
  } else if (warp < 4) {
    // ---------------------------------------------------------------- partial logits
    // (the bias is read here, off the producer's critical path; it is used after the
    // block barrier below)
    for (int e = threadIdx.x; e < 256; e += 128)
      s_bias[e] = (e < p.E && p.bias != nullptr) ? __ldg(p.bias + e) : 0.f;
    int ok = 1;
    if (lane == 0) ok = mbar_wait_bounded(tfull, 0, abort_flag, p.limit_ns, p.status);
    ok = __shfl_sync(0xffffffffu, ok, 0);
    float4* dst = reinterpret_cast<float4*>(s_part + (warp * 32 + lane) * EN_T);
    if (ok) {
      tc_fence_after();
      const uint32_t trow = tmem_base + (static_cast<uint32_t>(warp * 32) << 16);
#pragma unroll
      for (int c0 = 0; c0 < EN_T; c0 += 16) {
        uint32_t r[16];
        tmem_ld_32x32b_x16(trow + c0, r);
        tmem_ld_wait();
#pragma unroll
        for (int q = 0; q < 4; ++q)
          dst[c0 / 4 + q] = make_float4(__uint_as_float(r[4 * q]), __uint_as_float(r[4 * q + 1]),
                                        __uint_as_float(r[4 * q + 2]), __uint_as_float(r[4 * q + 3]));
      }
    } else {
#pragma unroll
      for (int c = 0; c < EN_T / 4; ++c) dst[c] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  __syncthreads();
  cluster_sync_all();  // every CTA's partial logits are visible to the cluster

  // ------------------------------------------------------------------ reduce my 16 tokens
  const int row0 = static_cast<int>(rank) * kTokPerCta;
  for (int c = threadIdx.x; c < kTokPerCta * EN_T / 4; c += kThreads) {
    const int rl = c / (EN_T / 4), c4 = c - rl * (EN_T / 4);
    const float* src = s_part + (row0 + rl) * EN_T + c4 * 4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int r = 0; r < kCluster; ++r) {
      const float4 v = ld_cluster_f4(cluster_map(src, static_cast<uint32_t>(r)));
      acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
    const float a4[4] = {acc.x, acc.y, acc.z, acc.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int e = c4 * 4 + q;
      s_red[rl * EN_T + e] = (e < p.E) ? rank_key(a4[q] + s_bias[e]) : -INFINITY;
    }
  }
  __syncthreads();

  if (warp < 4) {
    // ---------------------------------------------------------------- epilogue
    const int tl = threadIdx.x / kLanesPerTok, g = threadIdx.x % kLanesPerTok;
    const int t = tile * kTokens + row0 + tl;
    float v[V];
    uint32_t taken = 0;  // bit q: expert q * 8 + g is selected (or is padding past E)
#pragma unroll
    for (int q = 0; q < V; ++q) {
      const int e = q * kLanesPerTok + g;
      v[q] = s_red[tl * EN_T + e];
      if (e >= p.E) taken |= 1u << q;
    }
    if (p.zkeys != nullptr && t < p.T) {
#pragma unroll
      for (int q = 0; q < V; ++q) {
        const int e = q * kLanesPerTok + g;
        if (e < p.E) p.zkeys[static_cast<size_t>(t) * p.E + e] = v[q];
      }
    }
    // Rank of each of my experts in the token's order (logit descending, then expert index
    // ascending), counted against the token's whole row, which the 8 lanes read from
    // shared memory as a broadcast: rank r < k means slot r.  The row maximum is the
    // top logit.
    const float* zrow = s_red + tl * EN_T;
    int rk[V];
#pragma unroll
    for (int q = 0; q < V; ++q) rk[q] = 0;
    float m = -INFINITY;
#pragma unroll 8
    for (int e2 = 0; e2 < EN_T; ++e2) {
      const float z2 = zrow[e2];
      m = fmaxf(m, z2);
#pragma unroll
      for (int q = 0; q < V; ++q) {
        const int e = q * kLanesPerTok + g;
        rk[q] += (z2 > v[q] || (z2 == v[q] && e2 < e)) ? 1 : 0;
      }
    }
    // The token's exps of the selected logits go to their slots, and the lanes' partial sums
    // of all exps to their places; both are then added up in a fixed order (slot order for
    // the selected total) by every lane of the token.
    float ex[V];
    float dpart = 0.f;
#pragma unroll
    for (int q = 0; q < V; ++q) {
      const int e = q * kLanesPerTok + g;
      ex[q] = (e < p.E) ? expf(v[q] - m) : 0.f;
      dpart += ex[q];
      if (e < p.E && rk[q] < p.k) s_gsel[tl * 32 + rk[q]] = ex[q];
    }
    s_gden[tl * kLanesPerTok + g] = dpart;
    __syncwarp();
    float denom_all = 0.f;
#pragma unroll
    for (int g2 = 0; g2 < kLanesPerTok; ++g2) denom_all += s_gden[tl * kLanesPerTok + g2];
    const bool prob = p.gate_mode != MOE_GATE_TOPK_SOFTMAX;  // gates are probabilities first
    float sel = 0.f;
    for (int j = 0; j < p.k; ++j) sel += prob ? s_gsel[tl * 32 + j] / denom_all : s_gsel[tl * 32 + j];
    if (t < p.T) {
#pragma unroll
      for (int q = 0; q < V; ++q) {
        const int e = q * kLanesPerTok + g;
        if (e < p.E && rk[q] < p.k) {
          const float gp = prob ? ex[q] / denom_all : ex[q];
          const float gj = (p.gate_mode == MOE_GATE_SOFTMAX_TOPK) ? gp : gp / sel;
          p.ids[static_cast<size_t>(t) * p.k + rk[q]] = e;
          p.gates[static_cast<size_t>(t) * p.k + rk[q]] = gj;
          atomicAdd(&s_hist[e], 1);
        }
      }
    }
    if (p.tile_psum != nullptr) {
      const float inv = (t < p.T) ? 1.f / denom_all : 0.f;
#pragma unroll
      for (int q = 0; q < V; ++q) {
        const int e = q * kLanesPerTok + g;
        s_p[tl * EN_T + e] = (e < p.E) ? expf(v[q] - m) * inv : 0.f;
      }
    }
  }
  __syncthreads();
  if (p.tile_psum != nullptr && threadIdx.x < EN_T) {
    float a = 0.f;
    for (int tl = 0; tl < kTokPerCta; ++tl) a += s_p[tl * EN_T + threadIdx.x];
    s_psum[threadIdx.x] = a;
  }
  cluster_sync_all();  // every CTA's histogram and probability sums are visible
  if (rank == 0) {
    for (int e = threadIdx.x; e < p.E; e += kThreads) {
      int h = 0;
      float ps = 0.f;
      for (int r = 0; r < kCluster; ++r) {
        h += ld_cluster_s32(cluster_map(&s_hist[e], static_cast<uint32_t>(r)));
        if (p.tile_psum != nullptr) ps += ld_cluster_f32(cluster_map(&s_psum[e], static_cast<uint32_t>(r)));
      }
      if (p.tile_hist != nullptr) p.tile_hist[static_cast<size_t>(tile) * p.E + e] = h;
      if (p.tile_psum != nullptr) p.tile_psum[static_cast<size_t>(tile) * p.E + e] = ps;
    }
  }
  cluster_sync_all();  // CTA 0 has read the others' shared memory before any of them exits
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5) tmem_dealloc(tmem_base, p.tmem_cols);
  // One arrival per tile (CTA 0 wrote its histogram row).  No CTA of the cluster reads the
  // partial-logit array any more: it is scratch for the dispatch prep.
  if (rank == 0 && p.prep.ticket != nullptr)
    dispatch_prep_arrive(p.prep, reinterpret_cast<int*>(s_part));
}

template <int EN_T>
cudaError_t launch_cluster_en(const RouteMaps& maps, const RouteParams& p, int grid, int smem,
                              cudaStream_t s) {
  static DeviceOnce once;
  cudaError_t e = once.run([] {
    return cudaFuncSetAttribute(router_cluster_kernel<EN_T>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmemPerCta);
  });
  if (e != cudaSuccess) return e;
  return launch_pdl_cluster(router_cluster_kernel<EN_T>, dim3(grid), dim3(kThreads), smem,
                            kCluster, s, maps, p);
}

template <int EN_T, int KMAX>
cudaError_t launch_kmax(const RouteMaps& maps, const RouteParams& p, int grid, int smem,
                        cudaStream_t s) {
  static DeviceOnce once;
  cudaError_t e = once.run([] {
    cudaError_t r = cudaFuncSetAttribute(router_tc_kernel<EN_T, KMAX>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         1024 + kRingBudget + 8192);
    if (r != cudaSuccess) return r;
    return prefer_max_shared(router_tc_kernel<EN_T, KMAX>);
  });
  if (e != cudaSuccess) return e;
  return launch_pdl(router_tc_kernel<EN_T, KMAX>, dim3(grid), dim3(kThreads), smem, s, maps, p);
}

template <int EN_T>
cudaError_t launch_en(const RouteMaps& maps, const RouteParams& p, int grid, int smem,
                      cudaStream_t s) {
  if (p.k <= 1) return launch_kmax<EN_T, 1>(maps, p, grid, smem, s);
  if (p.k <= 2) return launch_kmax<EN_T, 2>(maps, p, grid, smem, s);
  if (p.k <= 4) return launch_kmax<EN_T, 4>(maps, p, grid, smem, s);
  if (p.k <= 8) return launch_kmax<EN_T, 8>(maps, p, grid, smem, s);
  if (p.k <= 16) return launch_kmax<EN_T, 16>(maps, p, grid, smem, s);
  return launch_kmax<EN_T, 32>(maps, p, grid, smem, s);
}

}  // namespace

cudaError_t launch_router_sm100(const moe_config& c, const void* x, const void* w_router,
                                const float* bias, int32_t* ids, float* gates,
                                int32_t* tile_hist, const RouterExtras& extra,
                                const DispatchPrep& prep, int32_t* status, cudaStream_t s) {
  float* tile_psum = extra.tile_psum;
  // Logit columns (MMA N): 16, 32 or 64 when E fits, so the epilogue can keep a token's
  // logits in registers; otherwise E rounded up to a multiple of 16.
  const int EN = c.E <= 16 ? 16 : c.E <= 32 ? 32 : c.E <= 64 ? 64 : ((c.E + 15) / 16) * 16;
  int cols = 32;
  while (cols < EN) cols *= 2;
  const int stage_bytes = A_BYTES + EN * BK * 2;
  int stages = kRingBudget / stage_bytes;
  if (stages > kMaxStages) stages = kMaxStages;
  const int k_blocks = c.d / BK;
  if (stages > k_blocks) stages = k_blocks;
  RouteMaps maps;
  if (!encode_2d_box(&maps.x, x, c.d, c.T, kTokens) ||
      !encode_2d_box(&maps.w, w_router, c.d, c.E, EN))
    return cudaErrorInvalidValue;
  RouteParams p{bias, c.T, c.d, c.E, c.k, EN, c.gate_mode, stages, cols,
                ids, gates, tile_hist, tile_psum, extra.zkeys, status, kWaitLimitNs, prep};
  const int ntiles = (c.T + kTokens - 1) / kTokens;
  if (EN <= 64 && k_blocks >= kCluster) {
    // one 128-token tile per cluster of 8 CTAs, each with 1/8 of d
    const int fixed = 1024 + (kTokens + 2 * kTokPerCta) * EN * 4 + 256 + 3 * 256 * 4 +
                      kTokPerCta * (32 + kLanesPerTok) * 4;
    int cstages = (k_blocks + kCluster - 1) / kCluster;
    if (cstages > stages) cstages = stages;
    if (cstages > (kMaxSmemPerCta - fixed) / stage_bytes) cstages = (kMaxSmemPerCta - fixed) / stage_bytes;
    // As many CTAs per SM (up to 4) as still leave a two-stage ring: a CTA spends most of
    // its life in the cluster reduction and the top-k epilogue, which then overlap the
    // other CTAs' TMA streams (the grid rarely fits in one wave of one CTA per SM).
    for (int per_sm = 4; per_sm >= 2; --per_sm) {
      const int fit = (kSmemPerSm / per_sm - kSmemReservedPerCta - fixed) / stage_bytes;
      if (fit >= 2) {
        if (cstages > fit) cstages = fit;
        break;
      }
    }
    RouteParams pc = p;
    pc.stages = cstages;
    const int csmem = fixed + cstages * stage_bytes;
    const int cgrid = ntiles * kCluster;
    if (EN == 16) return launch_cluster_en<16>(maps, pc, cgrid, csmem, s);
    if (EN == 32) return launch_cluster_en<32>(maps, pc, cgrid, csmem, s);
    return launch_cluster_en<64>(maps, pc, cgrid, csmem, s);
  }
  const int grid = ntiles;
  const int smem = 1024 + stages * stage_bytes + 256 + 2 * 256 * 4 + (tile_psum ? 4 * 256 * 4 : 0);
  if (EN == 16) return launch_en<16>(maps, p, grid, smem, s);
  if (EN == 32) return launch_en<32>(maps, p, grid, smem, s);
  if (EN == 64) return launch_en<64>(maps, p, grid, smem, s);
  return launch_en<0>(maps, p, grid, smem, s);
}

}  // namespace moe

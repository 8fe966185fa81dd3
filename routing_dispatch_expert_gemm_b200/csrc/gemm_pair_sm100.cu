// bf16 expert FFN, column tiles over a pair of SMs (tcgen05 cta_group::2).  Same products
// as gemm_sm100.cu and gemm_cols_sm100.cu:
//   gate/up:  H[r, f] = SiLU(sum_i X[r,i] Wg_e[f,i]) * (sum_i X[r,i] Wu_e[f,i])
//   down:     Y[r, c] = sum_f H[r,f] Wd_e[c,f]
// Source: "MoE Inference Visualized", Expert Execution; "271,104 Routes: What I Missed About
// Mixture-of-Experts", sections 3 and 5.
//
// Why: column tiles (weights on the MMA's M side, an expert segment's tokens on N, padded
// to a multiple of 32) waste little work on ragged segments, but a one-SM column tile reads
// as many shared-memory bytes per MMA as its two operands hold.  A pair of SMs runs one
// M = 256 MMA in which each SM holds its own 128 weight rows and HALF of the token tile, so
// each SM reads 128 + N/2 operand rows per MMA instead of 128 + N.
//
// A cluster of 2 CTAs per pair; rank 0 (the leader) issues the MMAs.  Per CTA, 10 warps:
//   warp 8    TMA producer: its own weight tile(s) [128 rows x 64 K] and its half of the
//             token tile [N/2 rows x 64 K] per stage; the loads signal the LEADER's stage
//             barrier (which expects both CTAs' bytes).
//   warp 9    leader: tcgen05.mma.cta_group::2 M=256, N (x2 for gate and up) per K=16 step;
//             commits free both CTAs' stage and announce a finished accumulator to both.
//             Both CTAs' warp 9 allocate and free the pair's tensor memory.
//   warps 0-7 epilogue, in both CTAs: the CTA's 128 weight rows x all N tokens, SwiGLU or
//             plain conversion, transposed through shared memory into token-major rows;
//             each warp then tells the leader that the accumulator has been read.
// Gate/up pair tile: 256 f (leader f0..f0+127, peer f0+128..f0+255) x up to 128 tokens
// (gate and up accumulators side by side, double-buffered: 512 TMEM columns).  Down pair
// tile: 256 output columns x up to 256 tokens.  Every wait is bounded; on a timeout the
// CTA records MOE_ERR_TIMEOUT and stops.  No TMA multicast is used: each CTA loads its own
// operand rows.
#include "gemm_common.cuh"
#include "internal.h"

namespace moe {
namespace {

using gemm::BK;
using gemm::kMaxSeg;
using gemm::find_seg;
using gemm::silu_f;

constexpr int BW = 128;           // weight rows per CTA (the pair: 256)
constexpr int kTokBox = 16;       // token rows per TMA box
constexpr int kEpiWarps = 8;
constexpr int kProducerWarp = kEpiWarps;
constexpr int kMmaWarp = kEpiWarps + 1;
constexpr int kThreads = 32 * (kEpiWarps + 2);
constexpr int kStageRowBytes = 80;
constexpr int kEpiStageBytes = 32 * kStageRowBytes;
constexpr int W_BYTES = BW * BK * 2;
constexpr int kBoxBytes = kTokBox * BK * 2;

struct PairMaps {
  CUtensorMap x_routed;   // tokens [rows, K], 16-row boxes
  CUtensorMap x_shared;   // x [T, d] (gate/up shared segment), 16-row boxes
  CUtensorMap w0_routed;  // W_gate or W_down [E*N, K], 128-row boxes
  CUtensorMap w1_routed;  // W_up
  CUtensorMap w0_shared;
  CUtensorMap w1_shared;
};

struct PairParams {
  const int32_t* offsets;
  const int32_t* counts;
  int nseg, E, K, N;      // N: weight rows of one expert = output columns
  __nv_bfloat16* out;
  int ldo;
  int32_t* status;
  int64_t limit_ns;
};

template <int MODE>  // 0: SwiGLU gate|up; 1: down
struct PairCfg {
  static constexpr int NW = (MODE == 0) ? 2 : 1;         // weight tiles per stage
  static constexpr int NT = (MODE == 0) ? 128 : 256;     // tokens per pair tile, at most
  static constexpr int X_BYTES = (NT / 2) * BK * 2;      // this CTA's half of the token tile
  static constexpr int STAGE_BYTES = NW * W_BYTES + X_BYTES;
  static constexpr int STAGES = (MODE == 0) ? 5 : 6;
  static constexpr int ACC_COLS = NW * NT;               // 256 either way
  static constexpr int TMEM_COLS = 2 * ACC_COLS;         // 512
  static constexpr int SMEM =
      1024 + STAGES * STAGE_BYTES + kEpiWarps * kEpiStageBytes + 256 + 3 * kMaxSeg * 4;
};

struct PairTile {
  int s, wb, tb, ntok, npad;  // npad: MMA N (tokens rounded up to 32)
};

template <int NT>
__device__ __forceinline__ PairTile decode_pair_tile(const int* s_pre, const int* s_rows, int nseg,
                                                     int tile) {
  PairTile c;
  c.s = find_seg(s_pre, nseg, tile);
  const int rows = s_rows[c.s];
  const int tbc = (rows + NT - 1) / NT;
  const int local = tile - s_pre[c.s];
  c.wb = local / tbc;
  c.tb = local - c.wb * tbc;
  c.ntok = min(NT, rows - c.tb * NT);
  c.npad = (c.ntok + 31) & ~31;
  return c;
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_pair_kernel(const __grid_constant__ PairMaps maps, const PairParams p) {
  using C = PairCfg<MODE>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sW = base;                                  // [STAGES][NW][128 x 64]
  uint8_t* sX = sW + C::STAGES * C::NW * W_BYTES;      // [STAGES][NT/2 x 64]
  uint8_t* sEpi = sX + C::STAGES * C::X_BYTES;
  uint8_t* ctl = sEpi + kEpiWarps * kEpiStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(ctl);   // leader's are the ones used
  uint64_t* empty = full + 8;
  uint64_t* tfull = empty + 8;
  uint64_t* tempty = tfull + 2;                        // leader's are the ones used
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctl + 192);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(ctl + 196);
  int* s_pre = reinterpret_cast<int*>(ctl + 256);
  int* s_row0 = s_pre + kMaxSeg;
  int* s_rows = s_row0 + kMaxSeg;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = (rank == 0);
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int n_wblocks = p.N / (2 * BW);  // weight blocks of 256 rows
  const int k_blocks = p.K / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(&tfull[b], 1); mbar_init(&tempty[b], 2 * kEpiWarps); }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kProducerWarp && lane == 0) {
    tma_prefetch_desc(&maps.x_routed);
    tma_prefetch_desc(&maps.w0_routed);
    if (MODE == 0) tma_prefetch_desc(&maps.w1_routed);
  }
  if (warp == kMmaWarp) {
    tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  pdl_trigger();
  pdl_wait();
  if (warp == 0)
    gemm::build_segment_table(p.offsets, p.counts, p.nseg, p.E, C::NT, n_wblocks, s_pre, s_row0,
                              s_rows);
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers are initialised before any remote use
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = s_pre[p.nseg];

  if (warp == kProducerWarp && lane == 0) {
    // ------------------------------------------------------------ TMA producer (both)
    int stage = 0;
    uint32_t phase = 0;
    bool wrapped = false, ok = true;
    for (int tile = pair; tile < total && ok; tile += npairs) {
      const PairTile tc = decode_pair_tile<C::NT>(s_pre, s_rows, p.nseg, tile);
      const int nbox = (tc.npad / 2) / kTokBox;  // this CTA's half
      const bool shared = (tc.s == p.E);
      const CUtensorMap* mx = (MODE == 0 && shared) ? &maps.x_shared : &maps.x_routed;
      const int x_row = ((MODE == 0 && shared) ? 0 : s_row0[tc.s]) + tc.tb * C::NT +
                        static_cast<int>(rank) * (tc.npad / 2);
      const CUtensorMap* mw0 = shared ? &maps.w0_shared : &maps.w0_routed;
      const CUtensorMap* mw1 = shared ? &maps.w1_shared : &maps.w1_routed;
      const int w_row = (shared ? 0 : tc.s * p.N) + tc.wb * 2 * BW + static_cast<int>(rank) * BW;
      // the leader's barrier counts both CTAs' bytes
      const uint32_t bytes_pair = 2 * (C::NW * W_BYTES + nbox * kBoxBytes);
      for (int kb = 0; kb < k_blocks; ++kb) {
        if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, p.limit_ns, p.status)) {
          ok = false;
          break;
        }
        if (leader) mbar_arrive_expect_tx(&full[stage], bytes_pair);
        const uint32_t bar = cluster_map(&full[stage], 0);
        uint8_t* w_dst = sW + stage * C::NW * W_BYTES;
        uint8_t* x_dst = sX + stage * C::X_BYTES;
        const int kx = kb * BK;
        tma_load_2d_pair(w_dst, mw0, bar, kx, w_row);
        if (MODE == 0) tma_load_2d_pair(w_dst + W_BYTES, mw1, bar, kx, w_row);
        for (int i = 0; i < nbox; ++i)
          tma_load_2d_pair(x_dst + i * kBoxBytes, mx, bar, kx, x_row + i * kTokBox);
        if (++stage == C::STAGES) { stage = 0; phase ^= 1u; wrapped = true; }
      }
    }
    if (!ok && leader) {  // drain the copies the leader's barriers still count
      for (int s = 0; s < C::STAGES; ++s) {
        if (!wrapped && s >= stage) continue;
        const uint32_t par = (s < stage) ? phase : (phase ^ 1u);
        mbar_wait_bounded(&full[s], par, nullptr, p.limit_ns, p.status);
      }
    }
  } else if (warp == kMmaWarp && lane == 0 && leader) {
    // ------------------------------------------------------------ MMA issuer (leader)
    int stage = 0, acc = 0;
    uint32_t phase = 0, acc_phase = 0;
    bool ok = true;
    for (int tile = pair; tile < total && ok; tile += npairs) {
      const PairTile tc = decode_pair_tile<C::NT>(s_pre, s_rows, p.nseg, tile);
      const uint32_t idesc = idesc_bf16_f32(2 * BW, tc.npad);
      if (!mbar_wait_bounded(&tempty[acc], acc_phase ^ 1u, abort_flag, p.limit_ns, p.status)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * C::ACC_COLS);
      for (int kb = 0; kb < k_blocks; ++kb) {
        if (!mbar_wait_bounded(&full[stage], phase, abort_flag, p.limit_ns, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t xd = smem_desc_k_sw128(sX + stage * C::X_BYTES);
        const uint64_t w0d = smem_desc_k_sw128(sW + stage * C::NW * W_BYTES);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk)
          tc_mma_bf16_pair(d_tmem, w0d + 2 * kk, xd + 2 * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
        if (MODE == 0) {
          const uint64_t w1d = smem_desc_k_sw128(sW + stage * C::NW * W_BYTES + W_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            tc_mma_bf16_pair(d_tmem + C::NT, w1d + 2 * kk, xd + 2 * kk, idesc,
                             (kb | kk) != 0 ? 1u : 0u);
        }
        tc_commit_pair_mc(&empty[stage], 0x3);  // frees the stage in both CTAs
        if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
      tc_commit_pair_mc(&tfull[acc], 0x3);  // the accumulator is ready in both CTAs
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    if (!ok) {  // every issued MMA has finished before the memory goes away
      tc_commit_pair_mc(drain, 0x1);
      mbar_wait_bounded(drain, 0, nullptr, p.limit_ns, p.status);
    }
  } else if (warp < kEpiWarps) {
    // ------------------------------------------------------------ epilogue (both)
    const int quarter = warp & 3, half = warp >> 2;
    uint8_t* stage_mem = sEpi + warp * kEpiStageBytes;
    const uint32_t tempty0 = cluster_map(&tempty[0], 0);
    const uint32_t tempty1 = cluster_map(&tempty[1], 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = pair; tile < total; tile += npairs) {
      const PairTile tc = decode_pair_tile<C::NT>(s_pre, s_rows, p.nseg, tile);
      int ok = 1;
      if (lane == 0) ok = mbar_wait_bounded(&tfull[acc], acc_phase, abort_flag, p.limit_ns, p.status);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                              static_cast<uint32_t>(acc * C::ACC_COLS);
      __nv_bfloat16* out_tile = p.out + static_cast<size_t>(s_row0[tc.s] + tc.tb * C::NT) * p.ldo +
                                static_cast<size_t>(tc.wb) * 2 * BW + static_cast<int>(rank) * BW +
                                quarter * 32;
#pragma unroll 1
      for (int c0 = half * (C::NT / 2); c0 < (half + 1) * (C::NT / 2) && c0 < tc.ntok; c0 += 32) {
        float h[32];
        if (MODE == 0) {
          uint32_t g[32], u[32];
          tmem_ld_32x32b_x32(t_lane + c0, g);
          tmem_ld_32x32b_x32(t_lane + C::NT + c0, u);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) h[i] = silu_f(__uint_as_float(g[i])) * __uint_as_float(u[i]);
        } else {
          uint32_t v[32];
          tmem_ld_32x32b_x32(t_lane + c0, v);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) h[i] = __uint_as_float(v[i]);
        }
#pragma unroll
        for (int i = 0; i < 32; ++i)
          reinterpret_cast<__nv_bfloat16*>(stage_mem + i * kStageRowBytes)[lane] =
              __float2bfloat16_rn(h[i]);
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = i * 8 + (lane >> 2), q = lane & 3;
          const uint4 v = *reinterpret_cast<const uint4*>(stage_mem + r * kStageRowBytes + q * 16);
          if (c0 + r < tc.ntok)
            *reinterpret_cast<uint4*>(out_tile + static_cast<size_t>(c0 + r) * p.ldo + q * 8) = v;
        }
        __syncwarp();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(acc == 0 ? tempty0 : tempty1);  // leader's barrier
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no CTA frees its memory while the pair's MMAs may read it
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
}

template <int MODE>
cudaError_t launch_pair(const PairMaps& maps, const PairParams& p, long long tiles_bound,
                        cudaStream_t s) {
  using C = PairCfg<MODE>;
  static DeviceOnce once;
  cudaError_t e = once.run([] {
    cudaError_t r = cudaFuncSetAttribute(grouped_gemm_pair_kernel<MODE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (r != cudaSuccess) return r;
    return prefer_max_shared(grouped_gemm_pair_kernel<MODE>);
  });
  if (e != cudaSuccess) return e;
  // A persistent kernel needs every pair resident at once: launch no more pairs than the
  // device can co-schedule as 2-CTA clusters with this shared-memory footprint (clusters
  // live inside one GPC, so that can be fewer than SMs / 2).
  int pairs_max = sm_count() / 2;
  {
    cudaLaunchConfig_t q = {};
    q.gridDim = dim3(2 * pairs_max);
    q.blockDim = dim3(kThreads);
    q.dynamicSmemBytes = C::SMEM;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    q.attrs = attr;
    q.numAttrs = 1;
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, grouped_gemm_pair_kernel<MODE>, &q) == cudaSuccess &&
        clusters > 0 && clusters < pairs_max)
      pairs_max = clusters;
  }
  const int pairs = static_cast<int>(tiles_bound < pairs_max ? (tiles_bound > 0 ? tiles_bound : 1)
                                                             : pairs_max);
  return launch_pdl_cluster(grouped_gemm_pair_kernel<MODE>, dim3(2 * pairs), dim3(kThreads), C::SMEM,
                            2, s, maps, p);
}

}  // namespace

cudaError_t launch_ffn_pair_sm100(const moe_config& c, const FfnArgs& f, cudaStream_t s,
                                  cudaEvent_t mid) {
  if (c.d % 256 != 0 || c.d_ff % 256 != 0) return cudaErrorInvalidValue;  // 256-row weight blocks
  const int nseg = c.E + (c.has_shared ? 1 : 0);
  const long long rows_h = f.rmax + (c.has_shared ? c.T : 0);

  PairMaps m1;
  bool ok = encode_2d_box(&m1.x_routed, f.x_packed, c.d, f.rmax, kTokBox) &&
            encode_2d_box(&m1.w0_routed, f.w_gate, c.d, static_cast<uint64_t>(c.E) * c.d_ff, BW) &&
            encode_2d_box(&m1.w1_routed, f.w_up, c.d, static_cast<uint64_t>(c.E) * c.d_ff, BW);
  if (c.has_shared)
    ok = ok && encode_2d_box(&m1.x_shared, f.x, c.d, c.T, kTokBox) &&
         encode_2d_box(&m1.w0_shared, f.s_gate, c.d, c.d_ff, BW) &&
         encode_2d_box(&m1.w1_shared, f.s_up, c.d, c.d_ff, BW);
  else
    m1.x_shared = m1.x_routed, m1.w0_shared = m1.w0_routed, m1.w1_shared = m1.w1_routed;
  if (!ok) return cudaErrorInvalidValue;
  PairParams p1{f.offsets, f.counts, nseg, c.E, c.d, c.d_ff, static_cast<__nv_bfloat16*>(f.h),
                c.d_ff, f.status, kWaitLimitNs};
  const long long tb1 = (rows_h + PairCfg<0>::NT - 1) / PairCfg<0>::NT + nseg;
  cudaError_t e = launch_pair<0>(m1, p1, tb1 * (c.d_ff / (2 * BW)), s);
  if (e != cudaSuccess) return e;
  if (mid != nullptr && (e = record_event(mid, s)) != cudaSuccess) return e;

  PairMaps m2;
  ok = encode_2d_box(&m2.x_routed, f.h, c.d_ff, rows_h, kTokBox) &&
       encode_2d_box(&m2.w0_routed, f.w_down, c.d_ff, static_cast<uint64_t>(c.E) * c.d, BW);
  if (c.has_shared)
    ok = ok && encode_2d_box(&m2.w0_shared, f.s_down, c.d_ff, c.d, BW);
  else
    m2.w0_shared = m2.w0_routed;
  m2.x_shared = m2.x_routed;
  m2.w1_routed = m2.w0_routed;
  m2.w1_shared = m2.w0_shared;
  if (!ok) return cudaErrorInvalidValue;
  PairParams p2{f.offsets, f.counts, nseg, c.E, c.d_ff, c.d,
                static_cast<__nv_bfloat16*>(f.y_packed), c.d, f.status, kWaitLimitNs};
  const long long tb2 = (rows_h + PairCfg<1>::NT - 1) / PairCfg<1>::NT + nseg;
  return launch_pair<1>(m2, p2, tb2 * (c.d / (2 * BW)), s);
}

}  // namespace moe

// bf16 expert FFN, row tiles over a pair of SMs (tcgen05 cta_group::2).  Same products as
// gemm_sm100.cu:
//   gate/up:  H[r, f] = SiLU(sum_i X[r,i] Wg_e[f,i]) * (sum_i X[r,i] Wu_e[f,i])
//   down:     Y[r, c] = sum_f H[r,f] Wd_e[c,f]
// Source: "MoE Inference Visualized", Expert Execution; "271,104 Routes: What I Missed About
// Mixture-of-Experts", sections 3 and 5.
//
// A pair tile is 256 token rows x 256 weight rows.  One M = 256, N = 256 MMA per K = 16 step
// takes the token rows 0..127 from the leader's shared memory and 128..255 from the peer's,
// and the weight rows 0..127 from the leader's and 128..255 from the peer's; each CTA ends up
// with its 128 token rows x all 256 columns in its own tensor memory, exactly the row-tile
// kernel's accumulator.  In the gate/up GEMM the leader holds the 128 W_gate rows and the
// peer the same 128 W_up rows, so the SwiGLU stays local to each CTA's epilogue.
//
// Why: each SM stages 32 KB per k-block instead of the one-SM row tile's 48 KB, so six
// k-blocks fit in the ring instead of four, and the two SMs stream different halves of the
// weight tile instead of the same tile in step.
//
// A cluster of 2 CTAs per pair; rank 0 (the leader) issues the MMAs.  Per CTA, 10 warps:
//   warp 8    TMA producer: its 128 token rows and its 128 weight rows per k-block; the
//             loads signal the leader's stage barrier (which expects both CTAs' bytes).
//   warp 9    leader: the pair MMAs; commits free both CTAs' stage and announce a finished
//             accumulator to both.  Both CTAs' warp 9 allocate and free the tensor memory.
//   warps 0-7 epilogue, in both CTAs: the row-tile kernel's (SiLU(gate) * up or plain
//             conversion, staged through shared memory into 64-byte row segments); each
//             warp then tells the leader that the accumulator has been read.
// Every wait is bounded; on a timeout the CTA records MOE_ERR_TIMEOUT and stops.  No TMA
// multicast is used: each CTA loads its own operand rows.
#include "gemm_common.cuh"
#include "internal.h"

namespace moe {
namespace {

using gemm::BK;
using gemm::kMaxSeg;
using gemm::find_seg;
using gemm::pack_bf16;
using gemm::silu_f;

constexpr int BM = 128;           // token rows per CTA (the pair: 256)
constexpr int BN = 256;           // weight rows of a pair tile (128 per CTA)
constexpr int kEpiWarps = 8;
constexpr int kProducerWarp = kEpiWarps;
constexpr int kMmaWarp = kEpiWarps + 1;
constexpr int kThreads = 32 * (kEpiWarps + 2);
constexpr int kStageRowBytes = 80;
constexpr int kEpiStageBytes = 32 * kStageRowBytes;
constexpr int kHalfBytes = 128 * BK * 2;        // one 128-row box: 16 KB
constexpr int kStageBytes = 2 * kHalfBytes;     // this CTA's token rows + weight rows
constexpr int kStages = 6;
constexpr int kTmemCols = 2 * BN;               // two accumulators of 256 columns
constexpr int kSmem = 1024 + kStages * kStageBytes + kEpiWarps * kEpiStageBytes + 256 +
                      3 * kMaxSeg * 4;

struct RowPairMaps {
  CUtensorMap a_routed;   // packed rows (gate/up) or H (down): [rows, K], 128-row boxes
  CUtensorMap a_shared;   // x [T, K] for the shared expert in the gate/up GEMM
  CUtensorMap b0_routed;  // W_gate or W_down, experts stacked: [E*N, K]
  CUtensorMap b1_routed;  // W_up [E*N, K]
  CUtensorMap b0_shared;  // shared expert [N, K]
  CUtensorMap b1_shared;
};

struct RowPairParams {
  const int32_t* offsets;
  const int32_t* counts;
  int nseg, E, K, N;      // N: output columns of the whole problem (F or d)
  __nv_bfloat16* out;
  int ldo;
  int32_t* status;
  int64_t limit_ns;
  int routed, shared;     // which segments this launch runs (see build_segment_table)
};

template <int MODE>  // 0: SwiGLU gate|up; 1: down
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_rowpair_kernel(const __grid_constant__ RowPairMaps maps, const RowPairParams p) {
  constexpr int OUT_COLS = (MODE == 0) ? BN / 2 : BN;  // output columns of a pair tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = base;                                  // [kStages][128 x 64]
  uint8_t* sB = base + kStages * kHalfBytes;           // [kStages][128 x 64]
  uint8_t* sEpi = sB + kStages * kHalfBytes;
  uint8_t* ctl = sEpi + kEpiWarps * kEpiStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(ctl);   // the leader's are the ones used
  uint64_t* empty = full + 8;
  uint64_t* tfull = empty + 8;
  uint64_t* tempty = tfull + 2;                        // the leader's are the ones used
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
  const int n_blocks = p.N / OUT_COLS;
  const int k_blocks = p.K / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(&tfull[b], 1); mbar_init(&tempty[b], 2 * kEpiWarps); }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kProducerWarp && lane == 0) {
    tma_prefetch_desc(&maps.a_routed);
    tma_prefetch_desc(&maps.b0_routed);
    if (MODE == 0) tma_prefetch_desc(&maps.b1_routed);
  }
  if (warp == kMmaWarp) {
    tmem_alloc_pair(tmem_slot, kTmemCols);
    tmem_relinquish_pair();
  }
  pdl_trigger();
  pdl_wait();  // offsets, A rows and the output buffer belong to earlier kernels
  if (warp == 0)
    gemm::build_segment_table(p.offsets, p.counts, p.nseg, p.E, 2 * BM, n_blocks, s_pre, s_row0,
                              s_rows, p.routed != 0, p.shared != 0);
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
      const int s = find_seg(s_pre, p.nseg, tile);
      const int mt = (s_rows[s] + 2 * BM - 1) / (2 * BM);
      const int local = tile - s_pre[s];
      const int n = local / mt, m = local - n * mt;
      const bool shared = (s == p.E);
      const CUtensorMap* ma = (MODE == 0 && shared) ? &maps.a_shared : &maps.a_routed;
      const int a_row = ((MODE == 0 && shared) ? 0 : s_row0[s]) + m * 2 * BM +
                        static_cast<int>(rank) * BM;
      const CUtensorMap* mb;
      int b_row;
      if (MODE == 0) {  // leader: W_gate rows, peer: the same W_up rows
        mb = shared ? (leader ? &maps.b0_shared : &maps.b1_shared)
                    : (leader ? &maps.b0_routed : &maps.b1_routed);
        b_row = (shared ? 0 : s * p.N) + n * OUT_COLS;
      } else {
        mb = shared ? &maps.b0_shared : &maps.b0_routed;
        b_row = (shared ? 0 : s * p.N) + n * BN + static_cast<int>(rank) * (BN / 2);
      }
      for (int kb = 0; kb < k_blocks; ++kb) {
        if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, p.limit_ns, p.status)) {
          ok = false;
          break;
        }
        if (leader) mbar_arrive_expect_tx(&full[stage], 2 * kStageBytes);  // both CTAs' bytes
        const uint32_t bar = cluster_map(&full[stage], 0);
        const int kx = kb * BK;
        tma_load_2d_pair(sA + stage * kHalfBytes, ma, bar, kx, a_row);
        tma_load_2d_pair(sB + stage * kHalfBytes, mb, bar, kx, b_row);
        if (++stage == kStages) { stage = 0; phase ^= 1u; wrapped = true; }
      }
    }
    if (!ok && leader) {  // drain the copies the leader's barriers still count
      for (int s = 0; s < kStages; ++s) {
        if (!wrapped && s >= stage) continue;
        const uint32_t par = (s < stage) ? phase : (phase ^ 1u);
        mbar_wait_bounded(&full[s], par, nullptr, p.limit_ns, p.status);
      }
    }
  } else if (warp == kMmaWarp && lane == 0 && leader) {
    // ------------------------------------------------------------ MMA issuer (leader)
    constexpr uint32_t idesc = idesc_bf16_f32(2 * BM, BN);
    int stage = 0, acc = 0;
    uint32_t phase = 0, acc_phase = 0;
    bool ok = true;
    for (int tile = pair; tile < total && ok; tile += npairs) {
      if (!mbar_wait_bounded(&tempty[acc], acc_phase ^ 1u, abort_flag, p.limit_ns, p.status)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
      for (int kb = 0; kb < k_blocks; ++kb) {
        if (!mbar_wait_bounded(&full[stage], phase, abort_flag, p.limit_ns, p.status)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t ad = smem_desc_k_sw128(sA + stage * kHalfBytes);
        const uint64_t bd = smem_desc_k_sw128(sB + stage * kHalfBytes);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk)  // advance 16 elements = 32 bytes along K
          tc_mma_bf16_pair(d_tmem, ad + 2 * kk, bd + 2 * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
        tc_commit_pair_mc(&empty[stage], 0x3);  // frees the stage in both CTAs
        if (++stage == kStages) { stage = 0; phase ^= 1u; }
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
    // Warp w reads TMEM lanes 32*(w%4).. (this CTA's tile rows) and half of the output
    // columns (w/4); 32 x 32 chunks are converted, staged in the warp's padded shared-memory
    // slice and written back as 64-byte row segments, only for rows of the segment.
    const int quarter = warp & 3, half = warp >> 2;
    constexpr int COLS = OUT_COLS / 2;
    uint8_t* stage_mem = sEpi + warp * kEpiStageBytes;
    const uint32_t tempty0 = cluster_map(&tempty[0], 0);
    const uint32_t tempty1 = cluster_map(&tempty[1], 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = pair; tile < total; tile += npairs) {
      const int s = find_seg(s_pre, p.nseg, tile);
      const int rows = s_rows[s];
      const int mt = (rows + 2 * BM - 1) / (2 * BM);
      const int local = tile - s_pre[s];
      const int n = local / mt, m = local - n * mt;
      int ok = 1;
      if (lane == 0) ok = mbar_wait_bounded(&tfull[acc], acc_phase, abort_flag, p.limit_ns, p.status);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                             static_cast<uint32_t>(acc * BN);
      const int r0 = m * 2 * BM + static_cast<int>(rank) * BM;  // this CTA's first tile row
      const int valid = rows - r0 - quarter * 32;  // rows of this warp's 32 that exist
      __nv_bfloat16* out0 = p.out + static_cast<size_t>(s_row0[s] + r0 + quarter * 32) * p.ldo +
                            static_cast<size_t>(n) * OUT_COLS + half * COLS;
#pragma unroll 1
      for (int c0 = 0; c0 < COLS && valid > 0; c0 += 32) {
        uint32_t o[16];
        if (MODE == 0) {
          uint32_t g[32], u[32];
          tmem_ld_32x32b_x32(t_row + half * COLS + c0, g);
          tmem_ld_32x32b_x32(t_row + BN / 2 + half * COLS + c0, u);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float h0 = silu_f(__uint_as_float(g[2 * i])) * __uint_as_float(u[2 * i]);
            const float h1 = silu_f(__uint_as_float(g[2 * i + 1])) * __uint_as_float(u[2 * i + 1]);
            o[i] = pack_bf16(h0, h1);
          }
        } else {
          uint32_t v[32];
          tmem_ld_32x32b_x32(t_row + half * COLS + c0, v);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 16; ++i)
            o[i] = pack_bf16(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
        }
        uint4* srow = reinterpret_cast<uint4*>(stage_mem + lane * kStageRowBytes);
#pragma unroll
        for (int q = 0; q < 4; ++q) srow[q] = make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = i * 8 + (lane >> 2), q = lane & 3;
          const uint4 v = *reinterpret_cast<const uint4*>(stage_mem + r * kStageRowBytes + q * 16);
          if (r < valid)
            *reinterpret_cast<uint4*>(out0 + static_cast<size_t>(r) * p.ldo + c0 + q * 8) = v;
        }
        __syncwarp();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(acc == 0 ? tempty0 : tempty1);  // the leader's barrier
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no CTA frees its memory while the pair's MMAs may read it
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc_pair(tmem_base, kTmemCols);
}

template <int MODE>
cudaError_t launch_rowpair(const RowPairMaps& maps, const RowPairParams& p, long long tiles_bound,
                           cudaStream_t s) {
  static DeviceOnce once;
  cudaError_t e = once.run([] {
    cudaError_t r = cudaFuncSetAttribute(grouped_gemm_rowpair_kernel<MODE>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
    if (r != cudaSuccess) return r;
    return prefer_max_shared(grouped_gemm_rowpair_kernel<MODE>);
  });
  if (e != cudaSuccess) return e;
  // A persistent kernel needs every pair resident at once: no more pairs than the device
  // can co-schedule as 2-CTA clusters with this shared-memory footprint.
  int pairs_max = sm_count() / 2;
  {
    cudaLaunchConfig_t q = {};
    q.gridDim = dim3(2 * pairs_max);
    q.blockDim = dim3(kThreads);
    q.dynamicSmemBytes = kSmem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    q.attrs = attr;
    q.numAttrs = 1;
    int clusters = 0;
    if (cudaOccupancyMaxActiveClusters(&clusters, grouped_gemm_rowpair_kernel<MODE>, &q) ==
            cudaSuccess &&
        clusters > 0 && clusters < pairs_max)
      pairs_max = clusters;
  }
  const int pairs = static_cast<int>(tiles_bound < pairs_max ? (tiles_bound > 0 ? tiles_bound : 1)
                                                             : pairs_max);
  return launch_pdl_cluster(grouped_gemm_rowpair_kernel<MODE>, dim3(2 * pairs), dim3(kThreads),
                            kSmem, 2, s, maps, p);
}

}  // namespace

static bool rowpair_fits(const moe_config& c) { return c.d % BN == 0 && c.d_ff % (BN / 2) == 0; }

cudaError_t launch_rowpair_gate_up(const moe_config& c, const FfnArgs& f, cudaStream_t s,
                                   bool routed, bool shared) {
  if (!rowpair_fits(c)) return cudaErrorInvalidValue;
  const int nseg = c.E + (c.has_shared ? 1 : 0);
  const long long rows = (routed ? f.rmax : 0) + (c.has_shared && shared ? c.T : 0);
  const long long mt_bound = (rows + 2 * BM - 1) / (2 * BM) + nseg;
  // A = packed rows [rmax, d] (x [T, d] for the shared expert)
  RowPairMaps m;
  bool ok = encode_2d_box(&m.a_routed, f.x_packed, c.d, f.rmax, BM) &&
            encode_2d_box(&m.b0_routed, f.w_gate, c.d, static_cast<uint64_t>(c.E) * c.d_ff, BN / 2) &&
            encode_2d_box(&m.b1_routed, f.w_up, c.d, static_cast<uint64_t>(c.E) * c.d_ff, BN / 2);
  if (c.has_shared)
    ok = ok && encode_2d_box(&m.a_shared, f.x, c.d, c.T, BM) &&
         encode_2d_box(&m.b0_shared, f.s_gate, c.d, c.d_ff, BN / 2) &&
         encode_2d_box(&m.b1_shared, f.s_up, c.d, c.d_ff, BN / 2);
  else
    m.a_shared = m.a_routed, m.b0_shared = m.b0_routed, m.b1_shared = m.b1_routed;
  if (!ok) return cudaErrorInvalidValue;
  RowPairParams p{f.offsets, f.counts, nseg, c.E, c.d, c.d_ff, static_cast<__nv_bfloat16*>(f.h),
                  c.d_ff, f.status, kWaitLimitNs, routed ? 1 : 0, shared ? 1 : 0};
  return launch_rowpair<0>(m, p, mt_bound * (c.d_ff / (BN / 2)), s);
}

cudaError_t launch_rowpair_down(const moe_config& c, const FfnArgs& f, cudaStream_t s,
                                bool routed, bool shared) {
  if (!rowpair_fits(c)) return cudaErrorInvalidValue;
  const int nseg = c.E + (c.has_shared ? 1 : 0);
  const long long rows_h = f.rmax + (c.has_shared ? c.T : 0);
  const long long rows = (routed ? f.rmax : 0) + (c.has_shared && shared ? c.T : 0);
  const long long mt_bound = (rows + 2 * BM - 1) / (2 * BM) + nseg;
  // A = H [rows_h, F]
  RowPairMaps m;
  bool ok = encode_2d_box(&m.a_routed, f.h, c.d_ff, rows_h, BM) &&
            encode_2d_box(&m.b0_routed, f.w_down, c.d_ff, static_cast<uint64_t>(c.E) * c.d, BN / 2);
  if (c.has_shared)
    ok = ok && encode_2d_box(&m.b0_shared, f.s_down, c.d_ff, c.d, BN / 2);
  else
    m.b0_shared = m.b0_routed;
  m.a_shared = m.a_routed;
  m.b1_routed = m.b0_routed;
  m.b1_shared = m.b0_shared;
  if (!ok) return cudaErrorInvalidValue;
  RowPairParams p{f.offsets, f.counts, nseg, c.E, c.d_ff, c.d,
                  static_cast<__nv_bfloat16*>(f.y_packed), c.d, f.status, kWaitLimitNs,
                  routed ? 1 : 0, shared ? 1 : 0};
  return launch_rowpair<1>(m, p, mt_bound * (c.d / BN), s);
}

cudaError_t launch_ffn_rowpair_sm100(const moe_config& c, const FfnArgs& f, cudaStream_t s,
                                     cudaEvent_t mid) {
  cudaError_t e = launch_rowpair_gate_up(c, f, s, true, true);
  if (e != cudaSuccess) return e;
  if (mid != nullptr && (e = record_event(mid, s)) != cudaSuccess) return e;
  return launch_rowpair_down(c, f, s, true, true);
}

}  // namespace moe

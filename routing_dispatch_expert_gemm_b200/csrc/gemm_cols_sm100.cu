// bf16 expert FFN on the 5th-generation tensor cores, column tiles: the weights sit on the
// MMA's M side (128 weight rows per tile) and the expert segment's tokens on its N side
// (a multiple of 16, up to 128 per tile).  Same products as gemm_sm100.cu:
//   gate/up:  H[r, f] = SiLU(sum_i X[r,i] Wg_e[f,i]) * (sum_i X[r,i] Wu_e[f,i])
//   down:     Y[r, c] = sum_f H[r,f] Wd_e[c,f]
// computed as D = W X^T and written back transposed.
// Source: "MoE Inference Visualized", Expert Execution (down(SiLU(gate(x)) * up(x)));
// "271,104 Routes: What I Missed About Mixture-of-Experts", section 3 (one dense matmul per
// expert batch) and section 5 (with small batches the cost is moving the weights).
//
// Why a second tile shape: when experts receive few tokens (decode, or many experts with
// top-2), 128-row token tiles are mostly padding; a segment of 130 tokens costs two
// 128-row tiles (256 rows of MMA work) but only 144 token columns here.  The weights
// stream through the M side once per token block, exactly as in the row-tile kernel.
//
// Kernel shape (one CTA per SM, persistent, 10 warps), as in gemm_sm100.cu:
//   warp 8    TMA producer: per stage the weight tile(s) [128 rows x 64 K] (gate and up
//             for the gate/up GEMM) and the token tile [16 * nbox rows x 64 K], loaded as
//             nbox boxes of 16 rows, 128-byte swizzle, into a STAGES-deep ring.
//   warp 9    MMA issuer: tcgen05.mma kind::f16 M=128, N=16*nbox, K=16 x 4 per stage
//             (twice for gate/up: gate and up accumulators side by side); two
//             accumulator sets in tensor memory so the epilogue overlaps the next tile.
//   warps 0-7 epilogue: warp w reads TMEM lanes 32(w%4).. (weight rows) and token columns
//             64(w/4)..; each thread holds 32 tokens of one weight row, so the bf16 results
//             are transposed through shared memory and written as 64-byte row segments of
//             the token-major output, only for the tile's tokens.
// Fused steps (moe_forward with MOE_FUSE_*; bit-identical to the unfused path):
//   gather   4 more warps fill each stage's token tile straight from x by row_token with
//            16-byte cp.async copies, placing each chunk where the 128-byte swizzle puts it
//            (chunk c of row r at c ^ (r % 8)); each thread waits for its own copies, makes
//            them visible to the tensor core's proxy and arrives on the stage's barrier,
//            two stages behind its issue point.  The shared expert's tile (rows of x in
//            order) still comes by TMA.  No packed copy of the token rows is made.
//   combine  after the down GEMM's epilogue writes a token's 32 columns, the token's counter
//            for that column chunk is incremented; the tile that completes it (all of the
//            token's kept routes and the shared expert) sums the token's rows of y_packed
//            for those columns in slot order, adds the shared row and the residual, and
//            writes y: the same operations, in the same order, as the combine kernel.
// Tiles are ordered (segment, weight block, token block), token block fastest: CTAs running
// at the same time share a weight tile through L2, and the segment's tokens stay in L2
// while its weight blocks stream.  Every wait is bounded; on a timeout the CTA records
// MOE_ERR_TIMEOUT, drains its copies and MMAs, frees its tensor memory and returns.
// No TMA multicast is used.
#include "gemm_common.cuh"
#include "internal.h"

namespace moe {
namespace {

using gemm::BK;
using gemm::kMaxSeg;
using gemm::find_seg;
using gemm::silu_f;

constexpr int BW = 128;          // weight rows per tile (MMA M)
constexpr int NT = 128;          // token columns per tile, at most (MMA N)
constexpr int kTokBox = 16;      // token rows per TMA box (MMA N granularity)
constexpr int kEpiWarps = 8;
constexpr int kProducerWarp = kEpiWarps;
constexpr int kMmaWarp = kEpiWarps + 1;
constexpr int kGatherWarp0 = kEpiWarps + 2;   // gather warps 10..13 (fused gather only)
constexpr int kGatherThreads = 128;
constexpr int kGatherDepth = 2;               // stages a gather thread keeps in flight
template <bool GATHER>
constexpr int threads_of() { return 32 * (kEpiWarps + 2) + (GATHER ? kGatherThreads : 0); }
constexpr int kStageRowBytes = 80;  // 32 bf16 of a token row + 16 B pad
constexpr int kEpiStageBytes = 32 * kStageRowBytes;
constexpr int W_BYTES = BW * BK * 2;
constexpr int X_BYTES = NT * BK * 2;
constexpr int kBoxBytes = kTokBox * BK * 2;

struct ColMaps {
  CUtensorMap x_routed;   // tokens: packed rows [rmax, d] (gate/up) or H [rows_h, F] (down)
  CUtensorMap x_shared;   // x [T, d]: the shared expert's tokens in the gate/up GEMM
  CUtensorMap x_routed_full;  // the same two with 128-row boxes: one load for a full
  CUtensorMap x_shared_full;  // token block (more than 112 tokens)
  CUtensorMap w0_routed;  // W_gate or W_down, experts stacked: [E*N, K]
  CUtensorMap w1_routed;  // W_up [E*N, K]
  CUtensorMap w0_shared;  // shared expert [N, K]
  CUtensorMap w1_shared;
};

struct ColParams {
  const int32_t* offsets;  // [nseg + 1] segment row starts
  const int32_t* counts;   // [E] rows of each routed segment, or null
  int nseg, E, K, N;       // N: weight rows of one expert (F or d) = output columns
  __nv_bfloat16* out;
  int ldo;
  int32_t* status;
  int64_t limit_ns;
  const __nv_bfloat16* xg;     // gather: token rows x [T, K]
  const int32_t* gather_rows;  // gather: row_token [Rmax]
  FusedCombine fc;             // combine in the epilogue when fc.counters != null
};

template <int MODE>  // 0: SwiGLU gate|up; 1: down
struct ColCfg {
  static constexpr int NW = (MODE == 0) ? 2 : 1;  // weight tiles per stage
  static constexpr int STAGE_BYTES = NW * W_BYTES + X_BYTES;
  static constexpr int STAGES = (MODE == 0) ? 4 : 6;
  static constexpr int ACC_COLS = NW * NT;        // TMEM columns of one accumulator set
  static constexpr int TMEM_COLS = 2 * ACC_COLS;  // double-buffered: 512 / 256
  static constexpr int SMEM =
      1024 + STAGES * STAGE_BYTES + kEpiWarps * kEpiStageBytes + 256 + 3 * kMaxSeg * 4;
};

struct TileCoord {
  int s, wb, tb, ntok;
};

__device__ __forceinline__ TileCoord decode_tile(const int* s_pre, const int* s_rows, int nseg,
                                                 int tile) {
  TileCoord c;
  c.s = find_seg(s_pre, nseg, tile);
  const int rows = s_rows[c.s];
  const int tbc = (rows + NT - 1) / NT;
  const int local = tile - s_pre[c.s];
  c.wb = local / tbc;
  c.tb = local - c.wb * tbc;
  c.ntok = min(NT, rows - c.tb * NT);
  return c;
}

// The fused combine of one token's 32-column chunk cc (see the file comment): the token's
// rows of y_packed are read past L1 (other SMs wrote them during this kernel).
__device__ __forceinline__ void fused_combine_chunk(const ColParams& p, int shared_base, int t,
                                                    int cc) {
  const FusedCombine& f = p.fc;
  const int d = p.N;
  float acc[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) acc[i] = 0.f;
  const size_t col = static_cast<size_t>(cc) * 32;
#pragma unroll 1
  for (int j = 0; j < f.k; ++j) {
    const int r = __ldg(f.route_row + static_cast<size_t>(t) * f.k + j);
    if (r < 0) continue;  // a dropped route contributes nothing
    const float g = __ldg(f.gates + static_cast<size_t>(t) * f.k + j);
    const uint4* src = reinterpret_cast<const uint4*>(p.out + static_cast<size_t>(r) * d + col);
    uint4 v[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) v[q] = __ldcg(src + q);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float fv[8];
      Vec<__nv_bfloat16>::to_f32(v[q], fv);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[q * 8 + i] = fmaf(g, fv[i], acc[q * 8 + i]);
    }
  }
  if (f.has_shared) {
    const uint4* src =
        reinterpret_cast<const uint4*>(p.out + static_cast<size_t>(shared_base + t) * d + col);
    uint4 v[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) v[q] = __ldcg(src + q);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float fv[8];
      Vec<__nv_bfloat16>::to_f32(v[q], fv);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[q * 8 + i] += fv[i];
    }
  }
  if (f.residual != nullptr) {
    const uint4* src = reinterpret_cast<const uint4*>(
        static_cast<const __nv_bfloat16*>(f.residual) + static_cast<size_t>(t) * d + col);
    uint4 v[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) v[q] = __ldg(src + q);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float fv[8];
      Vec<__nv_bfloat16>::to_f32(v[q], fv);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[q * 8 + i] += fv[i];
    }
  }
  uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(f.y) +
                                        static_cast<size_t>(t) * d + col);
#pragma unroll
  for (int q = 0; q < 4; ++q) dst[q] = Vec<__nv_bfloat16>::from_f32(acc + q * 8);
}

__device__ __forceinline__ void cp_async_wait_depth() {
  asm volatile("cp.async.wait_group %0;" ::"n"(kGatherDepth) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

template <int MODE, bool GATHER>
__global__ void __launch_bounds__(threads_of<GATHER>(), 1)
    grouped_gemm_cols_kernel(const __grid_constant__ ColMaps maps, const ColParams p) {
  using C = ColCfg<MODE>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sW = base;                                  // [STAGES][NW][128 x 64] bf16
  uint8_t* sX = sW + C::STAGES * C::NW * W_BYTES;      // [STAGES][128 x 64] bf16
  uint8_t* sEpi = sX + C::STAGES * X_BYTES;            // per epilogue warp: 32 rows x 80 B
  uint8_t* ctl = sEpi + kEpiWarps * kEpiStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(ctl);
  uint64_t* empty = full + 8;
  uint64_t* tfull = empty + 8;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctl + 192);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(ctl + 196);
  int* s_pre = reinterpret_cast<int*>(ctl + 256);
  int* s_row0 = s_pre + kMaxSeg;
  int* s_rows = s_row0 + kMaxSeg;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_wblocks = p.N / BW;
  const int k_blocks = p.K / BK;

  if (threadIdx.x == 0) {
    // a stage is full when the producer's TMA bytes have landed and, with the fused gather,
    // every gather thread has arrived after its own copies
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1 + (GATHER ? kGatherThreads : 0));
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) { mbar_init(&tfull[b], 1); mbar_init(&tempty[b], kEpiWarps); }
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
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  pdl_trigger();
  pdl_wait();  // offsets, token rows and the output buffer belong to earlier kernels
  if (warp == 0)
    gemm::build_segment_table(p.offsets, p.counts, p.nseg, p.E, NT, n_wblocks, s_pre, s_row0,
                              s_rows);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int total = s_pre[p.nseg];

  if (warp == kProducerWarp && lane == 0) {
    // ------------------------------------------------------------ TMA producer
    int stage = 0;
    uint32_t phase = 0;
    bool wrapped = false, ok = true;
    for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
      const TileCoord tc = decode_tile(s_pre, s_rows, p.nseg, tile);
      const int nbox = (tc.ntok + kTokBox - 1) / kTokBox;
      const bool shared = (tc.s == p.E);
      const bool full_box = nbox * kTokBox > NT - kTokBox;  // 8 boxes: one 128-row load
      const CUtensorMap* mx =
          (MODE == 0 && shared) ? (full_box ? &maps.x_shared_full : &maps.x_shared)
                                : (full_box ? &maps.x_routed_full : &maps.x_routed);
      const int x_row = ((MODE == 0 && shared) ? 0 : s_row0[tc.s]) + tc.tb * NT;
      const CUtensorMap* mw0 = shared ? &maps.w0_shared : &maps.w0_routed;
      const CUtensorMap* mw1 = shared ? &maps.w1_shared : &maps.w1_routed;
      const int w_row = (shared ? 0 : tc.s * p.N) + tc.wb * BW;
      const bool tma_x = !GATHER || shared;  // else the gather warps fill the token tile
      const uint32_t bytes = C::NW * W_BYTES + (tma_x ? nbox * kBoxBytes : 0);
      for (int kb = 0; kb < k_blocks; ++kb) {
        if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, p.limit_ns, p.status)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&full[stage], bytes);
        uint8_t* w_dst = sW + stage * C::NW * W_BYTES;
        uint8_t* x_dst = sX + stage * X_BYTES;
        const int kx = kb * BK;
        tma_load_2d(w_dst, mw0, &full[stage], kx, w_row);
        if (MODE == 0) tma_load_2d(w_dst + W_BYTES, mw1, &full[stage], kx, w_row);
        if (tma_x) {
          if (full_box)
            tma_load_2d(x_dst, mx, &full[stage], kx, x_row);
          else
            for (int i = 0; i < nbox; ++i)
              tma_load_2d(x_dst + i * kBoxBytes, mx, &full[stage], kx, x_row + i * kTokBox);
        }
        if (++stage == C::STAGES) { stage = 0; phase ^= 1u; wrapped = true; }
      }
    }
    if (!ok) {  // drain our own copies in flight before the CTA leaves
      for (int s = 0; s < C::STAGES; ++s) {
        if (!wrapped && s >= stage) continue;
        const uint32_t par = (s < stage) ? phase : (phase ^ 1u);
        mbar_wait_bounded(&full[s], par, nullptr, p.limit_ns, p.status);
      }
    }
  } else if (warp == kMmaWarp && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    int stage = 0, acc = 0;
    uint32_t phase = 0, acc_phase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
      const TileCoord tc = decode_tile(s_pre, s_rows, p.nseg, tile);
      const int nbox = (tc.ntok + kTokBox - 1) / kTokBox;
      const uint32_t idesc = idesc_bf16_f32(BW, nbox * kTokBox);
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
        const uint64_t xd = smem_desc_k_sw128(sX + stage * X_BYTES);
        const uint64_t w0d = smem_desc_k_sw128(sW + stage * C::NW * W_BYTES);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk)  // 16 elements = 32 bytes along K
          tc_mma_bf16(d_tmem, w0d + 2 * kk, xd + 2 * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
        if (MODE == 0) {
          const uint64_t w1d = smem_desc_k_sw128(sW + stage * C::NW * W_BYTES + W_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            tc_mma_bf16(d_tmem + NT, w1d + 2 * kk, xd + 2 * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
        }
        tc_commit(&empty[stage]);  // frees the stage once these MMAs have read it
        if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
      tc_commit(&tfull[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    if (!ok) {  // wait for every MMA this thread issued before the memory goes away
      tc_commit(drain);
      mbar_wait_bounded(drain, 0, nullptr, p.limit_ns, p.status);
    }
  } else if (GATHER && warp >= kGatherWarp0) {
    // ------------------------------------------------------------ gather (fused)
    // Thread gi copies the 16-byte chunk gi % 8 of tile rows gi / 8 + 16 m, m = 0..7.
    const int gi = static_cast<int>(threadIdx.x) - kGatherWarp0 * 32;
    const int c16 = gi & 7, r0 = gi >> 3;
    int stage = 0, npend = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
      const TileCoord tc = decode_tile(s_pre, s_rows, p.nseg, tile);
      const bool shared = (tc.s == p.E);
      int tok[NT / 16];
#pragma unroll
      for (int m = 0; m < NT / 16; ++m) {
        const int ri = r0 + 16 * m;
        tok[m] = (!shared && ri < tc.ntok) ? __ldg(p.gather_rows + s_row0[tc.s] + tc.tb * NT + ri)
                                           : -1;
      }
      for (int kb = 0; kb < k_blocks; ++kb) {
        if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, p.limit_ns, p.status)) {
          ok = false;
          break;
        }
        uint8_t* x_dst = sX + stage * X_BYTES;
        const __nv_bfloat16* src0 = p.xg + static_cast<size_t>(kb) * BK + c16 * 8;
#pragma unroll
        for (int m = 0; m < NT / 16; ++m) {
          const int ri = r0 + 16 * m;
          if (tok[m] >= 0)
            cp_async_16(x_dst + ri * 128 + ((c16 ^ (ri & 7)) << 4),
                        src0 + static_cast<size_t>(tok[m]) * p.K);
        }
        cp_async_commit();
        ++npend;
        if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
        if (npend > kGatherDepth) {  // the oldest pending stage's copies are complete
          cp_async_wait_depth();
          fence_proxy_async_smem();
          const int old_stage = (stage - npend + 2 * C::STAGES) % C::STAGES;
          mbar_arrive(&full[old_stage]);
          --npend;
        }
      }
    }
    cp_async_wait_all();  // drain: every copy of this thread has landed
    if (ok) {
      fence_proxy_async_smem();
      for (; npend > 0; --npend) mbar_arrive(&full[(stage - npend + 2 * C::STAGES) % C::STAGES]);
    }
  } else if (warp < kEpiWarps) {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3, half = warp >> 2;
    uint8_t* stage_mem = sEpi + warp * kEpiStageBytes;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
      const TileCoord tc = decode_tile(s_pre, s_rows, p.nseg, tile);
      int ok = 1;
      if (lane == 0) ok = mbar_wait_bounded(&tfull[acc], acc_phase, abort_flag, p.limit_ns, p.status);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                              static_cast<uint32_t>(acc * C::ACC_COLS);
      // this warp's 32 weight rows = output columns col0 .. col0 + 31
      __nv_bfloat16* out_tile = p.out + static_cast<size_t>(s_row0[tc.s] + tc.tb * NT) * p.ldo +
                                static_cast<size_t>(tc.wb) * BW + quarter * 32;
#pragma unroll 1
      for (int c0 = half * (NT / 2); c0 < (half + 1) * (NT / 2) && c0 < tc.ntok; c0 += 32) {
        float h[32];
        if (MODE == 0) {
          uint32_t g[32], u[32];
          tmem_ld_32x32b_x32(t_lane + c0, g);
          tmem_ld_32x32b_x32(t_lane + NT + c0, u);
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
        // transpose: token i's row gets this lane's weight row as element `lane`
#pragma unroll
        for (int i = 0; i < 32; ++i)
          reinterpret_cast<__nv_bfloat16*>(stage_mem + i * kStageRowBytes)[lane] =
              __float2bfloat16_rn(h[i]);
        __syncwarp();
        // write back: 4 lanes per token row (64 bytes), 8 token rows per instruction
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = i * 8 + (lane >> 2), q = lane & 3;
          const uint4 v = *reinterpret_cast<const uint4*>(stage_mem + r * kStageRowBytes + q * 16);
          if (c0 + r < tc.ntok)
            *reinterpret_cast<uint4*>(out_tile + static_cast<size_t>(c0 + r) * p.ldo + q * 8) = v;
        }
        if (MODE == 1 && p.fc.counters != nullptr) {
          // fused combine: this warp's 32 columns of tokens c0 .. c0 + 31 are written;
          // lane l counts token c0 + l in and finishes its chunk if it is the last
          __threadfence();
          __syncwarp();
          const int r = c0 + lane;
          if (r < tc.ntok) {
            const int prow = s_row0[tc.s] + tc.tb * NT + r;
            const int t = (tc.s < p.E) ? __ldg(p.fc.row_token + prow) : prow - s_row0[p.E];
            const int cc = (tc.wb * BW + quarter * 32) >> 5;
            const int old = atomicAdd(p.fc.counters + static_cast<size_t>(t) * (p.N >> 5) + cc, 1);
            if (old == __ldg(p.fc.need + t) - 1) {
              __threadfence();  // every other contribution's stores are visible
              fused_combine_chunk(p, s_row0[p.E], t, cc);
            }
          }
        }
        __syncwarp();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

template <int MODE, bool GATHER>
cudaError_t launch_cols(const ColMaps& maps, const ColParams& p, long long tiles_bound,
                        cudaStream_t s) {
  using C = ColCfg<MODE>;
  static DeviceOnce once;
  cudaError_t e = once.run([] {
    cudaError_t r = cudaFuncSetAttribute(grouped_gemm_cols_kernel<MODE, GATHER>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (r != cudaSuccess) return r;
    return prefer_max_shared(grouped_gemm_cols_kernel<MODE, GATHER>);
  });
  if (e != cudaSuccess) return e;
  const int sms = sm_count();
  const int grid = static_cast<int>(tiles_bound < sms ? (tiles_bound > 0 ? tiles_bound : 1) : sms);
  return launch_pdl(grouped_gemm_cols_kernel<MODE, GATHER>, dim3(grid),
                    dim3(threads_of<GATHER>()), C::SMEM, s, maps, p);
}

}  // namespace

cudaError_t launch_ffn_cols_sm100(const moe_config& c, const FfnArgs& f, cudaStream_t s,
                                  cudaEvent_t mid) {
  const int nseg = c.E + (c.has_shared ? 1 : 0);
  const long long rows_h = f.rmax + (c.has_shared ? c.T : 0);
  const long long tb_bound = (rows_h + NT - 1) / NT + nseg;  // token blocks over all segments

  // gate/up + SwiGLU: tokens = packed rows [rmax, d] (x [T, d] for the shared expert)
  ColMaps m1;
  bool ok = encode_2d_box(&m1.x_routed, f.x_packed, c.d, f.rmax, kTokBox) &&
            encode_2d_box(&m1.x_routed_full, f.x_packed, c.d, f.rmax, NT) &&
            encode_2d_box(&m1.w0_routed, f.w_gate, c.d, static_cast<uint64_t>(c.E) * c.d_ff, BW) &&
            encode_2d_box(&m1.w1_routed, f.w_up, c.d, static_cast<uint64_t>(c.E) * c.d_ff, BW);
  if (c.has_shared)
    ok = ok && encode_2d_box(&m1.x_shared, f.x, c.d, c.T, kTokBox) &&
         encode_2d_box(&m1.x_shared_full, f.x, c.d, c.T, NT) &&
         encode_2d_box(&m1.w0_shared, f.s_gate, c.d, c.d_ff, BW) &&
         encode_2d_box(&m1.w1_shared, f.s_up, c.d, c.d_ff, BW);
  else
    m1.x_shared = m1.x_routed, m1.x_shared_full = m1.x_routed_full, m1.w0_shared = m1.w0_routed,
    m1.w1_shared = m1.w1_routed;
  if (!ok) return cudaErrorInvalidValue;
  ColParams p1{f.offsets, f.counts, nseg, c.E, c.d, c.d_ff, static_cast<__nv_bfloat16*>(f.h),
               c.d_ff, f.status, kWaitLimitNs, static_cast<const __nv_bfloat16*>(f.x),
               f.gather_rows, FusedCombine{}};
  if (f.gather_rows != nullptr && f.x == nullptr) return cudaErrorInvalidValue;
  cudaError_t e = f.gather_rows != nullptr ? launch_cols<0, true>(m1, p1, tb_bound * (c.d_ff / BW), s)
                                           : launch_cols<0, false>(m1, p1, tb_bound * (c.d_ff / BW), s);
  if (e != cudaSuccess) return e;
  if (mid != nullptr && (e = record_event(mid, s)) != cudaSuccess) return e;

  // down: tokens = H [rows_h, F]
  ColMaps m2;
  ok = encode_2d_box(&m2.x_routed, f.h, c.d_ff, rows_h, kTokBox) &&
       encode_2d_box(&m2.x_routed_full, f.h, c.d_ff, rows_h, NT) &&
       encode_2d_box(&m2.w0_routed, f.w_down, c.d_ff, static_cast<uint64_t>(c.E) * c.d, BW);
  if (c.has_shared)
    ok = ok && encode_2d_box(&m2.w0_shared, f.s_down, c.d_ff, c.d, BW);
  else
    m2.w0_shared = m2.w0_routed;
  m2.x_shared = m2.x_routed;
  m2.x_shared_full = m2.x_routed_full;
  m2.w1_routed = m2.w0_routed;
  m2.w1_shared = m2.w0_shared;
  if (!ok) return cudaErrorInvalidValue;
  ColParams p2{f.offsets, f.counts, nseg, c.E, c.d_ff, c.d, static_cast<__nv_bfloat16*>(f.y_packed),
               c.d, f.status, kWaitLimitNs, nullptr, nullptr,
               f.combine != nullptr ? *f.combine : FusedCombine{}};
  return launch_cols<1, false>(m2, p2, tb_bound * (c.d / BW), s);
}

}  // namespace moe

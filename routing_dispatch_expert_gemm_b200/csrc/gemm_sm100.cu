// bf16 expert FFN on the 5th-generation tensor cores: two persistent grouped GEMMs over
// the ragged expert segments produced by dispatch.
//   gate/up:  H[r, f] = SiLU(sum_i X[r,i] Wg_e[f,i]) * (sum_i X[r,i] Wu_e[f,i])
//   down:     Y[r, c] = sum_f H[r,f] Wd_e[c,f]
// Source: "MoE Inference Visualized", Expert Execution (down(SiLU(gate(x)) * up(x)));
// "271,104 Routes: What I Missed About Mixture-of-Experts", section 3 (one dense matmul per
// expert batch) and section 5 (once expert batches are large the matmuls dominate).
//
// Kernel shape (one CTA per SM, persistent, 10 warps):
//   warp 8    TMA producer: A tile [128 rows x 64 K] and B tile [BN rows x 64 K] per
//             stage, 128-byte swizzle, into a STAGES-deep shared-memory ring.
//   warp 9    MMA issuer: tcgen05.mma kind::f16 (bf16 in, fp32 accumulate) M=128,
//             N=BN, K=16 x 4 per stage into a tensor-memory accumulator; two accumulators
//             (2 x BN columns) so the epilogue of one tile overlaps the MMAs of the next.
//   warps 0-7 epilogue: tcgen05.ld of the accumulator (warp w owns TMEM lanes
//             32(w%4)..+31, i.e. tile rows, and half the columns), SiLU(gate)*up or plain
//             conversion to bf16, staged through shared memory so that the stores to
//             global memory are 64-byte row segments, only for rows of the segment.
// In the gate/up GEMM the B tile stacks 128 rows of W_gate over the same 128 rows of
// W_up, so one N=256 MMA produces both halves side by side in TMEM and the SwiGLU is
// applied in the epilogue with no extra pass.
// Tiles are ordered (segment, n-block, m-block), m fastest: CTAs running at the same time
// share weight tiles and the segment's packed rows through L2.
// Every wait is bounded (mbar_wait_bounded): if one runs out, the CTA records
// MOE_ERR_TIMEOUT, drains its own copies and MMAs, frees its tensor memory and returns.
// No TMA multicast is used.
#include <algorithm>

#include "gemm_common.cuh"
#include "internal.h"

namespace moe {

// Tensor map of a row-major bf16 matrix [rows, cols] read in boxes of 64 columns x
// box_rows rows with 128-byte swizzle; rows outside the matrix read as zero.
bool encode_2d_box(CUtensorMap* m, const void* ptr, uint64_t cols, uint64_t rows,
                   uint32_t box_rows) {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }();
  if (fn == nullptr || ptr == nullptr || rows == 0 || box_rows == 0 || box_rows > 256) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

using gemm::BK;
using gemm::kMaxSeg;
using gemm::find_seg;
using gemm::pack_bf16;
using gemm::silu_f;

constexpr int BM = 128;
constexpr int kEpiWarps = 8;                    // two per TMEM lane quarter
constexpr int kProducerWarp = kEpiWarps;        // warp 8
constexpr int kMmaWarp = kEpiWarps + 1;         // warp 9
constexpr int kThreads = 32 * (kEpiWarps + 2);
constexpr int kStageRowBytes = 80;              // 64 B of a row chunk + 16 B pad (no bank conflicts)
constexpr int kEpiStageBytes = 32 * kStageRowBytes;
constexpr int A_BYTES = BM * BK * 2;
constexpr int kBoxRows = 128;

struct Maps {
  CUtensorMap a_routed;   // packed rows (gate/up) or H (down): [rows, K]
  CUtensorMap a_shared;   // x [T, K] for the shared expert in the gate/up GEMM
  CUtensorMap b0_routed;  // W_gate or W_down, experts stacked: [E*N, K]
  CUtensorMap b1_routed;  // W_up [E*N, K]
  CUtensorMap b0_shared;  // shared expert [N, K]
  CUtensorMap b1_shared;
};

struct Params {
  const int32_t* offsets;  // [nseg + 1] segment row starts
  const int32_t* counts;   // [E] rows of each routed segment, or null: the gap to the next start
  int nseg, E, K, N;       // N: output columns of the whole problem (F or d)
  __nv_bfloat16* out;
  int ldo;
  int32_t* status;
  int64_t limit_ns;
  int routed, shared;      // which segments this launch runs (see build_segment_table)
};

template <int MODE, int BN>  // MODE 0: SwiGLU gate|up (BN = 256); MODE 1: plain (128/256)
struct Cfg {
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = (BN == 256) ? 4 : 6;
  static constexpr int OUT_COLS = (MODE == 0) ? BN / 2 : BN;
  static constexpr int TMEM_COLS = 2 * BN;
  static constexpr int SMEM =
      1024 + STAGES * STAGE_BYTES + kEpiWarps * kEpiStageBytes + 256 + 3 * kMaxSeg * 4;
};

template <int MODE, int BN>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ Maps maps, const Params p) {
  using C = Cfg<MODE, BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* sA = base;
  uint8_t* sB = base + C::STAGES * A_BYTES;
  uint8_t* sEpi = sB + C::STAGES * C::B_BYTES;  // per epilogue warp: 32 rows x 80 B
  uint8_t* ctl = sEpi + kEpiWarps * kEpiStageBytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(ctl);
  uint64_t* empty = full + 8;
  uint64_t* tfull = empty + 8;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ctl + 192);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(ctl + 196);
  int* s_pre = reinterpret_cast<int*>(ctl + 256);  // tile prefix per segment
  int* s_row0 = s_pre + kMaxSeg;                   // segment row starts
  int* s_rows = s_row0 + kMaxSeg;                  // segment row counts

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_blocks = p.N / C::OUT_COLS;
  const int k_blocks = p.K / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(&tfull[b], 1); mbar_init(&tempty[b], kEpiWarps); }
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
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  pdl_trigger();
  pdl_wait();  // offsets, A rows and the output buffer belong to earlier kernels
  if (warp == 0)  // segment table: row starts and exclusive prefix of tile counts
    gemm::build_segment_table(p.offsets, p.counts, p.nseg, p.E, BM, n_blocks, s_pre, s_row0,
                              s_rows, p.routed != 0, p.shared != 0);
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
      const int s = find_seg(s_pre, p.nseg, tile);
      const int mt = (s_rows[s] + BM - 1) / BM;
      const int local = tile - s_pre[s];
      const int n = local / mt, m = local - n * mt;
      const bool shared = (s == p.E);
      const CUtensorMap* ma = (MODE == 0 && shared) ? &maps.a_shared : &maps.a_routed;
      const int a_row = ((MODE == 0 && shared) ? 0 : s_row0[s]) + m * BM;
      const CUtensorMap* mb0 = shared ? &maps.b0_shared : &maps.b0_routed;
      const CUtensorMap* mb1 = shared ? &maps.b1_shared : &maps.b1_routed;
      const int b_row = (shared ? 0 : s * p.N) + n * C::OUT_COLS;
      for (int kb = 0; kb < k_blocks; ++kb) {
        if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, p.limit_ns, p.status)) {
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
        uint8_t* a_dst = sA + stage * A_BYTES;
        uint8_t* b_dst = sB + stage * C::B_BYTES;
        const int kx = kb * BK;
        tma_load_2d(a_dst, ma, &full[stage], kx, a_row);
        if (MODE == 0) {
          tma_load_2d(b_dst, mb0, &full[stage], kx, b_row);
          tma_load_2d(b_dst + kBoxRows * 128, mb1, &full[stage], kx, b_row);
        } else {
#pragma unroll
          for (int h = 0; h < BN / kBoxRows; ++h)
            tma_load_2d(b_dst + h * kBoxRows * 128, mb0, &full[stage], kx, b_row + h * kBoxRows);
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
    constexpr uint32_t idesc = idesc_bf16_f32(BM, BN);
    int stage = 0, acc = 0;
    uint32_t phase = 0, acc_phase = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
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
        const uint64_t ad = smem_desc_k_sw128(sA + stage * A_BYTES);
        const uint64_t bd = smem_desc_k_sw128(sB + stage * C::B_BYTES);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk)  // advance 16 elements = 32 bytes along K
          tc_mma_bf16(d_tmem, ad + 2 * kk, bd + 2 * kk, idesc, (kb | kk) != 0 ? 1u : 0u);
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
  } else if (warp < kEpiWarps) {
    // ------------------------------------------------------------ epilogue
    // Warp w reads TMEM lanes 32*(w%4).. (tile rows) and half of the output columns
    // (w/4).  Each 32 x 32 chunk is converted in registers, staged in this warp's padded
    // shared-memory slice and written back as 64-byte row segments (4 lanes per row).
    const int quarter = warp & 3, half = warp >> 2;
    constexpr int COLS = C::OUT_COLS / 2;  // output columns of this warp
    uint8_t* stage_mem = sEpi + warp * kEpiStageBytes;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
      const int s = find_seg(s_pre, p.nseg, tile);
      const int rows = s_rows[s];
      const int mt = (rows + BM - 1) / BM;
      const int local = tile - s_pre[s];
      const int n = local / mt, m = local - n * mt;
      int ok = 1;
      if (lane == 0) ok = mbar_wait_bounded(&tfull[acc], acc_phase, abort_flag, p.limit_ns, p.status);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                             static_cast<uint32_t>(acc * BN);
      const int valid = rows - m * BM - quarter * 32;  // rows of this warp's 32 that exist
      __nv_bfloat16* out0 = p.out + static_cast<size_t>(s_row0[s] + m * BM + quarter * 32) * p.ldo +
                            static_cast<size_t>(n) * C::OUT_COLS + half * COLS;
#pragma unroll 1
      for (int c0 = 0; c0 < COLS; c0 += 32) {
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
        // stage: lane = row, 64 bytes
        uint4* srow = reinterpret_cast<uint4*>(stage_mem + lane * kStageRowBytes);
#pragma unroll
        for (int q = 0; q < 4; ++q) srow[q] = make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
        __syncwarp();
        // write back: 4 lanes per row, 8 rows per instruction, 64 contiguous bytes per row
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
      if (lane == 0) mbar_arrive(&tempty[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

__global__ void debug_wait_kernel(int32_t* status, int64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // Nothing ever arrives on `bar`: the bounded wait must run out and report it.
  if (threadIdx.x == 0) mbar_wait_bounded(&bar, 0, &abort_flag, limit_ns, status);
}

// ---------------------------------------------------------------- host side

// Row-major bf16 matrix [rows, cols] read in boxes of 64 columns x 128 rows, 128-byte
// swizzle; rows outside the matrix read as zero.
bool encode_2d(CUtensorMap* m, const void* ptr, uint64_t cols, uint64_t rows) {
  return encode_2d_box(m, ptr, cols, rows, kBoxRows);
}

template <int MODE, int BN>
cudaError_t launch_gemm(const Maps& maps, const Params& p, long long tiles_bound, cudaStream_t s) {
  using C = Cfg<MODE, BN>;
  static DeviceOnce once;
  cudaError_t e = once.run([] {
    cudaError_t r = cudaFuncSetAttribute(grouped_gemm_kernel<MODE, BN>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (r != cudaSuccess) return r;
    return prefer_max_shared(grouped_gemm_kernel<MODE, BN>);
  });
  if (e != cudaSuccess) return e;
  const int grid = static_cast<int>(tiles_bound < sm_count() ? (tiles_bound > 0 ? tiles_bound : 1)
                                                             : sm_count());
  return launch_pdl(grouped_gemm_kernel<MODE, BN>, dim3(grid), dim3(kThreads), C::SMEM, s, maps, p);
}

}  // namespace

// SMs of the current device (a cheap host query, made per launch so that every device
// gets its own count).
int sm_count() {
  int dev = 0, v = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
    return 148;
  return v;
}

// Automatic tile shape: row tiles, or row tiles over SM pairs when the routed experts'
// segments are large.  Column tiles cut the padding of small expert segments (a 130-row
// segment costs 256 rows of row-tile MMA work but 144 token columns), but their N <= 128
// MMAs read about a third more shared memory per FLOP than the row tiles' N = 256 ones, and
// on B200 that costs more than the padding saves on every workload measured here.  They
// stay selectable, and they carry the fused gather and combine.  Row tiles over SM pairs
// stage 32 KB per SM and k-block instead of 48 KB (six k-blocks in flight instead of four):
// faster where segments fill several 256-row pair tiles (Mixtral-shaped prefill, ~2048 rows
// per expert: 4.30 -> 4.13 ms; Switch-shaped layers, ~1024: 4-5%), slower where half of a
// pair tile would be padding (the 64+1 layer at T = 4096, ~128 rows: +16%; decode: +13%;
// the Granite-shaped layer, ~353 rows: +6%).
bool row_pairs_fit(const moe_config& c) { return c.d % 256 == 0 && c.d_ff % 128 == 0; }
constexpr int64_t kPairRows = 512;  // average segment rows from which pairs pay

int32_t ffn_tile_shape(const moe_config& c) {
  if (c.fuse != 0) return MOE_TILES_COLUMNS;  // the fused steps live in the column kernel
  if (c.tiles == MOE_TILES_COLUMNS) return MOE_TILES_COLUMNS;
  if (c.tiles == MOE_TILES_PAIRS && c.d % 256 == 0 && c.d_ff % 256 == 0) return MOE_TILES_PAIRS;
  if (c.tiles == MOE_TILES_ROW_PAIRS && row_pairs_fit(c)) return MOE_TILES_ROW_PAIRS;
  if (c.tiles == MOE_TILES_AUTO && row_pairs_fit(c)) {
    // average rows of a routed expert's segment
    int64_t rows = static_cast<int64_t>(c.T) * c.k / c.E;
    if (c.capacity >= 0)
      rows = (c.layout == MOE_LAYOUT_PADDED) ? c.capacity : std::min<int64_t>(rows, c.capacity);
    if (rows >= kPairRows) return MOE_TILES_ROW_PAIRS;
  }
  return MOE_TILES_ROWS;
}

// With the automatic choice on row tiles, a shared expert of at least kPairRows rows (its
// segment is all T tokens) still runs on row tiles over SM pairs, in launches of its own
// before the routed segments' row tiles (the 64+1 layer at T = 4096: 14.38 -> 13.58 ms per
// layer on average over three alternating runs; at phi = 1 with reroute -2.4%).
bool ffn_shared_on_pairs(const moe_config& c) {
  return c.dtype == MOE_BF16 && c.has_shared && c.T >= kPairRows && c.tiles == MOE_TILES_AUTO &&
         c.fuse == 0 && row_pairs_fit(c) && ffn_tile_shape(c) == MOE_TILES_ROWS;
}

int ffn_launches(const moe_config& c) { return ffn_shared_on_pairs(c) ? 4 : 2; }

cudaError_t launch_ffn_sm100(const moe_config& c, const FfnArgs& f, cudaStream_t s,
                             cudaEvent_t mid) {
  const int32_t shape = ffn_tile_shape(c);
  if (shape == MOE_TILES_COLUMNS) return launch_ffn_cols_sm100(c, f, s, mid);
  if (shape == MOE_TILES_PAIRS) return launch_ffn_pair_sm100(c, f, s, mid);
  if (shape == MOE_TILES_ROW_PAIRS) return launch_ffn_rowpair_sm100(c, f, s, mid);
  const int nseg = c.E + (c.has_shared ? 1 : 0);
  const long long rows_h = f.rmax + (c.has_shared ? c.T : 0);
  const bool split = ffn_shared_on_pairs(c);  // the shared segment on row tiles over SM pairs
  const long long mt_bound = ((split ? f.rmax : rows_h) + BM - 1) / BM + nseg;

  // gate/up + SwiGLU:  A = packed rows [rmax, d] (x [T, d] for the shared expert)
  Maps m1;
  bool ok = encode_2d(&m1.a_routed, f.x_packed, c.d, f.rmax) &&
            encode_2d(&m1.b0_routed, f.w_gate, c.d, static_cast<uint64_t>(c.E) * c.d_ff) &&
            encode_2d(&m1.b1_routed, f.w_up, c.d, static_cast<uint64_t>(c.E) * c.d_ff);
  if (c.has_shared)
    ok = ok && encode_2d(&m1.a_shared, f.x, c.d, c.T) && encode_2d(&m1.b0_shared, f.s_gate, c.d, c.d_ff) &&
         encode_2d(&m1.b1_shared, f.s_up, c.d, c.d_ff);
  else
    m1.a_shared = m1.a_routed, m1.b0_shared = m1.b0_routed, m1.b1_shared = m1.b1_routed;
  if (!ok) return cudaErrorInvalidValue;
  Params p1{f.offsets, f.counts, nseg, c.E, c.d, c.d_ff, static_cast<__nv_bfloat16*>(f.h), c.d_ff,
            f.status, kWaitLimitNs, 1, split ? 0 : 1};
  cudaError_t e;
  if (split && (e = launch_rowpair_gate_up(c, f, s, false, true)) != cudaSuccess) return e;
  e = launch_gemm<0, 256>(m1, p1, mt_bound * (c.d_ff / 128), s);
  if (e != cudaSuccess) return e;
  if (mid != nullptr && (e = record_event(mid, s)) != cudaSuccess) return e;

  // down:  A = H [rows_h, F]
  Maps m2;
  ok = encode_2d(&m2.a_routed, f.h, c.d_ff, rows_h) &&
       encode_2d(&m2.b0_routed, f.w_down, c.d_ff, static_cast<uint64_t>(c.E) * c.d);
  if (c.has_shared)
    ok = ok && encode_2d(&m2.b0_shared, f.s_down, c.d_ff, c.d);
  else
    m2.b0_shared = m2.b0_routed;
  m2.a_shared = m2.a_routed;
  m2.b1_routed = m2.b0_routed;
  m2.b1_shared = m2.b0_shared;
  if (!ok) return cudaErrorInvalidValue;
  Params p2{f.offsets, f.counts, nseg, c.E, c.d_ff, c.d, static_cast<__nv_bfloat16*>(f.y_packed),
            c.d, f.status, kWaitLimitNs, 1, split ? 0 : 1};
  if (split && (e = launch_rowpair_down(c, f, s, false, true)) != cudaSuccess) return e;
  if (c.d % 256 == 0) return launch_gemm<1, 256>(m2, p2, mt_bound * (c.d / 256), s);
  return launch_gemm<1, 128>(m2, p2, mt_bound * (c.d / 128), s);
}

cudaError_t launch_debug_wait(int32_t* status, int64_t limit_ns, cudaStream_t s) {
  debug_wait_kernel<<<1, 32, 0, s>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace moe

// Pieces shared by the two tcgen05 grouped-GEMM kernels (gemm_sm100.cu: tokens on the
// MMA's M side; gemm_cols_sm100.cu: weights on M, tokens on N).
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"

namespace moe {

// Tensor map of a row-major bf16 matrix [rows, cols] read in boxes of 64 columns x
// box_rows rows with 128-byte swizzle; rows outside the matrix read as zero.
bool encode_2d_box(CUtensorMap* m, const void* ptr, uint64_t cols, uint64_t rows,
                   uint32_t box_rows);

// SMs of the current device.
int sm_count();

namespace gemm {

constexpr int BK = 64;        // 64 bf16 = one 128-byte swizzle row
constexpr int kMaxSeg = 260;  // routed experts (<= 256) + the shared expert + slack

// Largest s with pre[s] <= tile (pre: exclusive prefix of tiles per segment).
__device__ __forceinline__ int find_seg(const int* pre, int nseg, int tile) {
  int lo = 0, hi = nseg - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (pre[mid] <= tile) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// SiLU(g) = g / (1 + e^-g) with the fast approximate exponential and division (about 2 ulp
// in fp32; the result is rounded to bf16).  For g -> -inf the denominator overflows and the
// quotient is 0, the limit of SiLU.
__device__ __forceinline__ float silu_f(float g) { return __fdividef(g, 1.f + __expf(-g)); }

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Segment table in shared memory, built by one warp: row starts s_row0[0..nseg], row
// counts s_rows[0..nseg) (from `counts` for routed segments when given, else the gap to
// the next start) and the exclusive prefix s_pre[0..nseg] of the tiles of each segment,
// tiles = ceil(rows / rows_per_tile) * blocks_per_row_tile, or 0 for the segments a launch
// leaves to another one (the routed segments s < E unless `routed`, the shared expert's
// segment unless `shared`).
__device__ __forceinline__ void build_segment_table(const int32_t* offsets, const int32_t* counts,
                                                    int nseg, int E, int rows_per_tile,
                                                    int blocks, int* s_pre, int* s_row0,
                                                    int* s_rows, bool routed = true,
                                                    bool shared = true) {
  const int lane = threadIdx.x & 31;
  for (int i = lane; i <= nseg; i += 32) s_row0[i] = __ldg(offsets + i);
  __syncwarp();
  for (int i = lane; i < nseg; i += 32)
    s_rows[i] = (counts != nullptr && i < E) ? __ldg(counts + i) : s_row0[i + 1] - s_row0[i];
  __syncwarp();
  int carry = 0;
  for (int b = 0; b < nseg; b += 32) {
    const int s = b + lane;
    int t = 0;
    if (s < nseg && (s < E ? routed : shared))
      t = ((s_rows[s] + rows_per_tile - 1) / rows_per_tile) * blocks;
    int incl = t;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (s < nseg) s_pre[s] = carry + incl - t;
    carry += __shfl_sync(0xffffffffu, incl, 31);
  }
  if (lane == 0) s_pre[nseg] = carry;
}

}  // namespace gemm
}  // namespace moe

// The step between the per-tile expert histogram and the pack: exclusive prefixes over the
// token tiles, per-expert demand, the capacity cut and the segment table.  It needs every
// tile's counts, so it runs in the CTA that finishes last among the CTAs that write the
// histogram (a ticket counter): no extra launch and no grid-wide wait.
//
// Source: "271,104 Routes: What I Missed About Mixture-of-Experts", section 3 Dispatch (bincount
// + cumsum give each expert's segment) and its capacity subsection; "Mixture-of-Experts:
// routing and capacity", Capacity and Worked case (kept = min(demand, C) in arrival order).
#pragma once

#include "common.cuh"
#include "internal.h"

namespace moe {

// Called by every thread of each CTA that wrote one tile's row of p.tile_hist, after the
// writes.  `scratch` is shared memory of at least kPrepScratchInts ints that the CTA no
// longer needs (the function declares no shared memory of its own, so a kernel that opts
// into the whole dynamic shared-memory budget can still call it).  The CTA that arrives
// last replaces the histogram by per-tile exclusive prefixes (tile_hist[i][e] = routes to e
// in tiles < i), writes demand, the segment table and the filled-slot counts, and resets the
// ticket.  Returns after that CTA's work (others return at once).
constexpr int kPrepScratchInts = 3 * 257 + 1;

__device__ __forceinline__ void dispatch_prep_arrive(const DispatchPrep& p, int* scratch) {
  volatile int* s_last = scratch + 3 * 257;
  __syncthreads();  // every thread's histogram stores are issued; scratch is free
  if (threadIdx.x == 0) {
    __threadfence();  // this CTA's row is visible before its ticket
    *s_last = (atomicAdd(p.ticket, 1u) == static_cast<unsigned>(p.num_tiles - 1)) ? 1 : 0;
  }
  __syncthreads();
  if (!*s_last) return;
  __threadfence();  // every other CTA's row is visible to the reads below

  const int E = p.E, nt = p.num_tiles;
  const int nth = static_cast<int>(blockDim.x), tid = static_cast<int>(threadIdx.x);
  int* s_part = scratch;            // [parts][E] partial sums, then their exclusive prefix
  int* s_tot = scratch + 257;       // [E] demand
  int* s_off = scratch + 2 * 257;   // [E + 1] segment starts
  // (expert, part) pairs: each part is a contiguous range of tiles; with more experts than
  // threads (E > blockDim) a thread takes several experts with one part each.
  const int parts = nth / E >= 1 ? nth / E : 1;
  const int chunk = (nt + parts - 1) / parts;
  // 1. each pair sums its range of tiles (loads bypass L1: the rows were written by other
  //    SMs during this kernel); a thread with a single pair of up to kKeep tiles keeps the
  //    counts for step 3 instead of loading them again
  constexpr int kKeep = 8;
  const bool keep = parts * E <= nth && chunk <= kKeep;
  int counts[kKeep];
  for (int w = tid; w < parts * E; w += nth) {
    const int e = w % E, part = w / E;
    const int i0 = part * chunk, i1 = min(nt, i0 + chunk);
    int sum = 0;
    if (keep) {
#pragma unroll
      for (int q = 0; q < kKeep; ++q)
        counts[q] = (i0 + q < i1) ? __ldcg(p.tile_hist + static_cast<size_t>(i0 + q) * E + e) : 0;
#pragma unroll
      for (int q = 0; q < kKeep; ++q) sum += counts[q];
    } else {
      for (int i = i0; i < i1; ++i) sum += __ldcg(p.tile_hist + static_cast<size_t>(i) * E + e);
    }
    s_part[part * E + e] = sum;
  }
  __syncthreads();
  // 2. prefix over the parts, per expert
  for (int x = tid; x < E; x += nth) {
    int run = 0;
    for (int q = 0; q < parts; ++q) {
      const int v = s_part[q * E + x];
      s_part[q * E + x] = run;
      run += v;
    }
    s_tot[x] = run;
  }
  __syncthreads();
  // 3. rewrite the histogram as exclusive prefixes (each pair its own range, in order)
  for (int w = tid; w < parts * E; w += nth) {
    const int e = w % E, part = w / E;
    const int i0 = part * chunk, i1 = min(nt, i0 + chunk);
    int pre = s_part[part * E + e];
    if (keep) {
#pragma unroll
      for (int q = 0; q < kKeep; ++q)
        if (i0 + q < i1) {
          p.tile_hist[static_cast<size_t>(i0 + q) * E + e] = pre;
          pre += counts[q];
        }
    } else {
      for (int i = i0; i < i1; ++i) {
        int* q = p.tile_hist + static_cast<size_t>(i) * E + e;
        const int h = __ldcg(q);
        *q = pre;
        pre += h;
      }
    }
  }
  // 4. kept counts -> segment starts (warp 0); the padded buffer gives expert e rows e*C ..
  if (p.padded) {
    for (int x = tid; x <= E; x += nth) s_off[x] = x * p.capacity;
  } else if (tid < 32) {
    const int lane = tid;
    int carry = 0;
    for (int b = 0; b < E; b += 32) {
      const int x = b + lane;
      int kept = 0;
      if (x < E) kept = (p.capacity < 0) ? s_tot[x] : min(s_tot[x], p.capacity);
      int incl = kept;
#pragma unroll
      for (int s = 1; s < 32; s <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, s);
        if (lane >= s) incl += o;
      }
      if (x < E) s_off[x] = carry + incl - kept;
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) s_off[E] = carry;
  }
  __syncthreads();
  for (int x = tid; x <= E; x += nth) p.offsets[x] = s_off[x];
  if (tid == 0) p.offsets[E + 1] = s_off[E] + (p.has_shared ? p.T : 0);
  for (int x = tid; x < E; x += nth) {
    p.demand[x] = s_tot[x];
    if (p.padded) p.offsets[E + 2 + x] = min(s_tot[x], p.capacity);  // filled slots
  }
  if (tid == 0) *p.ticket = 0u;  // ready for the next call
}

}  // namespace moe

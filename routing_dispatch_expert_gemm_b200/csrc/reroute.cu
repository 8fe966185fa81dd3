// Reroute overflow policy on the padded dispatch buffer [E, C, d].
//
// Sources: "Mixture-of-Experts: routing and capacity", Capacity (the buffer has C slots
// per expert; empty slots are padding) and Overflow policies (reroute: the overflowing
// route is handled by the next-best expert by score, the router's decision overridden).
//
// Runs after the arrival-order pack, which has already placed every route that fit and
// left route_row = -1 on the ones that overflowed.  The reroute is sequential by definition
// (whether a route finds a free slot depends on every earlier reroute), but because every
// expert ranks routes by arrival order the result can be built in phases (see
// reroute_phase_kernel), one CTA, at most E + 1 phases.  A grid-wide kernel before it ranks
// each overflowing token's experts once; one after it copies each moved route's token row
// and re-evaluates that token's gates by the gate mode over its final experts.
#include <climits>

#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kThreads = 256;  // copy kernel
constexpr int kWarps = kThreads / 32;

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, s));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) v += __shfl_xor_sync(0xffffffffu, v, s);
  return v;
}

// Gates of token t over its final experts (warp-wide; lane j < k writes slot j).  Slot j's
// expert is the one whose block holds its row, or its original expert when it was dropped.
__device__ void regate(const int32_t* ids, const float* zkeys, const int32_t* route_row,
                       float* gates, int t, int k, int E, int C, int gate_mode, int lane) {
  const float* zrow = zkeys + static_cast<size_t>(t) * E;
  int e = -1;
  if (lane < k) {
    const int r = route_row[static_cast<size_t>(t) * k + lane];
    e = (r >= 0) ? r / C : ids[static_cast<size_t>(t) * k + lane];
  }
  const bool valid = e >= 0 && e < E;
  const float zf = valid ? zrow[e] : -INFINITY;
  float g;
  if (gate_mode != MOE_GATE_SOFTMAX_TOPK) {
    // softmax over the final experts' logits.  For the renormalised mode this is
    // p_i / sum_j p_j with the full softmax's normaliser cancelled; shifting by the
    // final experts' own max keeps it finite when the token no longer holds its top
    // expert and every selected p would underflow.
    const float m = warp_max(zf);
    const float ex = valid ? expf(zf - m) : 0.f;
    g = ex / warp_sum(ex);
  } else {  // the full-softmax probability of each final expert
    float m = -INFINITY;
    for (int q = lane; q < E; q += 32) m = fmaxf(m, zrow[q]);
    m = warp_max(m);
    float den = 0.f;
    for (int q = lane; q < E; q += 32) den += expf(zrow[q] - m);
    den = warp_sum(den);
    g = valid ? expf(zf - m) / den : 0.f;
  }
  if (lane < k) gates[static_cast<size_t>(t) * k + lane] = g;
}

// ---------------------------------------------------------------------------------
// Phased placement.  Every expert ranks the overflowed routes by arrival order, so the
// sequential walk is reproduced exactly in phases: each pending route proposes the expert
// it would take if the experts full at the phase start were the only full ones (its
// token's best-ranked expert that it does not hold and that is not full, or the next-best
// one after the token's earlier routes of the same phase); a scan in arrival order counts
// each expert's proposals and finds the first route whose expert has run out of slots.
// Every route before it is placed exactly as the walk would place it.  The phase then
// restarts at that route with at least one more expert full, so there are at most E + 1
// phases.  A route proposes again only once its expert is full or an earlier route of its
// token proposed again.
//
// reroute_first_kernel ranks, for every token with an overflowed route, the experts it does
// not hold (one warp per token), and makes the first proposals; reroute_phase_kernel runs
// the phases on one CTA, with the pending routes in shared memory when they fit, so that a
// proposal is a walk along the token's ranking that skips full experts and the token's
// placed routes.
// ---------------------------------------------------------------------------------
constexpr int kPhThreads = 256;
constexpr int kPhWarps = kPhThreads / 32;
constexpr int kFirstWarps = 8;      // first kernel: one warp per token
constexpr int kSmemRoutes = 20480;  // pending-route arrays in shared memory up to T k routes
constexpr int kNoRoute = -2;        // first-proposal value of a route that did not overflow

// A proposal with the position in the token's ranking that the next walk starts from
// (expert 0xffff: none; the position is then the ranking's length).
__host__ __device__ constexpr int prop_pack(int expert, int at) {
  return (at << 16) | (expert & 0xffff);
}
__host__ __device__ constexpr int prop_expert(int v) {
  return ((v & 0xffff) == 0xffff) ? -1 : (v & 0xffff);
}
__host__ __device__ constexpr int prop_at(int v) { return v >> 16; }

__host__ __device__ constexpr int pref_stride(int E) { return (E + 15) & ~15; }

// Ascending bitonic sort of 32 NW keys held by a warp, key q of lane l at position 32 q + l.
template <int NW>
__device__ __forceinline__ void warp_bitonic_sort(uint64_t (&v)[NW], int lane) {
  constexpr int N = 32 * NW;
#pragma unroll
  for (int size = 2; size <= N; size <<= 1) {
#pragma unroll
    for (int j = size >> 1; j > 0; j >>= 1) {
      if (j >= 32) {  // partner in another register of the same lane
#pragma unroll
        for (int q = 0; q < NW; ++q) {
          const int p = q ^ (j >> 5);
          if (p > q) {
            const bool asc = ((32 * q + lane) & size) == 0;
            const uint64_t x = v[q], y = v[p];
            if ((x > y) == asc) { v[q] = y; v[p] = x; }
          }
        }
      } else {  // partner in another lane
#pragma unroll
        for (int q = 0; q < NW; ++q) {
          const uint64_t o = __shfl_xor_sync(0xffffffffu, v[q], j);
          const bool asc = ((32 * q + lane) & size) == 0;
          const bool take_min = ((lane & j) == 0) == asc;
          v[q] = take_min ? (o < v[q] ? o : v[q]) : (o > v[q] ? o : v[q]);
        }
      }
    }
  }
}

struct FirstArgs {
  const int32_t* ids;      // [T, k]
  const float* zkeys;      // [T, E]
  const int32_t* route_row;
  const int32_t* offsets;  // filled-slot counts at offsets[E + 2 + e]
  int32_t* prop;           // [T * k] first proposal (prop_pack), kNoRoute: did not overflow
  uint8_t* pref;           // [T, pref_stride(E)] experts the token does not hold, best first
  int32_t* pref_len;       // [T] entries of the token's list
  int T, k, E, C;
};

// One warp per token with an overflowed route.  It ranks the experts the token does not
// hold (descending key, equal keys to the lower index; NaN keys rank as -inf) with a warp
// bitonic sort, stores that order, and makes the first proposals: with nothing placed yet,
// the token's overflowed routes take, in slot order, the first, second, ... experts of the
// order that are not full after the arrival-order pass.
template <int NW>
__global__ void __launch_bounds__(kFirstWarps * 32) reroute_first_kernel(FirstArgs a) {
  __shared__ uint32_t s_full[8];
  __shared__ uint32_t s_list[kFirstWarps][64];  // 256 expert bytes per warp
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int k = a.k, E = a.E, Ep = pref_stride(E);
  pdl_wait();  // route_row and the counts come from the pack, the keys from the router
  pdl_trigger();
  if (warp < NW) {
    const int e = warp * 32 + lane;
    const bool full = e >= E || a.offsets[E + 2 + e] >= a.C;
    const uint32_t b = __ballot_sync(0xffffffffu, full);
    if (lane == 0) s_full[warp] = b;
  }
  __syncthreads();
  uint8_t* lst = reinterpret_cast<uint8_t*>(s_list[warp]);
  for (int t = blockIdx.x * kFirstWarps + warp; t < a.T; t += gridDim.x * kFirstWarps) {
    const int32_t* row = a.ids + static_cast<size_t>(t) * k;
    int id = -1;
    bool ovf = false;
    if (lane < k) {
      id = row[lane];
      ovf = a.route_row[static_cast<size_t>(t) * k + lane] < 0 && route_id_valid(row, lane, id, E);
    }
    const uint32_t ovm = __ballot_sync(0xffffffffu, ovf);
    if (ovm == 0) {
      if (lane < k) a.prop[static_cast<size_t>(t) * k + lane] = kNoRoute;
      continue;
    }
    uint32_t held[NW];
    int nheld = 0;
#pragma unroll
    for (int w = 0; w < NW; ++w) {
      const bool mine = lane < k && id >= 0 && id < E && (id >> 5) == w;
      held[w] = __reduce_or_sync(0xffffffffu, mine ? 1u << (id & 31) : 0u);
      nheld += __popc(held[w]);
    }
    // sort keys: the key's order flipped (larger keys first; -0 as +0, NaN as -inf) above the
    // expert index (equal keys: lower index first); held experts and e >= E sort last
    const float* zrow = a.zkeys + static_cast<size_t>(t) * E;
    uint64_t key[NW];
#pragma unroll
    for (int q = 0; q < NW; ++q) {
      const int e = lane + 32 * q;
      key[q] = ~0ull;
      if (e < E && !((held[q] >> lane) & 1u)) {
        float v = zrow[e];
        v = (v != v) ? -INFINITY : (v == 0.f ? 0.f : v);
        const uint32_t u = __float_as_uint(v);
        const uint32_t ordered = (u & 0x80000000u) ? ~u : (u | 0x80000000u);  // ascending in v
        key[q] = (static_cast<uint64_t>(~ordered) << 32) | static_cast<uint32_t>(e);
      }
    }
    warp_bitonic_sort<NW>(key, lane);
#pragma unroll
    for (int q = 0; q < NW; ++q)  // position 32 q + lane of the ranking
      lst[32 * q + lane] = static_cast<uint8_t>(key[q] & 0xffu);
    __syncwarp();
    const int len = E - nheld;
    uint32_t* dst = reinterpret_cast<uint32_t*>(a.pref + static_cast<size_t>(t) * Ep);
    for (int w4 = lane; w4 < Ep / 4; w4 += 32) dst[w4] = s_list[warp][w4];
    if (lane == 0) a.pref_len[t] = len;
    // the o-th overflowed route takes the o-th entry whose expert is not full
    const int ord = ovf ? __popc(ovm & ((1u << lane) - 1u)) : -1;
    const int last = __popc(ovm) - 1;
    int pick = prop_pack(-1, len), before = 0;
    for (int p0 = 0; p0 < len && before <= last; p0 += 32) {
      const int p = p0 + lane;
      const int e = (p < len) ? lst[p] : 0;
      const bool free_slot = p < len && !((s_full[e >> 5] >> (e & 31)) & 1u);
      uint32_t b = __ballot_sync(0xffffffffu, free_slot);
      const int nb = __popc(b);
      if (ord >= before && ord < before + nb) {
        for (int r = 0; r < ord - before; ++r) b &= b - 1u;
        const int at = p0 + __ffs(b) - 1;
        pick = prop_pack(lst[at], at);
      }
      before += nb;
    }
    if (lane < k) a.prop[static_cast<size_t>(t) * k + lane] = ovf ? pick : kNoRoute;
    __syncwarp();
  }
}

struct PhaseArgs {
  const float* zkeys;      // [T, E]
  const int32_t* prop;     // [T * k] first proposals
  const uint8_t* pref;     // [T, pref_stride(E)]
  const int32_t* pref_len; // [T]
  int32_t* row_token;      // [E * C]
  int32_t* route_row;      // [T, k]
  int32_t* offsets;        // filled-slot counts at offsets[E + 2 + e]
  int32_t* list;           // [0]: n overflowed routes, then (token, row) each; token -1: dropped
  int32_t* g_r;            // [T * k] pending-route arrays when they are not in shared memory
  int32_t* g_c;
  uint8_t* g_dirty;
  uint8_t* g_at;
  int T, k, E, C;
  int in_smem;             // 1: the pending-route arrays live in dynamic shared memory
};

// The first chunks of a token's ranking, requested together.
template <int NW>
struct Ranking {
  static constexpr int kChunks = (NW * 2 < 4) ? NW * 2 : 4;  // <= the row's pref_stride(E) / 16
  uint4 ck[kChunks];
  int len;
};

template <int NW>
__device__ __forceinline__ void load_ranking(const PhaseArgs& a, int t, Ranking<NW>& r) {
  const uint4* row =
      reinterpret_cast<const uint4*>(a.pref + static_cast<size_t>(t) * pref_stride(a.E));
  r.len = a.pref_len[t];
#pragma unroll
  for (int c = 0; c < Ranking<NW>::kChunks; ++c)
    r.ck[c] = (c * 16 < a.E) ? row[c] : make_uint4(0, 0, 0, 0);
}

// Route i proposes again, with the experts in s_full full and routes before `pos` placed:
// the (m+1)-th entry of its token's ranking that is neither full nor taken by one of the
// token's placed routes, m being the token's earlier routes still pending.  Pending routes
// are stored as token << 5 | slot.  With m = 0 the walk resumes at the route's last
// position `at`: every entry before it was full, or taken by the token's placed or earlier
// routes, and stays so.  The excluded experts are one 64-bit register for E <= 64, else the
// calling thread's column of words in shared memory (word w at ex[w * kPhThreads]).
// Returns the expert (-1: none) and updates `at`.
template <int NW>
__device__ __forceinline__ int propose(const PhaseArgs& a, const int* ag_r, const int* ag_c, int i,
                                       int pos, const uint32_t* s_full, uint32_t* ex, int& at) {
  const int t = ag_r[i] >> 5;
  Ranking<NW> rk;
  load_ranking(a, t, rk);
  uint64_t ex64 = 0;
  if constexpr (NW <= 2) {
    ex64 = s_full[0] | (static_cast<uint64_t>(NW == 2 ? s_full[1] : 0xffffffffu) << 32);
  } else {
#pragma unroll
    for (int w = 0; w < NW; ++w) ex[w * kPhThreads] = s_full[w];
  }
  int m = 0;
  for (int q = i - 1; q >= 0 && (ag_r[q] >> 5) == t; --q) {
    if (q >= pos) {
      ++m;
    } else {
      const int cq = ag_c[q];
      if (cq >= 0) {
        if constexpr (NW <= 2) ex64 |= 1ull << cq;
        else ex[(cq >> 5) * kPhThreads] |= 1u << (cq & 31);
      }
    }
  }
  const int len = rk.len;
  const int start = (m == 0) ? at : 0;
  for (int p0 = start & ~15; p0 < len; p0 += 16) {
    const int c = p0 >> 4;
    uint4 cur = rk.ck[0];
    bool have = false;
#pragma unroll
    for (int cc = 0; cc < Ranking<NW>::kChunks; ++cc)
      if (c == cc) { cur = rk.ck[cc]; have = true; }
    if (!have)
      cur = reinterpret_cast<const uint4*>(a.pref + static_cast<size_t>(t) * pref_stride(a.E))[c];
    const uint32_t w4[4] = {cur.x, cur.y, cur.z, cur.w};
    // all sixteen tests at once (entries outside [start, len) are masked off afterwards; the
    // index is clamped so that their bytes stay inside the excluded set's words)
    uint32_t avail = 0;
#pragma unroll
    for (int b = 0; b < 16; ++b) {
      const int e = ((w4[b >> 2] >> (8 * (b & 3))) & 0xff) & (32 * NW - 1);
      uint32_t bit;
      if constexpr (NW <= 2) bit = static_cast<uint32_t>(~ex64 >> e) & 1u;
      else bit = (~ex[(e >> 5) * kPhThreads] >> (e & 31)) & 1u;
      avail |= bit << b;
    }
    if (len - p0 < 16) avail &= (1u << (len - p0)) - 1u;
    if (start > p0) avail &= ~0u << (start - p0);
    const int na = __popc(avail);
    if (m < na) {
      for (int r = 0; r < m; ++r) avail &= avail - 1u;
      const int b = __ffs(avail) - 1;
      const uint32_t w = (b < 4) ? cur.x : (b < 8) ? cur.y : (b < 12) ? cur.z : cur.w;
      at = p0 + b;
      return (w >> (8 * (b & 3))) & 0xff;
    }
    m -= na;
  }
  at = len;
  return -1;
}

// The ranking of a pending route's token into this SM's L1, ahead of a proposal.
__device__ __forceinline__ void prefetch_ranking(const PhaseArgs& a, int t) {
  const uint8_t* row = a.pref + static_cast<size_t>(t) * pref_stride(a.E);
  for (int off = 0; off < pref_stride(a.E); off += 128)
    asm volatile("prefetch.global.L1 [%0];" ::"l"(row + off));
  asm volatile("prefetch.global.L1 [%0];" ::"l"(a.pref_len + t));
}

__device__ __forceinline__ int warp_incl_scan(int v, int lane) {
#pragma unroll
  for (int s = 1; s < 32; s <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, v, s);
    if (lane >= s) v += o;
  }
  return v;
}

template <int NW, bool SMEM>
__global__ void __launch_bounds__(kPhThreads, 1) reroute_phase_kernel(PhaseArgs a) {
  extern __shared__ int s_dyn[];
  __shared__ int s_wc[kPhWarps][257];  // per-warp proposal counts per expert in the block
  __shared__ int s_cnt[2][256];         // filled slots: this phase's, and the next phase's
  __shared__ uint32_t s_full[2][8];     // full experts (and e >= E), likewise
  __shared__ int s_carry[256];          // proposals per expert in the phase's earlier blocks
  __shared__ int s_wtot[2][kPhWarps];
  __shared__ int s_istar[2];
  __shared__ uint32_t s_ex[NW * kPhThreads];  // per-thread excluded-expert words (propose)
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t lt = (1u << lane) - 1u;
  const int E = a.E, k = a.k, C = a.C;
  const int total = a.T * k;  // <= INT_MAX / 2 (validated on the host)
  // pending routes in arrival order: token << 5 | slot, proposed / final expert (-1: none),
  // a flag set when an earlier route of the same token proposed again, and the position in
  // the token's ranking of the last proposal
  int* ag_r = SMEM ? s_dyn : a.g_r;
  int* ag_c = SMEM ? s_dyn + total : a.g_c;
  uint8_t* dirty = SMEM ? reinterpret_cast<uint8_t*>(s_dyn + 2 * total) : a.g_dirty;
  uint8_t* at = SMEM ? reinterpret_cast<uint8_t*>(s_dyn + 2 * total) + total : a.g_at;
  pdl_wait();

  for (int x = tid; x < kPhWarps * 257; x += kPhThreads) (&s_wc[0][0])[x] = 0;
  for (int e = tid; e < 256; e += kPhThreads) {  // a warp covers one 32-expert word
    const int cnt = (e < E) ? a.offsets[E + 2 + e] : C;
    s_cnt[0][e] = cnt;
    const uint32_t b = __ballot_sync(0xffffffffu, e >= E || cnt >= C);
    if (lane == 0) s_full[0][e >> 5] = b;
  }

  // 1. overflowed routes in arrival order, sixteen consecutive routes per thread
  int n = 0;
  for (int base = 0, pass = 0; base < total; base += 16 * kPhThreads, ++pass) {
    const int r0 = base + 16 * tid;
    int v[16];
    if (r0 + 16 <= total) {  // prop is 16-byte aligned
      const int4* p4 = reinterpret_cast<const int4*>(a.prop + r0);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int4 q = p4[u];
        v[4 * u] = q.x; v[4 * u + 1] = q.y; v[4 * u + 2] = q.z; v[4 * u + 3] = q.w;
      }
    } else {
#pragma unroll
      for (int u = 0; u < 16; ++u) v[u] = (r0 + u < total) ? a.prop[r0 + u] : kNoRoute;
    }
    uint32_t bits = 0;
#pragma unroll
    for (int u = 0; u < 16; ++u)
      if (v[u] != kNoRoute) bits |= 1u << u;
    const int cnt = __popc(bits);
    const int incl = warp_incl_scan(cnt, lane);
    if (lane == 31) s_wtot[pass & 1][warp] = incl;
    __syncthreads();
    const int wv = (lane < kPhWarps) ? s_wtot[pass & 1][lane] : 0;
    const int wincl = warp_incl_scan(wv, lane);
    const int wexcl = __shfl_sync(0xffffffffu, wincl - wv, warp);
    const int ptot = __shfl_sync(0xffffffffu, wincl, 31);
    int out = n + wexcl + incl - cnt;
    if (bits != 0) {
      int t = r0 / k, j = r0 - t * k;
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        if ((bits >> u) & 1u) {
          ag_r[out] = (t << 5) | j;
          ag_c[out] = prop_expert(v[u]);
          at[out] = static_cast<uint8_t>(prop_at(v[u]));
          dirty[out] = 0;
          ++out;
        }
        if (++j == k) { j = 0; ++t; }
      }
    }
    n += ptot;
  }
  if (tid == 0) s_istar[0] = n;
  __syncthreads();
  if (tid < n) prefetch_ranking(a, ag_r[tid] >> 5);

  // 2. phases.  Each scan block first brings its routes' proposals up to date: a route
  //    proposes again when its expert is full, when an earlier pending route of its token in
  //    the block does, or when it is marked dirty (a route of its token in an earlier block
  //    proposed again).  Routes past the scanned blocks are brought up to date when a later
  //    phase reaches them: a proposal whose expert is not full stays what it would be.
  //    Placements of a phase go to the next phase's counts and full set, so that one
  //    barrier ends a phase.
  int pos = 0, cur = 0;
  while (pos < n) {
    const int nxt = cur ^ 1;
    int istar = n;
    for (int base = pos; base < n; base += kPhThreads) {
      const int i = base + tid;
      if (base == pos) {  // a phase's first block: start the next phase's state from this one's
        for (int e = tid; e < 256; e += kPhThreads) {
          s_cnt[nxt][e] = s_cnt[cur][e];
          s_carry[e] = 0;
        }
        if (tid < 8) s_full[nxt][tid] = s_full[cur][tid];
        if (tid == 0) s_istar[nxt] = n;
      }
      const uint32_t* full = s_full[cur];
      // (each thread judges its token's earlier routes in the block itself; the new
      // proposals and flags are stored only after the next barrier)
      int c = -1, tr = 0;
      bool again = false;
      if (i < n) {
        c = ag_c[i];
        tr = ag_r[i];
        again = dirty[i] != 0 || (c >= 0 && ((full[c >> 5] >> (c & 31)) & 1u));
        const int t = tr >> 5;
        for (int q = i - 1; !again && q >= base && (ag_r[q] >> 5) == t; --q) {
          const int cq = ag_c[q];
          again = dirty[q] != 0 || (cq >= 0 && ((full[cq >> 5] >> (cq & 31)) & 1u));
        }
      }
      int at_i = 0;
      if (again) {
        at_i = at[i];
        c = propose<NW>(a, ag_r, ag_c, i, pos, full, s_ex + tid, at_i);
      }
      // scan in arrival order; place every route before the first one whose expert has no
      // slot left for it.  A route's rank among the block's proposals to its expert is its
      // rank in its warp plus the earlier warps' counts.
      const uint32_t peers = __match_any_sync(0xffffffffu, c);
      const int wrank = __popc(peers & lt);
      const bool lead = c >= 0 && wrank == 0;
      __syncwarp();  // this warp's counts of the previous block are cleared
      if (lead) s_wc[warp][c] = __popc(peers);
      __syncthreads();
      if (again) {
        ag_c[i] = c;
        at[i] = static_cast<uint8_t>(at_i);
        dirty[i] = 0;
        const int t = tr >> 5;
        for (int q = i + 1; q < n && (ag_r[q] >> 5) == t; ++q)
          if (q >= base + kPhThreads) dirty[q] = 1;
      }
      int rank = 0;
      if (c >= 0) {
        rank = s_carry[c] + wrank;
#pragma unroll
        for (int w = 0; w < kPhWarps; ++w)
          if (w < warp) rank += s_wc[w][c];
      }
      const uint32_t over = __ballot_sync(0xffffffffu, c >= 0 && s_cnt[cur][c] + rank >= C);
      if (over != 0 && lane == __ffs(over) - 1) atomicMin(&s_istar[cur], i);  // warp's first
      __syncthreads();
      istar = s_istar[cur];
      {  // the route this thread handles in the next block: its ranking into L1
        const int nx = ((istar < n) ? istar : base + kPhThreads) + tid;
        if (nx < n) prefetch_ranking(a, ag_r[nx] >> 5);
      }
      if (lead) {
        s_wc[warp][c] = 0;
        if (istar == n) atomicAdd(&s_carry[c], __popc(peers));
      }
      const bool placed = c >= 0 && i < istar;
      const uint32_t grp = peers & __ballot_sync(0xffffffffu, placed);
      if (i < istar && i < n) {  // placed, or dropped for good when no expert is left
        const int t = tr >> 5;
        if (c >= 0) {
          const int slot = s_cnt[cur][c] + rank;
          const int row = c * C + slot;
          a.route_row[static_cast<size_t>(t) * k + (tr & 31)] = row;
          a.row_token[row] = t;
          a.list[1 + 2 * i] = t;
          a.list[2 + 2 * i] = row;
          // the group's last placed lane holds its highest slot
          if ((grp >> lane) == 1u) atomicMax(&s_cnt[nxt][c], slot + 1);
          if (slot + 1 == C) atomicOr(&s_full[nxt][c >> 5], 1u << (c & 31));
        } else {
          a.list[1 + 2 * i] = -1;
        }
      }
      if (istar < n) break;
    }
    __syncthreads();
    cur = nxt;
    pos = istar;
  }
  for (int e = tid; e < E; e += kPhThreads) a.offsets[E + 2 + e] = s_cnt[cur][e];
  if (tid == 0) a.list[0] = n;
  __syncthreads();
  pdl_trigger();
}

constexpr int kRouteSmemBytes = 2 * sizeof(int) + 2;  // ag_r, ag_c, dirty, at

template <int NW>
cudaError_t launch_placement(const FirstArgs& fa, const PhaseArgs& pa, cudaStream_t s) {
  static DeviceOnce once;
  cudaError_t e = once.run([] {
    return cudaFuncSetAttribute(reroute_phase_kernel<NW, true>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize,
                                kSmemRoutes * kRouteSmemBytes);
  });
  if (e != cudaSuccess) return e;
  int grid = (fa.T + kFirstWarps - 1) / kFirstWarps;
  if (grid > 8 * 148) grid = 8 * 148;
  e = launch_pdl(reroute_first_kernel<NW>, dim3(grid), dim3(kFirstWarps * 32), 0, s, fa);
  if (e != cudaSuccess) return e;
  if (pa.in_smem)
    return launch_pdl(reroute_phase_kernel<NW, true>, dim3(1), dim3(kPhThreads),
                      static_cast<size_t>(pa.T) * pa.k * kRouteSmemBytes, s, pa);
  return launch_pdl(reroute_phase_kernel<NW, false>, dim3(1), dim3(kPhThreads), 0, s, pa);
}

// Scratch: the moved-route list (2 T k + 1, padded to 4), first proposals and the pending-
// route arrays (4 T k), the ranking lengths (T), then the rankings (T pref_stride(E) bytes).
size_t list_ints(const moe_config& c) {  // rounded up so that what follows is 16-byte aligned
  return (2 * static_cast<size_t>(c.T) * c.k + 1 + 3) & ~static_cast<size_t>(3);
}
size_t scratch_ints(const moe_config& c) {
  return list_ints(c) + 4 * static_cast<size_t>(c.T) * c.k + static_cast<size_t>(c.T);
}
size_t pref_offset(const moe_config& c) {
  return (scratch_ints(c) * 4 + 15) & ~static_cast<size_t>(15);
}

}  // namespace

size_t reroute_scratch_bytes(const moe_config& c) {
  return pref_offset(c) + static_cast<size_t>(c.T) * pref_stride(c.E);
}

namespace {

struct CopyArgs {
  const void* x;
  void* x_packed;
  const int32_t* list;
  const int32_t* ids;
  const float* zkeys;
  const int32_t* route_row;
  float* gates;
  int d, k, E, C, gate_mode;
};

// One warp per overflowed route that moved: copy x[t] to its new row of the padded buffer
// and re-evaluate token t's gates (a token with two moved routes is evaluated twice, to the
// same values).
template <typename T>
__global__ void __launch_bounds__(kThreads) reroute_copy_kernel(CopyArgs a) {
  constexpr int VEC = Vec<T>::N;
  pdl_trigger();
  pdl_wait();
  const int n = a.list[0];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nvec = a.d / VEC;
  for (int i = blockIdx.x * kWarps + warp; i < n; i += gridDim.x * kWarps) {
    const int t = a.list[1 + 2 * i], row = a.list[2 + 2 * i];
    if (t < 0) continue;  // no expert had a slot left
    const T* src = static_cast<const T*>(a.x) + static_cast<size_t>(t) * a.d;
    T* dst = static_cast<T*>(a.x_packed) + static_cast<size_t>(row) * a.d;
    for (int v = lane; v < nvec; v += 32) st_vec(dst + v * VEC, ld_vec(src + v * VEC));
    regate(a.ids, a.zkeys, a.route_row, a.gates, t, a.k, a.E, a.C, a.gate_mode, lane);
  }
}

}  // namespace

cudaError_t launch_reroute(const moe_config& c, const void* x, const int32_t* ids,
                           const float* zkeys, float* gates, void* x_packed, int32_t* row_token,
                           int32_t* route_row, int32_t* offsets, int32_t* scratch, int32_t* status,
                           cudaStream_t s) {
  (void)status;
  const size_t slots = static_cast<size_t>(c.E) * c.capacity;
  const size_t routes = static_cast<size_t>(c.T) * c.k;
  int32_t* list = scratch;
  int32_t* prop = scratch + list_ints(c);
  int32_t* pref_len = prop + 4 * routes;
  uint8_t* pref = reinterpret_cast<uint8_t*>(scratch) + pref_offset(c);
  const FirstArgs fa{ids,  zkeys,    route_row, offsets, prop,      pref,
                     pref_len, c.T, c.k,       c.E,     c.capacity};
  const PhaseArgs pa{zkeys, prop, pref, pref_len, row_token, route_row, offsets, list,
                     prop + routes, prop + 2 * routes,
                     reinterpret_cast<uint8_t*>(prop + 3 * routes),
                     reinterpret_cast<uint8_t*>(prop + 3 * routes) + routes, c.T, c.k, c.E,
                     c.capacity,
                     routes <= static_cast<size_t>(kSmemRoutes) ? 1 : 0};
  cudaError_t e = c.E <= 32   ? launch_placement<1>(fa, pa, s)
                  : c.E <= 64  ? launch_placement<2>(fa, pa, s)
                  : c.E <= 128 ? launch_placement<4>(fa, pa, s)
                               : launch_placement<8>(fa, pa, s);
  if (e != cudaSuccess) return e;
  int grid = static_cast<int>((slots + kWarps - 1) / kWarps);
  if (grid > 4 * 148) grid = 4 * 148;
  if (grid < 1) grid = 1;
  const CopyArgs ca{x, x_packed, list, ids, zkeys, route_row, gates, c.d, c.k, c.E, c.capacity,
                    c.gate_mode};
  if (c.dtype == MOE_BF16)
    return launch_pdl(reroute_copy_kernel<__nv_bfloat16>, dim3(grid), dim3(kThreads), 0, s, ca);
  return launch_pdl(reroute_copy_kernel<float>, dim3(grid), dim3(kThreads), 0, s, ca);
}

}  // namespace moe

// Routing statistics of one layer call: per-expert dispatch fraction f, mean router
// probability P, the auxiliary load-balancing value, load imbalance, drop and padding
// rates.
//
// Sources: "Mixture of Experts: Routing, Dispatch, and Load Balancing", section 4
// (loss_aux = alpha * N * sum_i f_i P_i: f_i the fraction of tokens dispatched to expert i,
// P_i the mean routing probability); "Mixture-of-experts routing", Load imbalance
// (I = max_e D_e / mean_e D_e); "Mixture-of-Experts: routing and capacity", Worked case
// (routes dropped by capacity and empty slots of the E x C buffer).
//
// Input: the router's per-tile sums of every token's full softmax ([num_tiles, E] fp32,
// 128 tokens per tile) and the dispatch counts.  Each CTA sums a contiguous run of tiles
// per expert in fp64 and writes one row of partials; the CTA that arrives last (a ticket
// counter that it resets to zero) adds the rows in CTA order and evaluates the
// statistics with fixed-order tree reductions, so the result does not depend on which
// CTA finishes when.
#include "common.cuh"
#include "internal.h"

namespace moe {
namespace {

constexpr int kThreads = 256;  // one thread per expert in the final step (E <= 256)
constexpr int kTilesPerBlock = 16;

struct StatsArgs {
  const float* tile_psum;   // [ntiles, E]
  const int32_t* demand;    // [E]
  const int32_t* offsets;   // [E + 2]
  double* partial;          // [gridDim.x, E]
  unsigned int* counter;    // zero on entry; the last CTA puts it back to zero
  float* f;                 // [E] or null
  float* P;                 // [E] or null
  moe_routing_summary* out;
  int T, E, k, C, ntiles, chunk, padded;
  float alpha;
};

__global__ void __launch_bounds__(kThreads) stats_kernel(StatsArgs a) {
  __shared__ double s_fp[kThreads];
  __shared__ long long s_sum[kThreads];
  __shared__ int s_max[kThreads], s_arg[kThreads];
  __shared__ int s_last;
  const int tid = threadIdx.x;
  pdl_trigger();
  pdl_wait();  // demand / offsets / tile sums come from the kernels before this one

  const int t0 = blockIdx.x * a.chunk;
  const int t1 = min(a.ntiles, t0 + a.chunk);
  for (int e = tid; e < a.E; e += kThreads) {
    double acc = 0.0;
    for (int t = t0; t < t1; ++t)
      acc += static_cast<double>(__ldcg(a.tile_psum + static_cast<size_t>(t) * a.E + e));
    a.partial[static_cast<size_t>(blockIdx.x) * a.E + e] = acc;
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(a.counter, 1u) == gridDim.x - 1) ? 1 : 0;
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  // ---- last CTA: thread e owns expert e ----
  const int e = tid;
  double fp = 0.0;
  int dem = -1;
  if (e < a.E) {
    double ps = 0.0;
    for (int b = 0; b < static_cast<int>(gridDim.x); ++b)
      ps += __ldcg(a.partial + static_cast<size_t>(b) * a.E + e);  // L2: written by other CTAs
    dem = __ldcg(a.demand + e);
    const double Pe = ps / static_cast<double>(a.T);
    const double fe = static_cast<double>(dem) / (static_cast<double>(a.T) * a.k);
    fp = fe * Pe;
    if (a.f != nullptr) a.f[e] = static_cast<float>(fe);
    if (a.P != nullptr) a.P[e] = static_cast<float>(Pe);
  }
  s_fp[e] = fp;
  s_sum[e] = dem > 0 ? dem : 0;
  s_max[e] = dem;
  s_arg[e] = e;
  __syncthreads();
  for (int s = kThreads / 2; s > 0; s >>= 1) {
    if (e < s) {
      s_fp[e] += s_fp[e + s];
      s_sum[e] += s_sum[e + s];
      // larger demand wins; on equal demand the lower expert index
      if (s_max[e + s] > s_max[e] || (s_max[e + s] == s_max[e] && s_arg[e + s] < s_arg[e])) {
        s_max[e] = s_max[e + s];
        s_arg[e] = s_arg[e + s];
      }
    }
    __syncthreads();
  }
  if (e == 0) {  // kept routes: the ragged segment end, or the padded buffer's filled slots
    int R = 0;
    if (a.padded)
      for (int q = 0; q < a.E; ++q) R += __ldcg(a.offsets + a.E + 2 + q);
    else
      R = __ldcg(a.offsets + a.E);
    const long long Tk = static_cast<long long>(a.T) * a.k;
    const double mean = static_cast<double>(s_sum[0]) / a.E;
    moe_routing_summary r;
    r.aux_loss = static_cast<float>(static_cast<double>(a.alpha) * a.E * s_fp[0]);
    r.imbalance = mean > 0.0 ? static_cast<float>(s_max[0] / mean) : 0.f;
    r.drop_rate = static_cast<float>(static_cast<double>(Tk - R) / static_cast<double>(Tk));
    const long long slots = static_cast<long long>(a.E) * a.C;
    r.padding_rate = (a.C > 0) ? static_cast<float>(static_cast<double>(slots - R) / slots) : 0.f;
    r.kept = R;
    r.dropped = static_cast<int32_t>(Tk - R);
    r.max_demand = s_max[0];
    r.busiest_expert = s_arg[0];
    *a.out = r;
    *a.counter = 0u;
  }
}

}  // namespace

cudaError_t launch_routing_stats(const moe_config& c, const float* tile_psum,
                                 const int32_t* demand, const int32_t* offsets, float alpha,
                                 double* partial, unsigned int* counter, float* f, float* P,
                                 moe_routing_summary* out, cudaStream_t s) {
  const int ntiles = num_tiles_for(c.T, c.E);
  int nb = (ntiles + kTilesPerBlock - 1) / kTilesPerBlock;
  if (nb > kStatsMaxBlocks) nb = kStatsMaxBlocks;
  if (nb < 1) nb = 1;
  const int chunk = (ntiles + nb - 1) / nb;
  StatsArgs a{tile_psum, demand, offsets, partial, counter, f, P, out,
              c.T, c.E, c.k, c.capacity, ntiles, chunk, c.layout == MOE_LAYOUT_PADDED ? 1 : 0, alpha};
  return launch_pdl(stats_kernel, dim3(nb), dim3(kThreads), 0, s, a);
}

}  // namespace moe

// Per-expert statistics over token chunks, in one launch:
//   count[e]          = sum over chunks of the chunk's selections of e (before capacity)
//   prob_sum[e]       = sum over chunks of the chunk's probability mass on e, fixed order
//   chunk_base[c][e]  = exclusive scan over chunks of the selections of e (token order)
//   kept[e]           = min(count_e, C) (dropless: count_e)
// One block per expert, no atomics. The scan over experts (offsets) and the load-balancing loss
// (Quartz: weight 0.01) are formed by the scatter kernel that follows, which needs the offsets
// anyway (permute.cuh). Chunks are RT_TM tokens, the router's CTA, so the router's per-CTA
// counts are the permutation's histogram (Moonfrost expert card: routing under a per-expert
// capacity over stacked experts). Every sum has a fixed order.
#pragma once
#include "common.cuh"

namespace moe {

constexpr int ST_THREADS = 256;

struct StatsArgs {
  const int32_t *chunk_cnt;  // [nchunk][E]
  const float *chunk_prob;   // [nchunk][E] or null
  int nchunk, E, C;          // C < 0: dropless
  int32_t *count_out;        // [E] or null
  float *prob_out;           // [E] or null (needs chunk_prob)
  int32_t *chunk_base;       // [nchunk][E] or null
  int32_t *kept;             // [E] or null
};

__global__ void __launch_bounds__(ST_THREADS) moe_stats_kernel(StatsArgs a) {
  const KernelStamp stamp(K_STATS);
  griddep_wait();
  stamp.started();
  griddep_launch();
  const int e = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int E = a.E;
  __shared__ int s_wc[ST_THREADS / 32 + 1];
  __shared__ float s_wp[ST_THREADS / 32];
  // One pass over the chunks, ST_THREADS at a time: the exclusive scan in chunk order gives
  // chunk_base and the count total; thread t adds the probability sums of chunks t, t+256, ...
  int run = 0;
  float p = 0.0f;
  for (int b0 = 0; b0 < a.nchunk; b0 += ST_THREADS) {
    const int b = b0 + tid;
    const int v = b < a.nchunk ? a.chunk_cnt[(size_t)b * E + e] : 0;
    if (a.chunk_prob && b < a.nchunk) p += a.chunk_prob[(size_t)b * E + e];
    const int incl = warp_incl_scan(v);
    if (lane == 31) s_wc[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const int wv = lane < ST_THREADS / 32 ? s_wc[lane] : 0;
      const int wi = warp_incl_scan(wv);
      if (lane < ST_THREADS / 32) s_wc[lane] = wi - wv;
      if (lane == ST_THREADS / 32 - 1) s_wc[ST_THREADS / 32] = wi;
    }
    __syncthreads();
    if (a.chunk_base && b < a.nchunk) a.chunk_base[(size_t)b * E + e] = run + s_wc[warp] + incl - v;
    run += s_wc[ST_THREADS / 32];
    __syncthreads();
  }
  // probability total in a fixed tree: lanes, then warps in order
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) p += __shfl_xor_sync(0xffffffffu, p, o);
  if (lane == 0) s_wp[warp] = p;
  __syncthreads();
  if (tid == 0) {
    float psum = 0.0f;
#pragma unroll
    for (int w = 0; w < ST_THREADS / 32; ++w) psum += s_wp[w];
    if (a.count_out) a.count_out[e] = run;
    if (a.prob_out) a.prob_out[e] = psum;
    if (a.kept) a.kept[e] = a.C < 0 ? run : min(run, a.C);
  }
}

// Loss-free balancing step (dormouse pages: a router bias balances the load in place of the
// auxiliary loss, after arXiv 2408.15664): b_i <- b_i + u * sign(mean - count_i) with
// mean = sum(count) / E. The sign compares sum(count) with E * count_i exactly in int64; u * s is
// exact (s in {-1, 0, 1}), so the fp32 add is the only rounding.
__global__ void __launch_bounds__(256) bias_update_kernel(const int32_t *__restrict__ count,
                                                          float *__restrict__ bias, int E,
                                                          float u) {
  griddep_wait();
  griddep_launch();
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  __shared__ long long s_part[8];
  long long t = 0;
  for (int i = tid; i < E; i += 256) t += count[i];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
  if (lane == 0) s_part[warp] = t;
  __syncthreads();
  long long total = 0;
#pragma unroll
  for (int w = 0; w < 8; ++w) total += s_part[w];
  for (int i = tid; i < E; i += 256) {
    const long long ec = (long long)E * count[i];
    const float sgn = total > ec ? 1.0f : (total < ec ? -1.0f : 0.0f);
    bias[i] = __fadd_rn(bias[i], u * sgn);
  }
}

}  // namespace moe

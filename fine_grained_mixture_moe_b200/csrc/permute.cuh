// Token permutation grouped by expert (Moonfrost expert card: experts as stacked (E, hidden,
// ffn) tensors routed under a per-expert capacity, replacing a per-expert loop that synchronised
// the host once per expert; here nothing returns to the host at all).
//
// Stable counting sort of the (token, slot) pairs by expert, with the capacity mask:
//   rank(t, e) = #{t' < t : e in topk(t')};   kept iff rank < C;   row = offsets[e] + rank.
// Tokens are cut into chunks of 16 (the router's CTA). Steps:
//   hist    per-chunk expert histogram -> chunk_count[chunk][E] (inside the layer call the
//           router's per-CTA counts already are this histogram, so it is only launched by
//           moe_permute on its own)
//   stats   per-expert exclusive scan over chunks -> chunk_base; offsets[E+1] (stats.cuh)
//   scatter per-chunk ranks from a per-expert lane bitmask, slot_pos / src_token, then
//           PM_SPLIT CTAs of eight warps copy the chunk's x rows to x_perm with 16-byte loads
//           and stores.
#pragma once
#include "common.cuh"

namespace moe {

constexpr int PM_CHUNK = 16;
constexpr int PM_SPLIT = 4;  // CTAs per chunk in the scatter

__global__ void __launch_bounds__(256) perm_hist_kernel(const int32_t *__restrict__ idx, int T,
                                                        int k, int E,
                                                        int32_t *__restrict__ chunk_count,
                                                        int nchunks, unsigned *stats_counter) {
  extern __shared__ int sh_cnt[];  // [8][E]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int *c = sh_cnt + warp * E;
  for (int e = lane; e < E; e += 32) c[e] = 0;
  __syncwarp();
  const int chunk = blockIdx.x * 8 + warp;
  if (blockIdx.x == 0 && threadIdx.x == 0) *stats_counter = 0u;  // consumed by moe_stats_kernel
  if (chunk >= nchunks) return;
  const int t = chunk * PM_CHUNK + lane;
  if (lane < PM_CHUNK && t < T) {
    for (int j = 0; j < k; ++j) {
      const int e = idx[(size_t)t * k + j];
      if (e >= 0 && e < E) atomicAdd(&c[e], 1);
      else set_device_error(MOE_ERR_DEVICE_CHECK, 100 + j);
    }
  }
  __syncwarp();
  for (int e = lane; e < E; e += 32) chunk_count[(size_t)chunk * E + e] = c[e];
}

template <typename Tin>
__global__ void __launch_bounds__(256) perm_scatter_kernel(
    const int32_t *__restrict__ idx, int T, int k, int E, int C,
    const int32_t *__restrict__ chunk_base, const int32_t *__restrict__ offsets,
    int32_t *__restrict__ slot_pos, int32_t *__restrict__ src, const Tin *__restrict__ x,
    Tin *__restrict__ x_perm, int d) {
  extern __shared__ unsigned smask[];  // [E]
  __shared__ int s_pos[PM_CHUNK * 8];
  __shared__ int s_tok[PM_CHUNK * 8];
  const bool active = (threadIdx.x & 31) < PM_CHUNK;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunk = blockIdx.x / PM_SPLIT, part = blockIdx.x % PM_SPLIT;
  const int t = chunk * PM_CHUNK + lane;
  if (warp == 0) {
    for (int e = lane; e < E; e += 32) smask[e] = 0u;
    __syncwarp();
    const bool valid = active && t < T;
    int ev[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      ev[j] = -1;
      if (j < k && valid) {
        const int e = idx[(size_t)t * k + j];
        if (e >= 0 && e < E) {
          ev[j] = e;
          atomicOr(&smask[e], 1u << lane);
        }
      }
    }
    __syncwarp();
    const unsigned lt = lanemask_lt();
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (j < k) {
        int pos = -1;
        const int e = ev[j];
        if (e >= 0) {
          const int rank = chunk_base[(size_t)chunk * E + e] + __popc(smask[e] & lt);
          if (C < 0 || rank < C) pos = offsets[e] + rank;
          if (part == 0) {
            slot_pos[(size_t)t * k + j] = pos;
            if (pos >= 0) src[pos] = t;
          }
        }
        if (active) {
          s_pos[lane * k + j] = pos;
          s_tok[lane * k + j] = t;
        }
      }
    }
  }
  __syncthreads();
  if (x_perm == nullptr) return;
  // the chunk's rows are shared by PM_SPLIT CTAs (slots part, part + PM_SPLIT, ...), so more
  // copies are in flight per SM than 16-token chunks alone would give
  const int nvec = d * (int)sizeof(Tin) / 16;
  for (int s = part + PM_SPLIT * warp; s < PM_CHUNK * k; s += PM_SPLIT * 8) {
    const int pos = s_pos[s];
    if (pos < 0) continue;
    const uint4 *srow = (const uint4 *)(x + (size_t)s_tok[s] * d);
    uint4 *drow = (uint4 *)(x_perm + (size_t)pos * d);
#pragma unroll 4
    for (int v = lane; v < nvec; v += 32) drow[v] = __ldg(srow + v);
  }
}

}  // namespace moe

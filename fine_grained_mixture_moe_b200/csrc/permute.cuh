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
//   scatter per-chunk ranks from a per-expert lane bitmask, slot_pos / src_token; PM_SPLIT
//           CTAs per chunk each copy 4 of its x rows to their k destinations in x_perm with
//           16-byte loads and stores (each row read once).
#pragma once
#include "common.cuh"

namespace moe {

constexpr int PM_CHUNK = 16;
constexpr int PM_SPLIT = 4;  // CTAs per chunk in the scatter

__global__ void __launch_bounds__(256) perm_hist_kernel(const int32_t *__restrict__ idx, int T,
                                                        int k, int E,
                                                        int32_t *__restrict__ chunk_count,
                                                        int nchunks, unsigned *stats_counter) {
  griddep_wait();
  griddep_launch();
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

// Scatter. CTA (chunk, part) owns tokens chunk*16 + part*TPC .. +TPC (TPC = 16 / PM_SPLIT): two
// warps per token, one half of the row each. Each warp loads its half-row into registers first
// (these loads do not depend on the routing, so they overlap the index work), warp 0 meanwhile
// ranks the chunk's (token, slot) pairs, and after one barrier every warp stores its half-row to
// the token's kept destinations: x is read once and written k times.
constexpr int PM_TPC = PM_CHUNK / PM_SPLIT;        // tokens per scatter CTA
constexpr int PM_VMAX = 4;                          // 16-byte vectors per lane held at once
static_assert(PM_TPC * 2 == 8, "two warps per token, eight warps per CTA");

template <typename Tin>
__global__ void __launch_bounds__(256) perm_scatter_kernel(
    const int32_t *__restrict__ idx, int T, int k, int E, int C,
    const int32_t *__restrict__ chunk_base, const int32_t *__restrict__ offsets,
    int32_t *__restrict__ slot_pos, int32_t *__restrict__ src, const Tin *__restrict__ x,
    Tin *__restrict__ x_perm, int d) {
  griddep_wait();
  griddep_launch();
  extern __shared__ unsigned smask[];  // [E]
  __shared__ int s_pos[PM_CHUNK * 8];
  const bool active = (threadIdx.x & 31) < PM_CHUNK;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunk = blockIdx.x / PM_SPLIT, part = blockIdx.x % PM_SPLIT;
  // this warp's token and half-row
  const int tl = part * PM_TPC + (warp >> 1);  // token within the chunk
  const int tw = chunk * PM_CHUNK + tl;
  const int nvec = d * (int)sizeof(Tin) / 16;   // 16-byte vectors per row
  const int hv = (nvec + 1) / 2;
  const int vbeg = (warp & 1) * hv, vend = min(nvec, vbeg + hv);
  const uint4 *srow = (const uint4 *)(x + (size_t)(tw < T ? tw : 0) * d);
  const bool copy = x_perm != nullptr && tw < T;
  uint4 held[PM_VMAX];
  int v0 = vbeg;
  if (copy) {
#pragma unroll
    for (int i = 0; i < PM_VMAX; ++i) {
      const int v = v0 + lane + 32 * i;
      if (v < vend) held[i] = __ldg(srow + v);
    }
  }
  if (warp == 0) {
    const int t = chunk * PM_CHUNK + lane;
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
        if (active) s_pos[lane * k + j] = pos;
      }
    }
  }
  __syncthreads();
  if (!copy) return;
  for (;;) {
    for (int j = 0; j < k; ++j) {
      const int pos = s_pos[tl * k + j];
      if (pos < 0) continue;
      uint4 *drow = (uint4 *)(x_perm + (size_t)pos * d);
#pragma unroll
      for (int i = 0; i < PM_VMAX; ++i) {
        const int v = v0 + lane + 32 * i;
        if (v < vend) drow[v] = held[i];
      }
    }
    // rows longer than 2 * 32 * PM_VMAX vectors: the next slice of the half-row
    v0 += 32 * PM_VMAX;
    if (v0 >= vend) break;
#pragma unroll
    for (int i = 0; i < PM_VMAX; ++i) {
      const int v = v0 + lane + 32 * i;
      if (v < vend) held[i] = __ldg(srow + v);
    }
  }
}

}  // namespace moe

// Token permutation grouped by expert (Moonfrost expert card: experts as stacked (E, hidden,
// ffn) tensors with capacity-based routing, replacing a per-expert loop that synchronised the
// host once per expert; here nothing returns to the host at all).
//
// Stable counting sort of the (token, slot) pairs by expert, with the capacity mask:
//   rank(t, e) = #{t' < t : e in topk(t')};   kept iff rank < C;   row = offsets[e] + rank.
// Tokens are cut into chunks of 32 (one warp). Three launches:
//   hist    per-chunk expert histogram                        -> chunk_count[chunk][E]
//   scan    per-expert exclusive scan over chunks (warp/expert) -> chunk_base; the last CTA
//           scans the kept counts over experts                  -> offsets[E+1]
//   scatter per-chunk ranks from a per-expert lane bitmask, slot_pos / src_token, then the
//           CTA's eight warps copy the chunk's x rows to x_perm with 16-byte loads and stores.
#pragma once
#include "common.cuh"

namespace moe {

constexpr int PM_CHUNK = 32;

__global__ void __launch_bounds__(256) perm_hist_kernel(const int32_t *__restrict__ idx, int T,
                                                        int k, int E,
                                                        int32_t *__restrict__ chunk_count,
                                                        int nchunks, unsigned *scan_counter) {
  extern __shared__ int sh_cnt[];  // [8][E]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int *c = sh_cnt + warp * E;
  for (int e = lane; e < E; e += 32) c[e] = 0;
  __syncwarp();
  const int chunk = blockIdx.x * 8 + warp;
  if (blockIdx.x == 0 && threadIdx.x == 0) *scan_counter = 0u;  // consumed by perm_scan_kernel
  if (chunk >= nchunks) return;
  const int t = chunk * PM_CHUNK + lane;
  if (t < T) {
    for (int j = 0; j < k; ++j) {
      const int e = idx[(size_t)t * k + j];
      if (e >= 0 && e < E) atomicAdd(&c[e], 1);
      else set_device_error(MOE_ERR_DEVICE_CHECK, 100 + j);
    }
  }
  __syncwarp();
  for (int e = lane; e < E; e += 32) chunk_count[(size_t)chunk * E + e] = c[e];
}

__global__ void __launch_bounds__(256) perm_scan_kernel(const int32_t *__restrict__ chunk_count,
                                                        int32_t *__restrict__ chunk_base,
                                                        int nchunks, int E, int C,
                                                        int32_t *__restrict__ total,
                                                        int32_t *__restrict__ offsets,
                                                        unsigned *counter) {
  extern __shared__ int sh_scan[];  // [E] + tmp
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int e = blockIdx.x * 8 + warp;
  if (e < E) {
    int run = 0;
    for (int c0 = 0; c0 < nchunks; c0 += 32) {
      const int c = c0 + lane;
      const int v = c < nchunks ? chunk_count[(size_t)c * E + e] : 0;
      const int incl = warp_incl_scan(v);
      if (c < nchunks) chunk_base[(size_t)c * E + e] = run + incl - v;
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) total[e] = run;
  }
  __threadfence();
  __syncthreads();
  __shared__ int s_last;
  if (threadIdx.x == 0) s_last = (atomicAdd(counter, 1u) == gridDim.x - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  int *a = sh_scan;
  int *tmp = sh_scan + E;
  for (int i = threadIdx.x; i < E; i += blockDim.x) {
    const int n = __ldcg(total + i);
    a[i] = C < 0 ? n : min(n, C);
  }
  __syncthreads();
  const int tot = block_excl_scan_inplace(a, E, tmp);
  for (int i = threadIdx.x; i < E; i += blockDim.x) offsets[i] = a[i];
  if (threadIdx.x == 0) {
    offsets[E] = tot;
    *counter = 0u;
  }
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
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunk = blockIdx.x;
  const int t = chunk * PM_CHUNK + lane;
  if (warp == 0) {
    for (int e = lane; e < E; e += 32) smask[e] = 0u;
    __syncwarp();
    const bool valid = t < T;
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
          slot_pos[(size_t)t * k + j] = pos;
          if (pos >= 0) src[pos] = t;
        }
        s_pos[lane * k + j] = pos;
        s_tok[lane * k + j] = t;
      }
    }
  }
  __syncthreads();
  if (x_perm == nullptr) return;
  const int nvec = d * (int)sizeof(Tin) / 16;
  for (int s = warp; s < PM_CHUNK * k; s += 8) {
    const int pos = s_pos[s];
    if (pos < 0) continue;
    const uint4 *srow = (const uint4 *)(x + (size_t)s_tok[s] * d);
    uint4 *drow = (uint4 *)(x_perm + (size_t)pos * d);
    for (int v = lane; v < nvec; v += 32) drow[v] = __ldg(srow + v);
  }
}

}  // namespace moe

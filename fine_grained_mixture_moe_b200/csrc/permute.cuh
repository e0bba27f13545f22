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
//   stats   per-expert exclusive scan over chunks -> chunk_base; kept counts (stats.cuh)
//   scatter offsets[E+1] = exclusive scan of the kept counts (every CTA, in shared memory; block
//           0 writes them out, with the load-balancing loss); per-chunk ranks from a
//           per-expert lane bitmask, slot_pos / src_token; PM_SPLIT CTAs per chunk each bring 4
//           of its x rows into shared memory and store each to its k destinations in x_perm
//           with 1-D bulk copies (each row read once).
#pragma once
#include "common.cuh"

namespace moe {

constexpr int PM_CHUNK = 16;
constexpr int PM_SPLIT = 4;  // CTAs per chunk in the scatter

__global__ void __launch_bounds__(256) perm_hist_kernel(const int32_t *__restrict__ idx, int T,
                                                        int k, int E,
                                                        int32_t *__restrict__ chunk_count,
                                                        int nchunks) {
  griddep_wait();
  griddep_launch();
  extern __shared__ int sh_cnt[];  // [8][E]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  int *c = sh_cnt + warp * E;
  for (int e = lane; e < E; e += 32) c[e] = 0;
  __syncwarp();
  const int chunk = blockIdx.x * 8 + warp;
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

// Scatter. CTA (chunk, part) owns tokens chunk*16 + part*TPC .. +TPC (TPC = 16 / PM_SPLIT).
// Thread 0 first starts 1-D bulk copies of the CTA's token rows into shared memory (they do not
// depend on the routing); the chunk's routing, its per-expert base ranks and the kept counts are
// read together and the kept counts scanned into the expert offsets; warp 0 then ranks the
// chunk's (token, slot) pairs, and one thread per kept pair stores the whole row to its x_perm
// row with a single shared -> global bulk copy. x is read once and written k times by the copy
// engine. Block 0 also writes offsets[0..E] and, when `aux` is set, the load-balancing loss
// alpha E sum_e (count_e / (T k)) (prob_e / T) (Quartz: weight 0.01), in the order of
// aux_loss_kernel, so that the fused layer and the separate call agree bit for bit.
constexpr int PM_TPC = PM_CHUNK / PM_SPLIT;        // tokens per scatter CTA

template <typename Tin>
__global__ void __launch_bounds__(256) perm_scatter_kernel(
    const int32_t *__restrict__ idx, int T, int k, int E, int C,
    const int32_t *__restrict__ chunk_base, const int32_t *__restrict__ kept,
    int32_t *__restrict__ offsets, int32_t *__restrict__ slot_pos, int32_t *__restrict__ src,
    const Tin *__restrict__ x, Tin *__restrict__ x_perm, int d, const int32_t *__restrict__ count,
    const float *__restrict__ prob, float alpha, float *__restrict__ aux) {
  // [PM_TPC rows][row_bytes] | lane masks [E] | chunk base [E] | offsets [E]
  extern __shared__ __align__(128) unsigned char sm_raw[];
  __shared__ int s_pos[PM_CHUNK * 8];
  __shared__ int s_scan[256 / 32 + 1];
  __shared__ __align__(8) uint64_t s_bar;
  __shared__ volatile int s_abort;
  const bool active = (threadIdx.x & 31) < PM_CHUNK;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int chunk = blockIdx.x / PM_SPLIT, part = blockIdx.x % PM_SPLIT;
  const uint32_t row_bytes = (uint32_t)d * (uint32_t)sizeof(Tin);
  unsigned char *rows = sm_raw;
  unsigned *smask = (unsigned *)(sm_raw + (size_t)PM_TPC * row_bytes);
  int *s_base = (int *)(smask + E);  // this chunk's per-expert base rank and the expert offsets
  int *s_off = s_base + E;           // (from the kept counts), read alongside the routing
  const int tfirst = chunk * PM_CHUNK + part * PM_TPC;
  const int nrows = max(0, min(PM_TPC, T - tfirst));
  const bool copy = x_perm != nullptr && nrows > 0;
  const uint32_t bar = smem_u32(&s_bar);
  // Before griddep_wait: this kernel always follows the statistics kernel, whose CTAs allow it
  // to start only after their own griddep_wait, i.e. once the kernel before the statistics (the
  // router or the histogram) has completed and flushed. So x (an input of the call) and the
  // routing are final here; only the statistics' outputs (chunk bases, kept counts) wait. The
  // routing is read through L2 (ld.global.cg).
  if (tid == 0) {  // the rows do not depend on the routing: their copies go out first
    s_abort = 0;
    mbar_init(bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    if (copy) {
      mbar_expect_tx(bar, (uint32_t)nrows * row_bytes);
      for (int r = 0; r < nrows; ++r)
        bulk_load_1d(smem_u32(rows + (size_t)r * row_bytes), x + (size_t)(tfirst + r) * d,
                     row_bytes, bar);
    }
  }
  // warp 0 reads the chunk's routing while the other warps read the bases and kept counts
  const int t = chunk * PM_CHUNK + lane;
  int ev[8];
  if (warp == 0) {
    const bool valid = active && t < T;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      ev[j] = -1;
      if (j < k && valid) {
        const int e = __ldcg(idx + (size_t)t * k + j);
        if (e >= 0 && e < E) ev[j] = e;
      }
    }
  }
  griddep_wait();
  griddep_launch();
  for (int e = tid; e < E; e += blockDim.x) {
    smask[e] = 0u;
    s_base[e] = chunk_base[(size_t)chunk * E + e];
    s_off[e] = kept[e];
  }
  __syncthreads();  // the barrier is initialised, masks cleared, bases and kept counts in place
  const int n_kept = block_excl_scan_inplace(s_off, E, s_scan);  // -> expert offsets
  if (blockIdx.x == 0) {
    for (int e = tid; e < E; e += blockDim.x) offsets[e] = s_off[e];
    if (tid == 0) offsets[E] = n_kept;
    if (aux != nullptr && warp == 0) {
      double sd = 0.0;
      for (int e = lane; e < E; e += 32) sd += (double)count[e] * (double)prob[e];
      sd = warp_sum_d(sd);
      if (lane == 0) {
        double L = 0.0;
        if (T > 0) L = (double)alpha * (double)E * sd / ((double)T * (double)k * (double)T);
        *aux = (float)L;
      }
    }
  }
  if (warp == 0) {
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (ev[j] >= 0) atomicOr(&smask[ev[j]], 1u << lane);
    __syncwarp();
    const unsigned lt = lanemask_lt();
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (j < k) {
        int pos = -1;
        const int e = ev[j];
        if (e >= 0) {
          const int rank = s_base[e] + __popc(smask[e] & lt);
          if (C < 0 || rank < C) pos = s_off[e] + rank;
          if (part == 0) {
            slot_pos[(size_t)t * k + j] = pos;
            if (pos >= 0) src[pos] = t;
          }
        }
        if (active) s_pos[lane * k + j] = pos;
      }
    }
  }
  if (!copy) return;  // uniform over the CTA
  // rows landed (bounded wait; on expiry the error is recorded and the copies drain)
  mbar_wait(bar, 0u, &s_abort, g_wait_limit_ns, INFO_WAIT_SCATTER);
  __syncthreads();  // s_pos ready; every thread has seen the rows land or the abort
  if (s_abort) {
    if (tid == 0) {
      volatile int never = 0;
      mbar_wait(bar, 0u, &never, g_wait_limit_ns, INFO_WAIT_DRAIN);
    }
    return;
  }
  if (tid < nrows * k) {
    const int r = tid / k, j = tid - r * k;
    const int pos = s_pos[(part * PM_TPC + r) * k + j];
    if (pos >= 0) {
      bulk_store_1d(x_perm + (size_t)pos * d, smem_u32(rows + (size_t)r * row_bytes), row_bytes);
      bulk_store_commit_wait_read();  // the rows stay in shared memory until read
    }
  }
}

}  // namespace moe

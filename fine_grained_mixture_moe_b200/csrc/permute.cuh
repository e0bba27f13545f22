// Token permutation grouped by expert (Moonfrost expert card: experts as stacked (E, hidden,
// ffn) tensors routed under a per-expert capacity, replacing a per-expert loop that synchronised
// the host once per expert; here nothing returns to the host at all).
//
// Stable counting sort of the (token, slot) pairs by expert, with the capacity mask:
//   rank(t, e) = #{t' < t : e in topk(t')};   kept iff rank < C;   row = offsets[e] + rank.
// Tokens are cut into chunks of 16 (the router's CTA), and the rank splits into the chunk's base
// (the pairs of e in earlier chunks) and the rank within the chunk:
//   hist    per-chunk expert histogram -> chunk_count[chunk][E] and the within-chunk ranks
//           lrank[t][j] (inside the layer call the router writes both: its per-CTA counts are
//           this histogram; so this kernel is launched only by moe_permute on its own)
//   stats   per-expert exclusive scan over chunks -> chunk_base; kept counts (stats.cuh)
//   scatter offsets[E+1] = exclusive scan of the kept counts (every CTA, in shared memory; block
//           0 writes them out, with the load-balancing loss); then a warp per token:
//           row = offsets[e] + chunk_base[chunk][e] + lrank, slot_pos / src_token, and the token's
//           x row, read once into registers, stored to its k rows of x_perm.
#pragma once
#include "common.cuh"
#include "fp8.cuh"

namespace moe {

constexpr int PM_CHUNK = 16;
constexpr int PM_THREADS = 256;
constexpr int PM_CTAS_PER_SM = 4;
constexpr int PM_VEC = 8;  // 16-byte vectors of a row a lane holds at a time (4 KB per warp)

// One warp per chunk: per-expert lane masks of the chunk's tokens give both the chunk's counts
// and each pair's rank among the chunk's earlier tokens on the same expert.
__global__ void __launch_bounds__(256) perm_hist_kernel(const int32_t *__restrict__ idx, int T,
                                                        int k, int E,
                                                        int32_t *__restrict__ chunk_count,
                                                        uint8_t *__restrict__ lrank,
                                                        int nchunks) {
  const KernelStamp stamp(K_PERM_HIST);
  griddep_wait();
  stamp.started();
  griddep_launch();
  extern __shared__ unsigned sh_mask[];  // [8][E]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  unsigned *m = sh_mask + warp * E;
  for (int e = lane; e < E; e += 32) m[e] = 0u;
  __syncwarp();
  const int chunk = blockIdx.x * 8 + warp;
  if (chunk >= nchunks) return;
  const int t = chunk * PM_CHUNK + lane;
  const bool valid = lane < PM_CHUNK && t < T;
  int ev[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    ev[j] = -1;
    if (j < k && valid) {
      const int e = idx[(size_t)t * k + j];
      if (e >= 0 && e < E) {
        ev[j] = e;
        atomicOr(&m[e], 1u << lane);
      } else {
        set_device_error(MOE_ERR_DEVICE_CHECK, 100 + j);
      }
    }
  }
  __syncwarp();
  const unsigned lt = lanemask_lt();
#pragma unroll
  for (int j = 0; j < 8; ++j)
    if (j < k && valid) lrank[(size_t)t * k + j] = ev[j] >= 0 ? (uint8_t)__popc(m[ev[j]] & lt) : 0;
  for (int e = lane; e < E; e += 32) chunk_count[(size_t)chunk * E + e] = __popc(m[e]);
}

// Scatter. A persistent grid of PM_CTAS_PER_SM CTAs per SM; warp w of the grid takes tokens
// w, w + W, ... Per token: lanes j < k read the pair's expert and within-chunk rank, then the
// chunk's base rank of that expert; every lane reads its share of the x row (16-byte vectors,
// streaming) while those loads are in flight, and stores it to each kept pair's row of x_perm.
// Before the per-token loop every CTA scans the kept counts into the expert offsets in shared
// memory; block 0 writes offsets[0..E] and, when `aux` is set, the load-balancing loss
// alpha E sum_e (count_e / (T k)) (prob_e / T) (Quartz: weight 0.01), in the order of
// aux_loss_kernel, so that the fused layer and the separate call agree bit for bit.
// Before griddep_wait: this kernel always follows the statistics kernel, whose CTAs allow it to
// start only after their own griddep_wait, i.e. once the kernel before the statistics (the
// router or the histogram) has completed and flushed. So x, the routing and the within-chunk
// ranks are final at entry; only the statistics' outputs (chunk bases, kept counts) wait.
template <typename Tin>
__global__ void __launch_bounds__(PM_THREADS, PM_CTAS_PER_SM) perm_scatter_kernel(
    const int32_t *__restrict__ idx, const uint8_t *__restrict__ lrank, int T, int k, int E,
    int C, const int32_t *__restrict__ chunk_base, const int32_t *__restrict__ kept,
    int32_t *__restrict__ offsets, int32_t *__restrict__ slot_pos, int32_t *__restrict__ src,
    const Tin *__restrict__ x, Tin *__restrict__ x_perm, int d,
    const int32_t *__restrict__ count, const float *__restrict__ prob, float alpha,
    float *__restrict__ aux) {
  extern __shared__ int s_off[];  // [E] expert offsets
  __shared__ int s_scan[PM_THREADS / 32 + 1];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nwarps = gridDim.x * (PM_THREADS / 32);
  const int gw = blockIdx.x * (PM_THREADS / 32) + warp;
  const int nvec = (int)(((size_t)d * sizeof(Tin)) >> 4);  // 16-byte vectors per row
  const bool copy = x_perm != nullptr;
  const uint4 *xv = (const uint4 *)x;
  uint4 *pv = (uint4 *)x_perm;

  // the first token's row and routing do not depend on the statistics: they load before the wait
  uint4 row[PM_VEC];
  int e_l = -1, r_l = 0;
  int t = gw;
  auto load_token = [&](int tt) {
    if (lane < k) {
      e_l = __ldcg(idx + (size_t)tt * k + lane);
      r_l = (int)__ldcg(lrank + (size_t)tt * k + lane);
    }
    if (copy) {
#pragma unroll
      for (int i = 0; i < PM_VEC; ++i) {
        const int v = lane + 32 * i;
        if (v < nvec) row[i] = __ldcs(xv + (size_t)tt * nvec + v);
      }
    }
  };
  const KernelStamp stamp(K_PERM_SCATTER);
  if (t < T) load_token(t);
  griddep_wait();
  stamp.started();
  griddep_launch();
  for (int e = tid; e < E; e += PM_THREADS) s_off[e] = kept[e];
  __syncthreads();
  const int n_kept = block_excl_scan_inplace(s_off, E, s_scan);  // -> expert offsets
  if (blockIdx.x == 0) {
    for (int e = tid; e < E; e += PM_THREADS) offsets[e] = s_off[e];
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
  for (; t < T; t += nwarps) {
    // the pair's row: offsets[e] + chunk base + within-chunk rank, -1 past the capacity
    int pos = -1;
    if (lane < k) {
      const int e = e_l;
      if (e >= 0 && e < E) {
        const int rank = __ldcg(chunk_base + (size_t)(t / PM_CHUNK) * E + e) + r_l;
        if (C < 0 || rank < C) pos = s_off[e] + rank;
        slot_pos[(size_t)t * k + lane] = pos;
        if (pos >= 0) src[pos] = t;
      } else {
        slot_pos[(size_t)t * k + lane] = -1;
        set_device_error(MOE_ERR_DEVICE_CHECK, 100 + lane);
      }
    }
    if (copy) {
      for (int j = 0; j < k; ++j) {
        const int pj = __shfl_sync(0xffffffffu, pos, j);
        if (pj < 0) continue;
#pragma unroll
        for (int i = 0; i < PM_VEC; ++i) {
          const int v = lane + 32 * i;
          if (v < nvec) pv[(size_t)pj * nvec + v] = row[i];
        }
      }
      // rows wider than PM_VEC vectors per lane: the rest in further passes
      for (int v0 = 32 * PM_VEC; v0 < nvec; v0 += 32 * PM_VEC) {
#pragma unroll
        for (int i = 0; i < PM_VEC; ++i) {
          const int v = v0 + lane + 32 * i;
          if (v < nvec) row[i] = __ldcs(xv + (size_t)t * nvec + v);
        }
        for (int j = 0; j < k; ++j) {
          const int pj = __shfl_sync(0xffffffffu, pos, j);
          if (pj < 0) continue;
#pragma unroll
          for (int i = 0; i < PM_VEC; ++i) {
            const int v = v0 + lane + 32 * i;
            if (v < nvec) pv[(size_t)pj * nvec + v] = row[i];
          }
        }
      }
    }
    if (t + nwarps < T) load_token(t + nwarps);
  }
}

// The same scatter for a layer whose experts take E4M3 rows: each bf16 token row is quantised
// on its way (per-row scale amax / 448, codes as quantize_rows_kernel makes them, bit for bit)
// and its codes and scale are stored to every kept pair's row: xq_perm [rows, d] bytes,
// sx_perm [rows]. The row is held in registers between its maximum and its conversion, so d is
// at most 32 * PM_VEC * 8 elements (moe_config checks).
__global__ void __launch_bounds__(PM_THREADS, PM_CTAS_PER_SM) perm_scatter_q8_kernel(
    const int32_t *__restrict__ idx, const uint8_t *__restrict__ lrank, int T, int k, int E,
    int C, const int32_t *__restrict__ chunk_base, const int32_t *__restrict__ kept,
    int32_t *__restrict__ offsets, int32_t *__restrict__ slot_pos, int32_t *__restrict__ src,
    const __nv_bfloat16 *__restrict__ x, uint8_t *__restrict__ xq_perm,
    float *__restrict__ sx_perm, int d, const int32_t *__restrict__ count,
    const float *__restrict__ prob, float alpha, float *__restrict__ aux) {
  extern __shared__ int s_off[];  // [E] expert offsets
  __shared__ int s_scan[PM_THREADS / 32 + 1];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nwarps = gridDim.x * (PM_THREADS / 32);
  const int gw = blockIdx.x * (PM_THREADS / 32) + warp;
  const int nvec = d >> 3;  // 16-byte vectors (8 bf16) per row
  const uint4 *xv = (const uint4 *)x;
  uint2 *qv = (uint2 *)xq_perm;  // 8 codes per input vector

  uint4 row[PM_VEC];
  int e_l = -1, r_l = 0;
  int t = gw;
  auto load_token = [&](int tt) {
    if (lane < k) {
      e_l = __ldcg(idx + (size_t)tt * k + lane);
      r_l = (int)__ldcg(lrank + (size_t)tt * k + lane);
    }
#pragma unroll
    for (int i = 0; i < PM_VEC; ++i) {
      const int v = lane + 32 * i;
      if (v < nvec) row[i] = __ldcs(xv + (size_t)tt * nvec + v);
    }
  };
  const KernelStamp stamp(K_PERM_SCATTER);
  if (t < T) load_token(t);
  griddep_wait();
  stamp.started();
  griddep_launch();
  for (int e = tid; e < E; e += PM_THREADS) s_off[e] = kept[e];
  __syncthreads();
  const int n_kept = block_excl_scan_inplace(s_off, E, s_scan);
  if (blockIdx.x == 0) {
    for (int e = tid; e < E; e += PM_THREADS) offsets[e] = s_off[e];
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
  for (; t < T; t += nwarps) {
    // the row's scale
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < PM_VEC; ++i) {
      if (lane + 32 * i < nvec) {
        const __nv_bfloat162 *h = (const __nv_bfloat162 *)&row[i];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = __bfloat1622float2(h[j]);
          amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
        }
      }
    }
    amax = warp_max_f(amax);
    const float sc = amax > 0.0f ? __fdiv_rn(amax, E4M3_MAX) : 1.0f;
    // the pair's row, as in perm_scatter_kernel
    int pos = -1;
    if (lane < k) {
      const int e = e_l;
      if (e >= 0 && e < E) {
        const int rank = __ldcg(chunk_base + (size_t)(t / PM_CHUNK) * E + e) + r_l;
        if (C < 0 || rank < C) pos = s_off[e] + rank;
        slot_pos[(size_t)t * k + lane] = pos;
        if (pos >= 0) {
          src[pos] = t;
          sx_perm[pos] = sc;
        }
      } else {
        slot_pos[(size_t)t * k + lane] = -1;
        set_device_error(MOE_ERR_DEVICE_CHECK, 100 + lane);
      }
    }
    // the codes of vector i replace its first 8 bytes in place (vectors past the row hold no
    // data: no division runs on them)
#pragma unroll
    for (int i = 0; i < PM_VEC; ++i) {
      if (lane + 32 * i >= nvec) continue;
      const __nv_bfloat162 *h = (const __nv_bfloat162 *)&row[i];
      uint32_t w[2];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const float2 a = __bfloat1622float2(h[2 * j]), b = __bfloat1622float2(h[2 * j + 1]);
        w[j] = e4m3_code(__fdiv_rn(a.x, sc)) | (e4m3_code(__fdiv_rn(a.y, sc)) << 8) |
               (e4m3_code(__fdiv_rn(b.x, sc)) << 16) | (e4m3_code(__fdiv_rn(b.y, sc)) << 24);
      }
      row[i].x = w[0];
      row[i].y = w[1];
    }
    for (int j = 0; j < k; ++j) {
      const int pj = __shfl_sync(0xffffffffu, pos, j);
      if (pj < 0) continue;
#pragma unroll
      for (int i = 0; i < PM_VEC; ++i) {
        const int v = lane + 32 * i;
        if (v < nvec) qv[(size_t)pj * nvec + v] = make_uint2(row[i].x, row[i].y);
      }
    }
    if (t + nwarps < T) load_token(t + nwarps);
  }
}

}  // namespace moe

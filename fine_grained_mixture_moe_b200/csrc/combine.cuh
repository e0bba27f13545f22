// Weighted un-permute and the load-balancing loss.
//
// combine: y[t] = y_shared[t] + sum_j [slot_pos[t,j] >= 0] w[t,j] * y_perm[slot_pos[t,j]]
// (Moonfrost expert card: a token passes through the shared expert and its top-k routed ones),
// summed in fp32 in slot order. The routed outputs y_perm are in the layer's dtype (bf16 rows
// average out in the weighted sum); the shared output and y are fp32, since a bf16 rounding of
// y itself would cost up to 2^-8 max|y| / rms(y), the whole error budget. A gather: no atomics,
// bitwise-deterministic.
//
// aux: L = alpha * E * sum_i (count_i / (T k)) * (prob_sum_i / T) (Quartz: the load-balancing
// term, weight 0.01), accumulated in fp64 in a fixed order.
#pragma once
#include "common.cuh"

namespace moe {

// One 16-byte vector of expert outputs: 4 fp32 (fp32 layers) or 8 bf16 (bf16 layers), loaded
// with the streaming hint (each row is read once) and accumulated in fp32.
template <typename Ty> struct YVec;
template <> struct YVec<float> {
  using raw_t = float4;
  static constexpr int N = 4;
  static __device__ __forceinline__ raw_t load(const float *p) { return __ldcs((const float4 *)p); }
  static __device__ __forceinline__ void fma(float w, raw_t q, float *a) {
    a[0] = fmaf(w, q.x, a[0]);
    a[1] = fmaf(w, q.y, a[1]);
    a[2] = fmaf(w, q.z, a[2]);
    a[3] = fmaf(w, q.w, a[3]);
  }
};
template <> struct YVec<__nv_bfloat16> {
  using raw_t = uint4;
  static constexpr int N = 8;
  static __device__ __forceinline__ raw_t load(const __nv_bfloat16 *p) {
    return __ldcs((const uint4 *)p);
  }
  static __device__ __forceinline__ void fma(float w, raw_t q, float *a) {
    const __nv_bfloat162 *h = (const __nv_bfloat162 *)&q;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(h[i]);
      a[2 * i] = fmaf(w, f.x, a[2 * i]);
      a[2 * i + 1] = fmaf(w, f.y, a[2 * i + 1]);
    }
  }
};

// One warp per token; each lane owns one 16-byte vector of expert outputs (N columns) per pass,
// with the pass's k row loads and the shared-output load issued before the sums. About 60
// registers, so 4 CTAs (32 warps) fit per SM and a Quartz-sized call is one wave. d is a
// multiple of 64, so a lane's vector is wholly inside or wholly outside the row.
// early: slot_pos and w were written at least two kernels before this one in the stream (inside
// the layer, the expert GEMMs lie between the scatter and the combine). The kernel just before
// lets this one start only after its own griddep_wait, so they are final at entry and are read
// (through L2) before griddep_wait; only y_perm and y_shared wait for it.
template <typename Ty>
__global__ void __launch_bounds__(256, sizeof(Ty) == 2 ? 4 : 3) combine_kernel(const Ty *__restrict__ y_perm,
                                                         const float *__restrict__ y_shared,
                                                         const int32_t *__restrict__ slot_pos,
                                                         const float *__restrict__ w,
                                                         float *__restrict__ y, int T, int k,
                                                         int d, bool early) {
  using YV = YVec<Ty>;
  constexpr int V = YV::N;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + warp;
  const KernelStamp stamp(K_COMBINE);
  if (!early) griddep_wait();
  int pos_l = -1;
  float w_l = 0.0f;
  if (t < T && lane < k) {
    pos_l = __ldcg(slot_pos + (size_t)t * k + lane);
    w_l = w ? __ldcg(w + (size_t)t * k + lane) : 1.0f;  // no weights: the plain sum (un-permute)
  }
  if (early) griddep_wait();
  stamp.started();
  griddep_launch();
  if (t >= T) return;
  int pos[8];
  float wj[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    pos[j] = __shfl_sync(0xffffffffu, pos_l, j);
    wj[j] = __shfl_sync(0xffffffffu, w_l, j);
  }
#pragma unroll 1
  for (int c = lane * V; c < d; c += 32 * V) {
    float acc[V];
#pragma unroll
    for (int i = 0; i < V; i += 4) {
      float4 q = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
      if (y_shared) q = __ldcs((const float4 *)(y_shared + (size_t)t * d + c + i));
      acc[i] = q.x;
      acc[i + 1] = q.y;
      acc[i + 2] = q.z;
      acc[i + 3] = q.w;
    }
    typename YV::raw_t v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (j < k && pos[j] >= 0) v[j] = YV::load(y_perm + (size_t)pos[j] * d + c);
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (j < k && pos[j] >= 0) YV::fma(wj[j], v[j], acc);
#pragma unroll
    for (int i = 0; i < V; i += 4)
      __stcs((float4 *)(y + (size_t)t * d + c + i),
             make_float4(acc[i], acc[i + 1], acc[i + 2], acc[i + 3]));
  }
}

__global__ void aux_loss_kernel(const int32_t *__restrict__ count, const float *__restrict__ prob,
                                int E, int T, int k, float alpha, float *__restrict__ loss) {
  const KernelStamp stamp(K_AUX);
  griddep_wait();
  stamp.started();
  griddep_launch();
  double s = 0.0;
  for (int e = threadIdx.x; e < E; e += 32) s += (double)count[e] * (double)prob[e];
  s = warp_sum_d(s);
  if (threadIdx.x == 0) {
    double L = 0.0;
    if (T > 0) L = (double)alpha * (double)E * s / ((double)T * (double)k * (double)T);
    *loss = (float)L;
  }
}

}  // namespace moe

// Weighted un-permute and the load-balancing loss.
//
// combine: y[t] = y_shared[t] + sum_j [slot_pos[t,j] >= 0] w[t,j] * y_perm[slot_pos[t,j]]
// (Moonfrost: "a token passes through 4 of 33" - the shared expert plus its top-3), summed in
// fp32 in slot order; expert outputs and y are fp32 (a bf16 rounding of y alone would cost
// up to 2^-8 max|y| / rms(y), the whole error budget). A gather: no atomics, bitwise-deterministic.
// One warp per token, 16-byte vectors along the hidden dimension.
//
// aux: L = alpha * E * sum_i (count_i / (T k)) * (prob_sum_i / T) (Quartz "0.01-weighted
// load-balancing loss"), accumulated in fp64 in a fixed order.
#pragma once
#include "common.cuh"

namespace moe {

template <typename T> struct Vec16;
template <> struct Vec16<float> {
  static constexpr int N = 4;
  static __device__ __forceinline__ void load(const float *p, float *v) {
    const float4 q = __ldg((const float4 *)p);
    v[0] = q.x; v[1] = q.y; v[2] = q.z; v[3] = q.w;
  }
  static __device__ __forceinline__ void store(float *p, const float *v) {
    *(float4 *)p = make_float4(v[0], v[1], v[2], v[3]);
  }
};
template <> struct Vec16<__nv_bfloat16> {
  static constexpr int N = 8;
  static __device__ __forceinline__ void load(const __nv_bfloat16 *p, float *v) {
    const uint4 q = __ldg((const uint4 *)p);
    const __nv_bfloat162 *h = (const __nv_bfloat162 *)&q;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(h[i]);
      v[2 * i] = f.x;
      v[2 * i + 1] = f.y;
    }
  }
  static __device__ __forceinline__ void store(__nv_bfloat16 *p, const float *v) {
    uint4 q;
    __nv_bfloat162 *h = (__nv_bfloat162 *)&q;
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
    *(uint4 *)p = q;
  }
};

__global__ void __launch_bounds__(256) combine_kernel(const float *__restrict__ y_perm,
                                                      const float *__restrict__ y_shared,
                                                      const int32_t *__restrict__ slot_pos,
                                                      const float *__restrict__ w,
                                                      float *__restrict__ y, int T, int k, int d) {
  using Tio = float;
  constexpr int V = Vec16<Tio>::N;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t = blockIdx.x * 8 + warp;
  if (t >= T) return;
  int pos_l = -1;
  float w_l = 0.0f;
  if (lane < k) {
    pos_l = slot_pos[(size_t)t * k + lane];
    w_l = w[(size_t)t * k + lane];
  }
  int pos[8];
  float wj[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    pos[j] = __shfl_sync(0xffffffffu, pos_l, j);
    wj[j] = __shfl_sync(0xffffffffu, w_l, j);
  }
  // two vectors per lane per pass, all loads of a pass issued before the sums
#pragma unroll 1
  for (int c0 = lane * V; c0 < d; c0 += 64 * V) {
    float acc[2][V];
    float v[2][8][V];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int c = c0 + h * 32 * V;
      if (c < d) {
        if (y_shared) Vec16<Tio>::load(y_shared + (size_t)t * d + c, acc[h]);
        else {
#pragma unroll
          for (int i = 0; i < V; ++i) acc[h][i] = 0.0f;
        }
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (j < k && pos[j] >= 0) Vec16<Tio>::load(y_perm + (size_t)pos[j] * d + c, v[h][j]);
      }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int c = c0 + h * 32 * V;
      if (c < d) {
#pragma unroll
        for (int j = 0; j < 8; ++j)
          if (j < k && pos[j] >= 0) {
#pragma unroll
            for (int i = 0; i < V; ++i) acc[h][i] = fmaf(wj[j], v[h][j][i], acc[h][i]);
          }
        __stcs((float4 *)(y + (size_t)t * d + c), make_float4(acc[h][0], acc[h][1], acc[h][2], acc[h][3]));
      }
    }
  }
}

__global__ void aux_loss_kernel(const int32_t *__restrict__ count, const float *__restrict__ prob,
                                int E, int T, int k, float alpha, float *__restrict__ loss) {
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

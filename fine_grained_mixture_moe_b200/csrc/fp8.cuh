// Per-row E4M3 quantisation (the fp8 rung of the low-rank experts' storage ladder: dormouse,
// "TSCT low-rank experts", the U diag(s) V^T factorisation stored as fp8 -> NVFP4 -> ternary).
//
// For each row v of a [rows, cols] matrix (bf16 or fp32):
//   amax = max |v_i| (exact);  s = amax / 448 rounded to fp32 (1 for an all-zero row);
//   q_i  = E4M3(v_i / s): the quotient rounded to fp32, then to the nearest E4M3 value with ties
//          to the even code, magnitudes past 448 saturated (the conversion instruction's
//          round-to-nearest-even, satfinite form).
// One warp per row: the row is read twice (the second time from L1 / L2), the codes written
// with 4-byte stores.
#pragma once
#include <cuda_fp8.h>

#include "common.cuh"

namespace moe {

constexpr float E4M3_MAX = 448.0f;

template <typename Tin> struct QLoad;
template <> struct QLoad<float> {  // four elements as fp32
  static __device__ __forceinline__ float4 ld(const float *p) { return __ldg((const float4 *)p); }
};
template <> struct QLoad<__nv_bfloat16> {
  static __device__ __forceinline__ float4 ld(const __nv_bfloat16 *p) {
    const uint2 u = __ldg((const uint2 *)p);
    const float2 a = __bfloat1622float2(*(const __nv_bfloat162 *)&u.x);
    const float2 b = __bfloat1622float2(*(const __nv_bfloat162 *)&u.y);
    return make_float4(a.x, a.y, b.x, b.y);
  }
};

__device__ __forceinline__ uint32_t e4m3_code(float v) {
  return (uint32_t)__nv_cvt_float_to_fp8(v, __NV_SATFINITE, __NV_E4M3);
}

// cols a multiple of 4; rows of `in` (row stride cols) to rows of q (row stride cols) and scale.
template <typename Tin>
__global__ void __launch_bounds__(256) quantize_rows_kernel(const Tin *__restrict__ in,
                                                            long long rows, int cols,
                                                            uint8_t *__restrict__ q,
                                                            float *__restrict__ scale) {
  const KernelStamp stamp(K_QUANT);
  griddep_wait();
  stamp.started();
  griddep_launch();
  const int lane = threadIdx.x & 31;
  const long long nwarps = (long long)gridDim.x * (blockDim.x >> 5);
  for (long long r = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows;
       r += nwarps) {
    const Tin *row = in + r * cols;
    float amax = 0.0f;
    for (int c = 4 * lane; c < cols; c += 128) {
      const float4 v = QLoad<Tin>::ld(row + c);
      amax = fmaxf(amax, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
    }
    amax = warp_max_f(amax);
    const float s = amax > 0.0f ? __fdiv_rn(amax, E4M3_MAX) : 1.0f;
    if (lane == 0) scale[r] = s;
    uint32_t *qrow = (uint32_t *)(q + r * cols);
    for (int c = 4 * lane; c < cols; c += 128) {
      const float4 v = QLoad<Tin>::ld(row + c);
      qrow[c >> 2] = e4m3_code(__fdiv_rn(v.x, s)) | (e4m3_code(__fdiv_rn(v.y, s)) << 8) |
                     (e4m3_code(__fdiv_rn(v.z, s)) << 16) | (e4m3_code(__fdiv_rn(v.w, s)) << 24);
    }
  }
}

}  // namespace moe

// fp32 operands of the tensor-core products as three bf16 terms (the fp32 configuration's
// contractions on tcgen05 kind::f16).
//
// v = hi + mid + lo with hi = bf16(v), mid = bf16(v - hi), lo = bf16(v - hi - mid): each
// subtraction is exact in fp32, so v - (hi + mid + lo) is lo's own rounding, at most 2^-9 of a
// value below 2^-16 |v|. A product a b is taken as the six cross terms of order up to 2^-16:
//   a_hi b_hi + a_hi b_mid + a_mid b_hi + a_hi b_lo + a_lo b_hi + a_mid b_mid,
// leaving out a_mid b_lo + a_lo b_mid + a_lo b_lo (below 2^-24 |a b|), each product exact in the
// fp32 accumulator. The split writes each operand as six K segments in that order (A: hi hi mid
// hi lo mid; B: hi mid hi lo hi mid), so the GEMM over K' = 6 K sums exactly these six terms.
// A matrix whose K is cut into pieces (the shared experts' down projections, one piece per
// expert) keeps its pieces: each piece becomes its own six segments.
#pragma once
#include "common.cuh"

namespace moe {

// The term (0 hi, 1 mid, 2 lo) of segment s for the A and the B operand.
__host__ __device__ constexpr int split_term(bool b_operand, int s) {
  return b_operand ? (s == 1 || s == 5 ? 1 : s == 3 ? 2 : 0)
                   : (s == 2 || s == 5 ? 1 : s == 4 ? 2 : 0);
}

// in [rows, cols] fp32 (row-major); out [rows, 6 cols] bf16: for piece p (cols / piece of them),
// segment s, element j: out[row][6 p piece + s piece + j] = term(s) of in[row][p piece + j].
__global__ void __launch_bounds__(256) split6_bf16_kernel(const float *__restrict__ in,
                                                          long long rows, int cols, int piece,
                                                          int b_operand,
                                                          __nv_bfloat16 *__restrict__ out) {
  griddep_wait();
  griddep_launch();
  const long long n = rows * cols;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (long long)gridDim.x * blockDim.x) {
    const long long row = i / cols;
    const int c = (int)(i - row * cols);
    const int p = c / piece, j = c - p * piece;
    const float v = in[i];
    __nv_bfloat16 t[3];
    t[0] = __float2bfloat16_rn(v);
    const float r1 = v - __bfloat162float(t[0]);
    t[1] = __float2bfloat16_rn(r1);
    t[2] = __float2bfloat16_rn(r1 - __bfloat162float(t[1]));
    __nv_bfloat16 *o = out + row * (6ll * cols) + 6ll * p * piece + j;
#pragma unroll
    for (int s = 0; s < 6; ++s) o[(long long)s * piece] = t[split_term(b_operand != 0, s)];
  }
}

}  // namespace moe

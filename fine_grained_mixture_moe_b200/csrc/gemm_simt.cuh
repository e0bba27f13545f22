// fp32 grouped GEMM on CUDA cores, for the fp32 configuration (the accuracy target there is
// 1e-4 relative, which single-pass TF32 tensor-core products cannot meet). Same grouped
// problem, tile scheduler and epilogues as the tensor-core kernel; 64x64 tiles, 4x4 per thread.
#pragma once
#include "grouped.cuh"

namespace moe {

constexpr int SM_BM = 64, SM_BN = 64, SM_BK = 16;

template <typename Tin, typename Tout, int MODE>
__global__ void __launch_bounds__(256) gemm_simt_kernel(GroupedGemm p) {
  __shared__ float As[SM_BK][SM_BM + 4];
  __shared__ float Bs0[SM_BK][SM_BN + 4];
  __shared__ float Bs1[SM_BK][SM_BN + 4];
  extern __shared__ int sh_prefix[];  // [G+1] + scan tmp
  const int G = p.E + p.has_shared;
  int *prefix = sh_prefix;
  int *tmp = sh_prefix + G + 1;
  const KernelStamp stamp(p.kind);
  griddep_wait();
  stamp.started();
  griddep_launch();
  const int total = build_tile_prefix(p, SM_BM, SM_BN, prefix, tmp);
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;

  for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
    const TileInfo ti = decode_tile(p, tile, prefix, SM_BM, SM_BN);
    const bool routed = ti.g < p.E;
    const Tin *A = (const Tin *)(routed ? p.A_r : p.A_s);
    const int lda = routed ? p.lda_r : p.lda_s;
    const Tin *B0 = (const Tin *)(routed ? p.B0_r : p.B0_s);
    const Tin *B1 = (const Tin *)(routed ? p.B1_r : p.B1_s);
    const int pk = routed ? ti.K : p.piece_k;
    const int prow = routed ? 0 : p.piece_rows;
    if (routed) {
      B0 += (size_t)ti.g * ti.N * ti.K;
      if (MODE == MODE_GATEUP) B1 += (size_t)ti.g * ti.N * ti.K;
    }
    float acc0[4][4], acc1[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc0[i][j] = acc1[i][j] = 0.0f;

    for (int k0 = 0; k0 < ti.K; k0 += SM_BK) {
      for (int i = tid; i < SM_BM * SM_BK; i += 256) {
        const int r = i / SM_BK, c = i % SM_BK;
        const int row = ti.m0 + r, kk = k0 + c;
        float v = 0.0f;
        if (row < ti.rows && kk < ti.K)
          v = Elem<Tin>::to_f(A[(size_t)(ti.a_row0 + row) * lda + kk]);
        As[c][r] = v;
      }
      for (int i = tid; i < SM_BN * SM_BK; i += 256) {
        const int n = i / SM_BK, c = i % SM_BK;
        const int col = ti.n0 + n, kk = k0 + c;
        float v0 = 0.0f, v1 = 0.0f;
        if (col < ti.N && kk < ti.K) {
          const int piece = kk / pk;
          const size_t off = (size_t)(piece * prow + col) * pk + (kk - piece * pk);
          v0 = Elem<Tin>::to_f(B0[off]);
          if (MODE == MODE_GATEUP) v1 = Elem<Tin>::to_f(B1[off]);
        }
        Bs0[c][n] = v0;
        if (MODE == MODE_GATEUP) Bs1[c][n] = v1;
      }
      __syncthreads();
#pragma unroll
      for (int c = 0; c < SM_BK; ++c) {
        float a[4], b0[4], b1[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          a[i] = As[c][ty * 4 + i];
          b0[i] = Bs0[c][tx * 4 + i];
          if (MODE == MODE_GATEUP) b1[i] = Bs1[c][tx * 4 + i];
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            acc0[i][j] = fmaf(a[i], b0[j], acc0[i][j]);
            if (MODE == MODE_GATEUP) acc1[i][j] = fmaf(a[i], b1[j], acc1[i][j]);
          }
      }
      __syncthreads();
    }
    Tout *out = (Tout *)(routed ? p.out_r : p.out_s);
    const int ldo = routed ? p.ldo_r : p.ldo_s;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int row = ti.m0 + ty * 4 + i;
      if (row >= ti.rows) continue;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int col = ti.n0 + tx * 4 + j;
        if (col >= ti.N) continue;
        float v;
        if (MODE == MODE_GATEUP) v = silu_f(acc0[i][j]) * acc1[i][j];
        else if (MODE == MODE_SCALE) v = acc0[i][j] * p.scale[(size_t)ti.g * ti.N + col];
        else v = acc0[i][j];
        out[(size_t)(ti.a_row0 + row) * ldo + col] = Elem<Tout>::from_f(v);
      }
    }
  }
}

}  // namespace moe

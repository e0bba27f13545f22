// Grouped-GEMM problem description of the tensor-core kernels (gemm_tc.cuh, gemm_tc2.cuh).
//
// A launch covers up to E routed groups plus one shared group:
//   routed group g < E : rows offsets[g]..offsets[g+1] of A_r / out_r, weight B*_r + g*N_r*K_r
//                        ([N_r, K_r] row-major, i.e. K-major), read from device memory only
//   shared group g = E : rows 0..T of A_s / out_s, weight B*_s. Its K may be split into pieces
//                        of width piece_k whose rows sit piece_rows apart: element (n, kk) of
//                        B*_s is at ((kk / piece_k) * piece_rows + n) * piece_k + kk % piece_k.
//                        This reads the shared down projections [S, d, fs] as one [d, S*fs]
//                        matrix, so S shared experts of width fs act as one of width S*fs.
// Epilogue modes: GATEUP out = silu(A B0^T) * (A B1^T) (SwiGLU, gate and up fused; GATEUP_F32
//                   the same stored as fp32);
//                 PLAIN  out = A B0^T;   SCALE out = (A B0^T) * scale[g][n] (low-rank s);
//                 GATEUP_RAW (backward) g = A B0^T and u = A B1^T (fp32) to out, in the
//                   blocked g, u layout of backward_epilogue.cuh (half = the width of g);
//                 SWIGLU_BWD (backward) dh = A B0^T with fp32 g, u read from aux (the same
//                   blocked layout); dg = dh u silu'(g), du = dh silu(g) and h = silu(g) u, each
//                   as two bf16 terms (v = hi + lo, hi = bf16(v), lo = bf16(v - hi)): out[., n] =
//                   dg_hi, out[., half + n] = du_hi, out[., 2 half + n] = dg_lo,
//                   out[., 3 half + n] = du_lo, out2[., n] = h_hi, out2[., half + n] = h_lo.
//                 SCALE_FP8 (E4M3 operands) z = (A B0^T) * row_scale[row] * col_scale[g][n]
//                   * scale[g][n] (the low-rank V projection with fp8 storage), stored as the
//                   row's E4M3 codes to out (bytes) and its scale to out2 (fp32 per row), as
//                   quantize_rows_kernel would make them from z; the tile is the whole row (N);
//                 PLAIN_FP8 (E4M3 operands) out = (A B0^T) * row_scale[row] * col_scale[g][n],
//                   fp32 out (the U projection). E4M3 operands have K-blocks of 128 elements
//                   (128 bytes, as for bf16); a K that is not a multiple of 128 is completed with
//                   the tensor map's zero fill.
// Groups along K (kgroup, backward weight gradients): group g is out rows [g M, g M + M) =
// A[M, K_g] B[N, K_g]^T, where A and B are K-major [M or N][ld] and group g takes their columns
// kseg koff[g] .. kseg koff[g+1] (koff padded to multiples of 64; kseg segments per group, so a
// sum of split terms runs as one product); M is rows_r and ld is K_r. With mn set, A and B are
// instead read MN-major from the row-major activations themselves (fields below).
// Output types in the tensor-core kernels: GATEUP and SCALE write bf16 (the next product's
// operand, SCALE optionally as a hi + lo pair) or, with out_f32, fp32; PLAIN writes the routed
// groups' rows in bf16 or fp32 (out_r_bf16) and the shared group's rows in fp32.
#pragma once
#include "common.cuh"

namespace moe {

enum GemmMode { MODE_GATEUP = 0, MODE_PLAIN = 1, MODE_SCALE = 2, MODE_GATEUP_RAW = 3,
                MODE_SWIGLU_BWD = 4, MODE_SCALE_FP8 = 5, MODE_PLAIN_FP8 = 6, MODE_GATEUP_F32 = 7 };

// Modes whose operands are E4M3 bytes (tcgen05 kind::f8f6f4) rather than bf16 (kind::f16).
__host__ __device__ constexpr bool mode_fp8(int mode) {
  return mode == MODE_SCALE_FP8 || mode == MODE_PLAIN_FP8;
}
// Elements of K per pipeline stage: one 128-byte swizzle row of either type.
__host__ __device__ constexpr int mode_bk(int mode) { return mode_fp8(mode) ? 128 : 64; }

struct GroupedGemm {
  const int32_t *offsets;  // [E+1] device
  int E;                   // routed groups in this launch (0: shared only)
  const void *A_r;
  int lda_r;
  int rows_r;              // rows held by the A_r / out_r buffers (T*top_k): tensor-map extent
  const void *B0_r, *B1_r;
  int N_r, K_r;
  void *out_r;
  int ldo_r;
  const float *scale;  // [E, N_r] for MODE_SCALE and MODE_SCALE_FP8
  const float *row_scale;  // fp8 modes: [rows_r] scale of each A row (routed groups only)
  const float *col_scale;  // fp8 modes: [E, N_r] scale of each B row
  int kb_r;            // row length of B_r when shorter than K_r: k wraps over B's columns
                       // (k-block at kk reads B columns kk % kb_r); 0 means K_r
  int lo_split;        // MODE_SCALE, bf16: > 0 stores v as hi = bf16(v) at column n and
                       // lo = bf16(v - hi) at column n + lo_split (a two-term bf16 split)
  int out_r_bf16;      // MODE_PLAIN, tensor-core kernels: routed rows stored as bf16 (else fp32)
  int out_f32;         // MODE_SCALE (single SM): z stored as fp32 (the fp32 configuration, whose
                       // operands are split bf16 terms; its gate/up is MODE_GATEUP_F32)
  int has_shared, T;
  const void *A_s;
  int lda_s;
  const void *B0_s, *B1_s;
  int N_s, K_s, piece_k, piece_rows;
  int b_rows_s;            // rows of the shared weight viewed as [b_rows_s, piece_k]
  void *out_s;
  int ldo_s;
  int kind;                // KernelKind of the launch (in-step stamps)
  // backward epilogues (GATEUP_RAW, SWIGLU_BWD): second half offset within a row of out / aux,
  // the h output and the g, u input (bf16)
  int half_r, half_s;
  void *out2_r, *out2_s;
  int ld2_r, ld2_s;
  const void *aux_r, *aux_s;
  const int32_t *aux_row0;  // [E] device: first row of each routed group in the blocked g, u
                            // buffer (group sizes rounded up to 64); the shared group starts at 0
  // groups along K (backward weight gradients)
  int kgroup;
  const int32_t *koff;     // [E+1] device: padded K offsets of the groups
  int kseg;                // K segments per group (kgroup)
  const int32_t *gorder;   // kgroup: [E] device, the group at each position of the tile list
                           // (longest K first); null: group order
  // kgroup with MN-major operands (mn != 0): A and B are row-major [rows, ld] matrices whose
  // rows are K; group g takes rows mn_row_a[g] + k of A and mn_row_b[g] + k of B for k < its
  // padded row count (koff[g+1] - koff[g]), once per segment s < kseg, segment s reading the
  // columns mn_col_a[s] + m of A and mn_col_b[s] + n of B (multiples of 64). The leading rows
  // beyond a group's own are zeros in one operand (the padded layout below) and, in the other,
  // rows of earlier groups or rows before row 0 (which the tensor map reads as zeros).
  int mn;
  const int32_t *mn_row_a, *mn_row_b;  // [E] device
  int mn_col_a[3], mn_col_b[3];
  int mn_lda, mn_ldb;                  // row lengths (elements)
  int mn_rows_a, mn_rows_b;            // row extents of the tensor maps
  // routed rows at padded positions, padding first: group g owns rows [aux_row0[g],
  // aux_row0[g+1]) (its row count rounded up to 64), zeros in the leading ones and its rows in
  // the trailing ones. SWIGLU_BWD (pad_out) writes out and out2 that way; a_row_end (non-null,
  // [E+1]) makes group g's A rows start at a_row_end[g+1] - rows (out rows stay at offsets[g])
  int pad_out;
  const int32_t *a_row_end;
};

// Tile list order: the shared group (its K may be several experts' widths: the longest tiles)
// first, then the routed groups, so that the last wave holds short tiles. Position o of the
// order is group group_at(p, o).
__device__ __forceinline__ int group_at(const GroupedGemm &p, int o) {
  if (!p.has_shared) return o;
  return o == 0 ? p.E : o - 1;
}

// Tile counts per group and their exclusive prefix (in tile-list order) in shared memory (all
// threads call).
__device__ __forceinline__ int build_tile_prefix(const GroupedGemm &p, int BM, int BN,
                                                 int *prefix, int *tmp) {
  const int G = p.E + p.has_shared;
  const int ntr = (p.N_r + BN - 1) / BN, nts = (p.N_s + BN - 1) / BN;
  for (int o = threadIdx.x; o < G; o += blockDim.x) {
    if (p.kgroup) {
      const int g = p.gorder ? p.gorder[o] : o;
      const int kg = p.kseg * (p.koff[g + 1] - p.koff[g]);
      prefix[o] = kg > 0 ? ((p.rows_r + BM - 1) / BM) * ntr : 0;
      continue;
    }
    const int g = group_at(p, o);
    const int rows = g < p.E ? (p.offsets[g + 1] - p.offsets[g]) : p.T;
    prefix[o] = ((rows + BM - 1) / BM) * (g < p.E ? ntr : nts);
  }
  __syncthreads();
  const int total = block_excl_scan_inplace(prefix, G, tmp);
  if (threadIdx.x == 0) prefix[G] = total;
  __syncthreads();
  return total;
}

struct TileInfo {
  int g, rows, m0, n0, N, K;
  int a_row0;    // first row of the group in A
  int out_row0;  // first row of the group in out
  int kofs;      // first column of the group in A and B (groups along K)
};

__device__ __forceinline__ TileInfo decode_tile(const GroupedGemm &p, int tile,
                                                const int *prefix, int BM, int BN) {
  const int G = p.E + p.has_shared;
  int lo = 0, hi = G - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= tile) lo = mid;
    else hi = mid - 1;
  }
  TileInfo ti;
  const int local = tile - prefix[lo];
  lo = p.kgroup ? (p.gorder ? p.gorder[lo] : lo) : group_at(p, lo);  // list position -> group
  ti.g = lo;
  const bool routed = lo < p.E;
  ti.N = routed ? p.N_r : p.N_s;
  ti.K = routed ? p.K_r : p.K_s;
  const int nt = (ti.N + BN - 1) / BN;
  ti.m0 = (local / nt) * BM;
  ti.n0 = (local % nt) * BN;
  ti.kofs = 0;
  if (p.kgroup) {
    ti.a_row0 = 0;
    ti.rows = p.rows_r;
    ti.out_row0 = lo * p.rows_r;
    ti.kofs = p.kseg * p.koff[lo];
    ti.K = p.kseg * p.koff[lo + 1] - ti.kofs;
    return ti;
  }
  if (routed) {
    ti.out_row0 = p.offsets[lo];
    ti.rows = p.offsets[lo + 1] - ti.out_row0;
    ti.a_row0 = p.a_row_end ? p.a_row_end[lo + 1] - ti.rows : ti.out_row0;
  } else {
    ti.a_row0 = 0;
    ti.rows = p.T;
    ti.out_row0 = 0;
  }
  return ti;
}

__device__ __forceinline__ float silu_f(float z) { return z / (1.0f + expf(-z)); }

}  // namespace moe

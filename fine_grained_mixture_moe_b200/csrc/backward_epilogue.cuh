// Epilogues of the CTA-pair GEMM (gemm_tc2.cuh) used only by the backward of the SwiGLU experts:
//   GATEUP_RAW  g = x W_g^T and u = x W_u^T (fp32), the forward's gate/up product recomputed
//   SWIGLU_BWD  dh = dY W_d with the SwiGLU derivative: dg = dh u silu'(g), du = dh silu(g) and
//               h = silu(g) u, each as two bf16 terms (v = hi + lo, hi = bf16(v), lo = bf16(v - hi))
// (Vertex AGI research page, "Training stack": the layer is trained with recomputation of the
// forward activations, which g and u are.)
//
// g and u pass between the two launches in a blocked buffer: blocks of 32 rows x 32 columns of
// fp32 (4 KB), g's block and u's block of the same rows and columns side by side (8 KB), in the
// order [row block][column block][g, u]. A group's rows start at a row aux_row0[g] (routed
// groups, padded to 64 rows) or 0 (the shared group). Inside a block, row r's 16-byte piece i
// (columns 4i .. 4i+3) sits at byte r * 128 + (i ^ (r & 7)) * 16: one lane per row reads its row
// from shared memory without bank conflicts, and the whole 8 KB arrives with one bulk copy.
#pragma once
#include "gemm_tc.cuh"

namespace moe {

constexpr int GU_BLOCK_FLOATS = 32 * 32;      // one 32 x 32 fp32 block
constexpr int GU_PAIR_BYTES = 2 * 4 * GU_BLOCK_FLOATS;  // g block + u block

// The g block of rows rbase .. rbase + 31 (group-local, rbase a multiple of 32) and columns
// col .. col + 31 of a tile's group in the blocked buffer `gu` (out for GATEUP_RAW, aux for
// SWIGLU_BWD); the u block follows it.
__device__ __forceinline__ float *gu_pair_block(const GroupedGemm &p, const TileInfo &ti,
                                                bool routed, const void *gu, int rbase, int col) {
  float *aux = (float *)gu;
  const int hf = routed ? p.half_r : p.half_s;
  const int row = (routed ? p.aux_row0[ti.g] : 0) + rbase;
  return aux + ((size_t)(row >> 5) * (hf >> 5) + (col >> 5)) * (2 * GU_BLOCK_FLOATS);
}

// GATEUP_RAW: the lane's row of g (r0) and u (r1), 32 columns each, staged per warp in the
// block's own layout (4 KB at stg) and copied to the block as 8 coalesced 512-byte stores.
__device__ __forceinline__ void gateup_raw_chunk(const uint32_t (&r0)[32], const uint32_t (&r1)[32],
                                                 unsigned char *stg, float *blk, int lane) {
#pragma unroll 1
  for (int part = 0; part < 2; ++part) {
    const uint32_t *rv = part ? r1 : r0;
#pragma unroll
    for (int i = 0; i < 8; ++i)
      *(uint4 *)(stg + lane * 128 + ((i ^ (lane & 7)) << 4)) =
          make_uint4(rv[4 * i], rv[4 * i + 1], rv[4 * i + 2], rv[4 * i + 3]);
    __syncwarp();
    uint4 *dst = (uint4 *)(blk + part * GU_BLOCK_FLOATS);
#pragma unroll
    for (int j = 0; j < 8; ++j) dst[32 * j + lane] = ((const uint4 *)stg)[32 * j + lane];
    __syncwarp();
  }
}

// SWIGLU_BWD: one epilogue warp's feed of g and u blocks into its 8 KB of shared memory, one
// block pair in flight at a time (issued one chunk ahead, and for a tile's first chunk before
// the accumulator is ready). Lane 0 issues; every wait is bounded.
struct GuFeed {
  uint32_t buf, bar;
  uint32_t phase;
  bool pending;
  __device__ __forceinline__ void issue(const float *src, int lane) {
    if (lane == 0) {
      mbar_expect_tx(bar, GU_PAIR_BYTES);
      bulk_load_1d(buf, src, GU_PAIR_BYTES, bar);
    }
    pending = true;
  }
  __device__ __forceinline__ bool wait(volatile int *abort_flag, uint64_t limit) {
    bool ok = true;
    if ((threadIdx.x & 31) == 0) ok = mbar_wait(bar, phase, abort_flag, limit, INFO_WAIT_TMA_FULL);
    ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    if (ok) {
      phase ^= 1u;
      pending = false;
    }
    return ok;
  }
  // before leaving the kernel: no copy may still be writing this CTA's shared memory
  __device__ __forceinline__ void drain(uint64_t limit) {
    if (!pending) return;
    volatile int never = 0;
    if ((threadIdx.x & 31) == 0) mbar_wait(bar, phase, &never, limit, INFO_WAIT_DRAIN);
    __syncwarp();
    pending = false;
  }
};

// SWIGLU_BWD: the lane's row of dh (r0, 32 columns) with g and u of the same row and columns
// from the warp's block pair in shared memory; writes dg, du and h as hi + lo bf16 terms to
// o[col..] (dg_hi), o + hf (du_hi), o + 2 hf (dg_lo), o + 3 hf (du_lo), o2 (h_hi), o2 + hf (h_lo),
// 16 columns (32 bytes, one sector) per store. The caller has waited for the block pair; the
// shared memory is released (the next pair may be issued) once g and u are in registers.
// o, o2 and 2 hf bytes are multiples of 32 bytes. A row past the group (!row_ok) stores nothing,
// or zeros in all six outputs when zero_row is set (the padding rows of a padded layout).
template <typename Issue>
__device__ __forceinline__ void swiglu_bwd_chunk(const uint32_t (&r0)[32], const unsigned char *buf,
                                                 int lane, bool row_ok, bool zero_row,
                                                 __nv_bfloat16 *o, __nv_bfloat16 *o2, int hf,
                                                 Issue issue_next) {
  float4 gq[8], uq[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int off = lane * 128 + ((i ^ (lane & 7)) << 4);
    gq[i] = *(const float4 *)(buf + off);
    uq[i] = *(const float4 *)(buf + 4 * GU_BLOCK_FLOATS + off);
  }
  // generic reads of the buffer ordered before the bulk copy that overwrites it
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  __syncwarp();
  issue_next();
  if (!row_ok) {
    if (zero_row) {
      const uint32_t z[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
#pragma unroll
      for (int h16 = 0; h16 < 2; ++h16) {
#pragma unroll
        for (int s4 = 0; s4 < 4; ++s4) st_global_32B(o + s4 * hf + 16 * h16, z);
        st_global_32B(o2 + 16 * h16, z);
        st_global_32B(o2 + hf + 16 * h16, z);
      }
    }
    return;
  }
#pragma unroll
  for (int h16 = 0; h16 < 2; ++h16) {
    uint32_t dgh[8], dgl[8], duh[8], dul[8], hh[8], hl[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {  // columns 16 h16 + 2i, + 1
      const float4 gp = gq[4 * h16 + (i >> 1)], up = uq[4 * h16 + (i >> 1)];
      const float g2[2] = {(i & 1) ? gp.z : gp.x, (i & 1) ? gp.w : gp.y};
      const float u2[2] = {(i & 1) ? up.z : up.x, (i & 1) ? up.w : up.y};
      float dgv[2], duv[2], hv[2];
#pragma unroll
      for (int z = 0; z < 2; ++z) {
        const float g = g2[z], u = u2[z], dh = __uint_as_float(r0[16 * h16 + 2 * i + z]);
        const float sg = 1.0f / (1.0f + __expf(-g)), si = g * sg;
        dgv[z] = dh * u * sg * (1.0f + g * (1.0f - sg));
        duv[z] = dh * si;
        hv[z] = si * u;
      }
      const __nv_bfloat162 a = __floats2bfloat162_rn(dgv[0], dgv[1]);
      const __nv_bfloat162 b = __floats2bfloat162_rn(duv[0], duv[1]);
      const __nv_bfloat162 h = __floats2bfloat162_rn(hv[0], hv[1]);
      const float2 af = __bfloat1622float2(a), bfv = __bfloat1622float2(b),
                   hf2 = __bfloat1622float2(h);
      const __nv_bfloat162 al = __floats2bfloat162_rn(dgv[0] - af.x, dgv[1] - af.y);
      const __nv_bfloat162 bl = __floats2bfloat162_rn(duv[0] - bfv.x, duv[1] - bfv.y);
      const __nv_bfloat162 hlo = __floats2bfloat162_rn(hv[0] - hf2.x, hv[1] - hf2.y);
      dgh[i] = *(const uint32_t *)&a;
      duh[i] = *(const uint32_t *)&b;
      hh[i] = *(const uint32_t *)&h;
      dgl[i] = *(const uint32_t *)&al;
      dul[i] = *(const uint32_t *)&bl;
      hl[i] = *(const uint32_t *)&hlo;
    }
    st_global_32B(o + 16 * h16, dgh);
    st_global_32B(o + hf + 16 * h16, duh);
    st_global_32B(o + 2 * hf + 16 * h16, dgl);
    st_global_32B(o + 3 * hf + 16 * h16, dul);
    st_global_32B(o2 + 16 * h16, hh);
    st_global_32B(o2 + hf + 16 * h16, hl);
  }
}

}  // namespace moe

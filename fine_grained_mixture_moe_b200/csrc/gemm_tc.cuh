// bf16 grouped expert GEMM on the 5th-generation tensor cores (sm_100a), single-SM form.
//
// It serves the low-rank V projection (SCALE, N = rank); the PLAIN form is kept for narrow
// outputs. The SwiGLU gate/up product and the down and low-rank U projections run on CTA pairs
// (gemm_tc2.cuh), which share this file's PTX wrappers, tensor maps and epilogue conventions.
//
// One persistent CTA per SM walks a device-side tile list built from the group offsets
// (Moonfrost's stacked (E, hidden, ffn) expert tensors, here indexed by expert on the device so
// the host never sees a count). Per CTA: 10 warps.
//   warp 0  TMA producer: A tile [128 x 64] and B tile [BN x 64] per k-block into a STAGES-deep
//           shared-memory ring (128-byte swizzle, K-major), completion on `full[s]`.
//   warp 1  TMEM owner and MMA issuer: one thread issues tcgen05.mma (kind::f16, bf16 x bf16 ->
//           fp32, M=128, N=BN, K=16) into one of two TMEM accumulators; tcgen05.commit frees the
//           smem stage (`empty[s]`) and, per tile, publishes the accumulator (`acc_full[b]`).
//   warps 2-9 epilogue: two warps per TMEM lane quarter, each taking half of the tile's columns;
//           tcgen05.ld (32 lanes x 32 columns per load) -> scale -> bf16 (the low-rank
//           projection, the next GEMM's operand) or bf16 / fp32 expert outputs -> global; then
//           `acc_empty[b]`, so the next tile's MMAs overlap this epilogue.
// Every wait is bounded (global timer); on expiry the CTA records MOE_ERR_TIMEOUT, drains what
// it has in flight (again bounded), frees its TMEM and returns.
#pragma once
#include <cuda.h>
#include "fp8.cuh"
#include "grouped.cuh"

namespace moe {

constexpr int TC_BM = 128;
constexpr int TC_BK = 64;  // one 128-byte swizzle atom of bf16
constexpr int TC_EPI_WARPS = 8;  // two per TMEM lane quarter, each taking half the columns
constexpr int TC_THREADS = 64 + 32 * TC_EPI_WARPS;

struct TcMaps {
  CUtensorMap a_r, a_s, b0_r, b1_r, b0_s, b1_s;
};

struct TcParams {
  TcMaps maps;
  GroupedGemm p;
  int stages;  // CTA-pair kernel: operand pipeline depth chosen from the group count
  int kpb;     // CTA-pair kernel: K-blocks per stage, 1 or 2 (2: 3-D tensor maps whose box spans
               // two K-blocks, one A and one B copy per two K-blocks)
};

template <int MODE, int BN> struct TcCfg {
  static_assert(MODE == MODE_PLAIN || MODE == MODE_SCALE || MODE == MODE_SCALE_FP8,
                "single-SM form: down and low-rank products (gate/up runs on CTA pairs)");
  static constexpr int NB = 1;                                    // B tiles per stage
  static constexpr int BK = mode_bk(MODE);                        // K elements per stage
  static constexpr int A_BYTES = TC_BM * 128;                     // 16 KB: 128-byte rows
  static constexpr int B_BYTES = BN * 128;
  static constexpr int STAGE_BYTES = A_BYTES + NB * B_BYTES;
  // PLAIN and SCALE: per-warp fp32 staging (SCALE stores fp32 z with out_f32); SCALE_FP8: the
  // row maxima of the two column halves, per accumulator buffer [2][2][128]
  static constexpr bool F32_OUT = MODE == MODE_PLAIN;
  static constexpr int STG_BYTES = MODE == MODE_PLAIN || MODE == MODE_SCALE ? TC_EPI_WARPS * 4096
                                   : MODE == MODE_SCALE_FP8 ? 2 * 2 * TC_BM * 4 : 0;
  static constexpr int STAGES = (200 * 1024 - STG_BYTES) / STAGE_BYTES > 8
                                    ? 8 : (200 * 1024 - STG_BYTES) / STAGE_BYTES;
  static constexpr int ACC_COLS = NB * BN;                        // fp32 columns per buffer
  static constexpr int TMEM_COLS = (2 * ACC_COLS <= 32) ? 32 : (2 * ACC_COLS <= 64) ? 64
                                   : (2 * ACC_COLS <= 128) ? 128 : (2 * ACC_COLS <= 256) ? 256 : 512;
  static_assert(2 * ACC_COLS <= 512, "TMEM holds 512 columns");
  static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "UMMA N for M=128, epilogue in 32s");
  static constexpr int MMA_N = NB * BN;
  static_assert(MMA_N <= 256, "UMMA N <= 256");
  // instruction descriptor: D fp32, A/B bf16 (kind::f16) or E4M3 (kind::f8f6f4, format 0), both
  // K-major, N>>3 at bit 17, M>>4 at bit 24
  static constexpr uint32_t IDESC = (1u << 4) | (mode_fp8(MODE) ? 0u : (1u << 7) | (1u << 10)) |
                                    ((uint32_t)(MMA_N >> 3) << 17) | ((uint32_t)(TC_BM >> 4) << 24);
};

// ---------------------------------------------------------------- PTX wrappers
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int c0, int c1,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"((uint64_t)map), "r"(c0), "r"(c1), "r"(bar)
      : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// The same with 8-bit operands (both E4M3 here): K = 32 elements (32 bytes) per instruction.
__device__ __forceinline__ void tc_mma_f8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row core groups 1024 B apart.
__device__ __forceinline__ uint64_t make_sdesc(uint32_t saddr) {
  uint64_t d = (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)1 << 16;             // leading byte offset (unused for swizzled K-major)
  d |= (uint64_t)(1024 >> 4) << 32;   // stride byte offset
  d |= (uint64_t)1 << 46;             // descriptor version (sm_100)
  d |= (uint64_t)2 << 61;             // SWIZZLE_128B
  return d;
}
// The same for an MN-major operand (rows of the tile are K): 64 M (or N) elements per 128-byte
// row, K rows in 8-row groups of 1024 bytes (stride byte offset), and the next 64 elements of M
// `lbo` bytes further (leading byte offset).
__device__ __forceinline__ uint64_t make_sdesc_mn(uint32_t saddr, uint32_t lbo) {
  uint64_t d = (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;  // leading byte offset: the next 64 of M / N
  d |= (uint64_t)(1024 >> 4) << 32;             // stride byte offset: the next 8 rows of K
  d |= (uint64_t)1 << 46;                       // descriptor version (sm_100)
  d |= (uint64_t)2 << 61;                       // SWIZZLE_128B
  return d;
}
// Instruction-descriptor bits of MN-major A and B (kind::f16).
constexpr uint32_t IDESC_MN_MAJOR = (1u << 15) | (1u << 16);
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

template <int MODE, int BN>
__host__ __device__ constexpr size_t tc_smem_bytes(int G) {
  using C = TcCfg<MODE, BN>;
  return 1024 /*alignment slack*/ + (size_t)C::STAGES * C::STAGE_BYTES + C::STG_BYTES +
         256 /*barriers*/ + (size_t)(G + 1 + TC_THREADS / 32 + 1) * sizeof(int);
}

template <int MODE, int BN>
__global__ void __launch_bounds__(TC_THREADS, 1) gemm_tc_kernel(const __grid_constant__ TcParams P) {
  using C = TcCfg<MODE, BN>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const GroupedGemm &p = P.p;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = p.E + p.has_shared;

  // carve shared memory (stages must be 1024-byte aligned for the 128-byte swizzle)
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t pad = ((raw + 1023u) & ~1023u) - raw;
  unsigned char *base = smem_raw + pad;
  unsigned char *stages = base;
  unsigned char *stg_all = base + (size_t)C::STAGES * C::STAGE_BYTES;  // [8 warps][4 KB]
  uint64_t *bars = (uint64_t *)(stg_all + C::STG_BYTES);
  // bars: full[STAGES], empty[STAGES], acc_full[2], acc_empty[2], drain
  uint32_t *tmem_slot = (uint32_t *)(bars + 2 * C::STAGES + 5);
  volatile int *abort_flag = (volatile int *)(tmem_slot + 1);
  int *prefix = (int *)(stg_all + C::STG_BYTES + 256);
  int *scan_tmp = prefix + G + 1;

  auto full_bar = [&](int s) { return smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + C::STAGES + s); };
  auto accf_bar = [&](int b) { return smem_u32(bars + 2 * C::STAGES + b); };
  auto acce_bar = [&](int b) { return smem_u32(bars + 2 * C::STAGES + 2 + b); };
  const uint32_t drain_bar = smem_u32(bars + 2 * C::STAGES + 4);

  if (tid == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(accf_bar(b), 1);
      mbar_init(acce_bar(b), TC_EPI_WARPS);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"((uint32_t)C::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (warp == 0 && lane == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&P.maps.a_r) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)&P.maps.b0_r) : "memory");
  }
  const KernelStamp stamp(p.kind);
  griddep_wait();
  stamp.started();
  griddep_launch();
  const int total = build_tile_prefix(p, TC_BM, BN, prefix, scan_tmp);  // contains __syncthreads
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint64_t limit = g_wait_limit_ns;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int issued_parity[8];
      bool issued[8];
      for (int s = 0; s < 8; ++s) { issued[s] = false; issued_parity[s] = 0; }
      bool ok = true;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        const TileInfo ti = decode_tile(p, tile, prefix, TC_BM, BN);
        const bool routed = ti.g < p.E;
        const CUtensorMap *ma = routed ? &P.maps.a_r : &P.maps.a_s;
        const CUtensorMap *mb0 = routed ? &P.maps.b0_r : &P.maps.b0_s;
        const int a_row = ti.a_row0 + ti.m0;
        const int nk = (ti.K + C::BK - 1) / C::BK;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, limit, INFO_WAIT_MMA_EMPTY)) {
            ok = false;
            break;
          }
          const uint32_t sA = smem_u32(stages + (size_t)stage * C::STAGE_BYTES);
          const uint32_t sB0 = sA + C::A_BYTES;
          mbar_expect_tx(full_bar(stage), C::STAGE_BYTES);
          const int kk = kb * C::BK;
          int b_row, b_col;
          if (routed) {
            b_row = ti.g * ti.N + ti.n0;
            b_col = p.kb_r ? kk % p.kb_r : kk;
          } else {
            const int piece = kk / p.piece_k;
            b_row = piece * p.piece_rows + ti.n0;
            b_col = kk - piece * p.piece_k;
          }
          tma_load_2d(sA, ma, kk, a_row, full_bar(stage));
          tma_load_2d(sB0, mb0, b_col, b_row, full_bar(stage));
          issued[stage] = true;
          issued_parity[stage] = (int)phase;
          if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        // drain: every issued load completes its barrier phase before shared memory goes away
        for (int s = 0; s < C::STAGES; ++s)
          if (issued[s]) {
            volatile int never = 0;
            mbar_wait(full_bar(s), (uint32_t)issued_parity[s], &never, limit, INFO_WAIT_DRAIN);
          }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true, any = false;
      for (int tile = blockIdx.x; tile < total && ok; tile += gridDim.x) {
        const TileInfo ti = decode_tile(p, tile, prefix, TC_BM, BN);
        const int nk = (ti.K + C::BK - 1) / C::BK;
        if (!mbar_wait(acce_bar(acc), acc_phase ^ 1u, abort_flag, limit, INFO_WAIT_ACC_EMPTY)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d0 = tmem_base + (uint32_t)(acc * C::ACC_COLS);
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(full_bar(stage), phase, abort_flag, limit, INFO_WAIT_TMA_FULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sA = smem_u32(stages + (size_t)stage * C::STAGE_BYTES);
          const uint32_t sB0 = sA + C::A_BYTES;
#pragma unroll
          for (int k16 = 0; k16 < 4; ++k16) {  // 32 bytes of K per instruction
            const uint64_t ad = make_sdesc(sA + k16 * 32);
            const uint64_t bd0 = make_sdesc(sB0 + k16 * 32);
            const uint32_t accum = (kb > 0 || k16 > 0) ? 1u : 0u;
            if (mode_fp8(MODE)) tc_mma_f8(d0, ad, bd0, C::IDESC, accum);
            else tc_mma(d0, ad, bd0, C::IDESC, accum);
          }
          any = true;
          tc_commit(empty_bar(stage));
          if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit(accf_bar(acc));
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      if (!ok && any) {
        // wait until every MMA issued so far has completed before TMEM is released
        tc_commit(drain_bar);
        volatile int never = 0;
        mbar_wait(drain_bar, 0u, &never, limit, INFO_WAIT_DRAIN);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..9)
    const int q = warp & 3;                            // TMEM lane quarter this warp may access
    const int half = (warp - 2) >> 2;                  // which half of the tile's columns
    const int cbeg = half * (BN / 2), cend = cbeg + BN / 2;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < total; tile += gridDim.x) {
      const TileInfo ti = decode_tile(p, tile, prefix, TC_BM, BN);
      const bool routed = ti.g < p.E;
      bool ok = true;
      if (lane == 0)
        ok = mbar_wait(accf_bar(acc), acc_phase, abort_flag, limit, INFO_WAIT_ACC_FULL);
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      tc_fence_after();
      const int row = ti.m0 + q * 32 + lane;
      const bool row_ok = row < ti.rows;
      void *out = routed ? p.out_r : p.out_s;
      const int ldo = routed ? p.ldo_r : p.ldo_s;
      const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * C::ACC_COLS);
      // fp32 outputs use a staged write-back: the warp's 32 rows x 32 columns
      // go to a private 4 KB buffer (16-byte chunk j of row r stored at chunk j ^ (r & 7), so
      // both the row-wise writes and the column-wise reads are conflict-free), then leave as 32
      // row stores of 128 contiguous bytes each instead of 32-row scattered 16-byte stores.
      unsigned char *stg = stg_all + (warp - 2) * 4096;
      if (MODE == MODE_SCALE_FP8) {
        // z = sum * (row scale) * (V row scale) * s, then the row's E4M3 codes and scale (the
        // tile is the whole row: BN = N). Pass 1: each of the two warps of this lane quarter
        // takes the maximum |z| over its half of the row; they meet at a named barrier (both
        // passed the same accumulator wait, so both arrive); pass 2 recomputes z, converts and
        // stores 32 codes per 32-byte store. rs = 0 on rows past the group: their z is not used.
        float *s_am = (float *)stg_all;
        const float rs = row_ok ? __ldg(p.row_scale + ti.a_row0 + row) : 0.0f;
        const float4 *cs = (const float4 *)(p.col_scale + (size_t)ti.g * ti.N);
        const float4 *ss = (const float4 *)(p.scale + (size_t)ti.g * ti.N);
        auto zchunk = [&](int c, float (&z)[32]) {
          uint32_t r0[32];
          __syncwarp();  // the collective TMEM load runs converged
          tmem_ld32(tbase + c, r0);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 v = __ldg(cs + c / 4 + i), w = __ldg(ss + c / 4 + i);
            z[4 * i] = __uint_as_float(r0[4 * i]) * rs * v.x * w.x;
            z[4 * i + 1] = __uint_as_float(r0[4 * i + 1]) * rs * v.y * w.y;
            z[4 * i + 2] = __uint_as_float(r0[4 * i + 2]) * rs * v.z * w.z;
            z[4 * i + 3] = __uint_as_float(r0[4 * i + 3]) * rs * v.w * w.w;
          }
        };
        float am = 0.0f;
#pragma unroll 1
        for (int c = cbeg; c < cend; c += 32) {
          float z[32];
          zchunk(c, z);
#pragma unroll
          for (int i = 0; i < 32; ++i) am = fmaxf(am, fabsf(z[i]));
        }
        s_am[(acc * 2 + half) * TC_BM + q * 32 + lane] = am;
        asm volatile("bar.sync %0, 64;" ::"r"(1 + q) : "memory");
        am = fmaxf(s_am[(acc * 2) * TC_BM + q * 32 + lane], s_am[(acc * 2 + 1) * TC_BM + q * 32 + lane]);
        const float sc = am > 0.0f ? __fdiv_rn(am, E4M3_MAX) : 1.0f;
        if (half == 0 && row_ok) ((float *)p.out2_r)[ti.a_row0 + row] = sc;
#pragma unroll 1
        for (int c = cbeg; c < cend; c += 32) {  // warp-uniform: tcgen05.ld is collective
          float z[32];
          zchunk(c, z);
          if (row_ok) {  // rows past the group: no conversion, no store
            uint32_t w8[8];
#pragma unroll
            for (int i = 0; i < 8; ++i)
              w8[i] = e4m3_code(__fdiv_rn(z[4 * i], sc)) |
                      (e4m3_code(__fdiv_rn(z[4 * i + 1], sc)) << 8) |
                      (e4m3_code(__fdiv_rn(z[4 * i + 2], sc)) << 16) |
                      (e4m3_code(__fdiv_rn(z[4 * i + 3], sc)) << 24);
            st_global_32B((uint8_t *)out + (size_t)(ti.a_row0 + row) * ldo + ti.n0 + c, w8);
          }
        }
      }
      constexpr int SUB = C::F32_OUT ? 1 : 2;  // 32-column TMEM loads per block
#pragma unroll 1
      for (int c = cbeg; c < (MODE == MODE_SCALE_FP8 ? cbeg : cend); c += 32 * SUB) {
        if (MODE == MODE_SCALE && p.out_f32) {
          // fp32 z = sum * s, SUB 32-column blocks, each staged per warp and written as 32
          // coalesced 128-byte row stores
#pragma unroll 1
          for (int sub = 0; sub < SUB && c + 32 * sub < cend; ++sub) {  // this warp's columns only
            uint32_t r0[32];
            tmem_ld32(tbase + c + 32 * sub, r0);
            tmem_wait_ld();
            const int col = ti.n0 + c + 32 * sub;
            if (col < ti.N) {
              const float *sc = p.scale + (size_t)ti.g * ti.N + col;
#pragma unroll
              for (int i = 0; i < 32; ++i)
                r0[i] = __float_as_uint(__uint_as_float(r0[i]) * __ldg(sc + i));
            }
#pragma unroll
            for (int i = 0; i < 8; ++i)
              *(uint4 *)(stg + lane * 128 + ((i ^ (lane & 7)) << 4)) =
                  make_uint4(r0[4 * i], r0[4 * i + 1], r0[4 * i + 2], r0[4 * i + 3]);
            __syncwarp();
            if (col < ti.N) {
              const int rbase = ti.m0 + q * 32;
              const int nrows = min(32, ti.rows - rbase);
              unsigned char *obase = (unsigned char *)out + ((size_t)(ti.a_row0 + rbase) * ldo + col) * 4;
              const size_t row_bytes = (size_t)ldo * 4;
              for (int rr = 0; rr < nrows; ++rr) {
                const uint32_t v = *(const uint32_t *)(stg + rr * 128 +
                                                       (((lane >> 2) ^ (rr & 7)) << 4) + ((lane & 3) << 2));
                *(uint32_t *)(obase + rr * row_bytes + lane * 4) = v;
              }
            }
            __syncwarp();
          }
          continue;
        }
        if (MODE == MODE_SCALE) {
          // bf16 low-rank projection: each lane already writes 64 contiguous bytes of its row, so
          // they go out directly
#pragma unroll
          for (int sub = 0; sub < SUB; ++sub) {
            uint32_t r0[32];
            tmem_ld32(tbase + c + 32 * sub, r0);
            tmem_wait_ld();
            const int col = ti.n0 + c + 32 * sub;
            if (row_ok && col < ti.N) {
              uint4 pk[4];
              __nv_bfloat162 *h = (__nv_bfloat162 *)pk;
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const float g0 = __uint_as_float(r0[2 * i]), g1 = __uint_as_float(r0[2 * i + 1]);
                const float v0 = g0 * __ldg(p.scale + (size_t)ti.g * ti.N + col + 2 * i);
                const float v1 = g1 * __ldg(p.scale + (size_t)ti.g * ti.N + col + 2 * i + 1);
                h[i] = __floats2bfloat162_rn(v0, v1);
              }
              uint4 *dst = (uint4 *)((__nv_bfloat16 *)out + (size_t)(ti.a_row0 + row) * ldo + col);
#pragma unroll
              for (int i = 0; i < 4; ++i) dst[i] = pk[i];
              if (MODE == MODE_SCALE && p.lo_split > 0) {
                // second term: the rounding residual v - hi, exact in fp32, rounded to bf16
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                  const float v0 = __uint_as_float(r0[2 * i]) * __ldg(p.scale + (size_t)ti.g * ti.N + col + 2 * i);
                  const float v1 = __uint_as_float(r0[2 * i + 1]) * __ldg(p.scale + (size_t)ti.g * ti.N + col + 2 * i + 1);
                  const float2 hf = __bfloat1622float2(h[i]);
                  h[i] = __floats2bfloat162_rn(v0 - hf.x, v1 - hf.y);
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) dst[p.lo_split / 8 + i] = pk[i];
              }
            }
          }
          continue;
        }
        if (routed && p.out_r_bf16) {
          // routed expert outputs in bf16: 64 contiguous bytes of the lane's row, stored directly
          uint32_t r0[32];
          tmem_ld32(tbase + c, r0);
          tmem_wait_ld();
          const int col = ti.n0 + c;
          if (row_ok && col < ti.N) {
            uint4 pk[4];
            __nv_bfloat162 *h = (__nv_bfloat162 *)pk;
#pragma unroll
            for (int i = 0; i < 16; ++i)
              h[i] = __floats2bfloat162_rn(__uint_as_float(r0[2 * i]), __uint_as_float(r0[2 * i + 1]));
            uint4 *dst = (uint4 *)((__nv_bfloat16 *)out + (size_t)(ti.a_row0 + row) * ldo + col);
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = pk[i];
          }
          continue;
        }
        {
          uint32_t r0[32];
          tmem_ld32(tbase + c, r0);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 8; ++i)
            *(uint4 *)(stg + lane * 128 + ((i ^ (lane & 7)) << 4)) =
                make_uint4(r0[4 * i], r0[4 * i + 1], r0[4 * i + 2], r0[4 * i + 3]);
        }
        __syncwarp();
        const int col = ti.n0 + c;
        if (col < ti.N) {
          const int rbase = ti.m0 + q * 32;
          const int nrows = min(32, ti.rows - rbase);
          unsigned char *obase = (unsigned char *)out + ((size_t)(ti.a_row0 + rbase) * ldo + col) * 4;
          const size_t row_bytes = (size_t)ldo * 4;
          for (int rr = 0; rr < nrows; ++rr) {
            const uint32_t v = *(const uint32_t *)(stg + rr * 128 + (((lane >> 2) ^ (rr & 7)) << 4) +
                                                   ((lane & 3) << 2));
            *(uint32_t *)(obase + rr * row_bytes + lane * 4) = v;
          }
        }
        __syncwarp();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acce_bar(acc));
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"((uint32_t)C::TMEM_COLS)
                 : "memory");
  }
}

}  // namespace moe

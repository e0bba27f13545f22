// bf16 grouped expert GEMM on CTA pairs (tcgen05 .cta_group::2, sm_100a).
//
// Same grouped problem, tile list and epilogues as gemm_tc.cuh, but each tile is 256 rows and is
// computed by a cluster of two CTAs on two SMs: CTA r loads rows [128r, 128r+128) of the A tile
// and half of the B tile (GATEUP: CTA 0 the gate rows, CTA 1 the up rows of the same 128 output
// columns; PLAIN: rows [128r, 128r+128) of a 256-column weight tile) into its own shared memory.
// The leader (CTA 0) issues one M=256, N=256, K=16 MMA per step that reads both CTAs' tiles
// and leaves rows [128r, 128r+128) of the fp32 accumulator in CTA r's TMEM. So each SM ingests
// 32 KB per 64-wide k-block instead of 48 KB for the same tensor work.
// Synchronisation: both CTAs' TMA loads complete on the leader's `full` barrier (the leader
// expects both CTAs' bytes); the leader's commits multicast to both CTAs' `empty` and
// `acc_full` barriers; all sixteen epilogue warps arrive on the leader's `acc_empty`. No TMA
// multicast is used. All waits are bounded as in gemm_tc.cuh.
#pragma once
#include "backward_epilogue.cuh"
#include "gemm_tc.cuh"

namespace moe {

constexpr int TC2_BM = 256;  // rows per tile (128 per CTA)

// TMA load into this CTA's shared memory whose completion is counted on the leader CTA's barrier
// (same shared-memory offset in CTA 0: the CTA-rank bit of the cluster address cleared).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap *map, int c0,
                                                 int c1, uint32_t bar_local) {
  const uint32_t bar0 = bar_local & 0xFEFFFFFFu;
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"((uint64_t)map), "r"(c0), "r"(c1), "r"(bar0)
      : "memory");
}
// The same with a 3-D box {64 columns, rows, 2 K-blocks}: two K-blocks' tiles, one after the other.
__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const CUtensorMap *map, int c0,
                                                 int c1, int c2, uint32_t bar_local) {
  const uint32_t bar0 = bar_local & 0xFEFFFFFFu;
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst),
      "l"((uint64_t)map), "r"(c0), "r"(c1), "r"(c2), "r"(bar0)
      : "memory");
}
__device__ __forceinline__ void tc2_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                        uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
__device__ __forceinline__ void tc2_mma_f8(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive once on the barrier at this shared offset in both CTAs of the pair when all prior
// tcgen05 operations of the issuing thread complete.
__device__ __forceinline__ void tc2_commit_both(uint32_t bar) {
  const uint16_t mask = 0x3;
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(bar),
      "h"(mask)
      : "memory");
}
// Relaxed: the arrival only has to follow this thread's completed TMEM reads (tcgen05.wait::ld
// precedes it in program order, and the MMA that may overwrite those columns is issued only after
// the arrival is observed). A release here would also wait for every global store the epilogue
// warp has in flight.
__device__ __forceinline__ void mbar_arrive_cta0(uint32_t bar_local) {
  asm volatile(
      "{\n\t.reg .b32 ra;\n\t"
      "mapa.shared::cluster.u32 ra, %0, 0;\n\t"
      "mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [ra];\n\t}" ::"r"(bar_local)
      : "memory");
}

// Modes whose B tile is two weights (gate rows in CTA 0, up rows in CTA 1).
__host__ __device__ constexpr bool tc2_two_b(int mode) {
  return mode == MODE_GATEUP || mode == MODE_GATEUP_RAW || mode == MODE_GATEUP_F32;
}

template <int MODE> struct Tc2Cfg {
  static_assert(MODE == MODE_GATEUP || MODE == MODE_PLAIN || MODE == MODE_GATEUP_RAW ||
                    MODE == MODE_SWIGLU_BWD || MODE == MODE_PLAIN_FP8 || MODE == MODE_GATEUP_F32,
                "pair kernel modes");
  static constexpr int BN = tc2_two_b(MODE) ? 128 : 256;  // output columns per tile
  static constexpr int MMA_N = 256;                           // accumulator columns
  static constexpr int BK = mode_bk(MODE);                    // K elements per stage
  static constexpr int A_BYTES = 128 * 128;                   // this CTA's 128 rows (128 B each)
  static constexpr int B_BYTES = 128 * 128;                   // this CTA's half of B
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;       // 32 KB
  // per-warp epilogue staging: 4 KB, or (SWIGLU_BWD) 8 KB for a g, u block pair and, after
  // all warps' buffers, one mbarrier per warp for its bulk copies
  static constexpr int STG_WARP = MODE == MODE_SWIGLU_BWD ? GU_PAIR_BYTES : 4096;
  static constexpr int STG_BYTES =
      TC_EPI_WARPS * STG_WARP + (MODE == MODE_SWIGLU_BWD ? TC_EPI_WARPS * 8 : 0);
  static constexpr int MAX_STAGES = 8;
  static constexpr int ACC_COLS = MMA_N;
  static constexpr int TMEM_COLS = 512;
  static constexpr uint32_t IDESC = (1u << 4) | (mode_fp8(MODE) ? 0u : (1u << 7) | (1u << 10)) |
                                    ((uint32_t)(MMA_N >> 3) << 17) |
                                    ((uint32_t)(TC2_BM >> 4) << 24);
};

// Shared memory beside the operand stages: alignment pad, staging, barriers, tile list.
template <int MODE> constexpr size_t tc2_fixed_bytes(int G) {
  return 1024 + (size_t)Tc2Cfg<MODE>::STG_BYTES + 256 +
         (size_t)(G + 1 + TC_THREADS / 32 + 1) * sizeof(int);
}
// Operand stages of kpb K-blocks that fit in the 227 KB a CTA may hold (at most MAX_STAGES K-blocks
// in all; < 2 means the tile list of G groups leaves no room for double buffering).
template <int MODE> constexpr int tc2_stages(int G, int kpb = 1) {
  const long long room = 227LL * 1024 - (long long)tc2_fixed_bytes<MODE>(G);
  const long long n = room < 0 ? 0 : room / ((long long)Tc2Cfg<MODE>::STAGE_BYTES * kpb);
  const int cap = Tc2Cfg<MODE>::MAX_STAGES / kpb;
  return n > cap ? cap : (int)n;
}
template <int MODE> constexpr size_t tc2_smem_bytes(int G, int kpb = 1) {
  return tc2_fixed_bytes<MODE>(G) +
         (size_t)tc2_stages<MODE>(G, kpb) * Tc2Cfg<MODE>::STAGE_BYTES * kpb;
}

template <int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(TC_THREADS, 1)
    gemm_tc2_kernel(const __grid_constant__ TcParams P) {
  using C = Tc2Cfg<MODE>;
  constexpr int BN = C::BN;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const GroupedGemm &p = P.p;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = p.E + p.has_shared;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int NST = P.stages;  // operand stages (2..MAX_STAGES), fixed by the host from G
  const int KPB = P.kpb;     // K-blocks per stage (1, or 2 with 3-D boxes)
  const uint32_t stage_bytes = (uint32_t)C::STAGE_BYTES * KPB;

  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t pad = ((raw + 1023u) & ~1023u) - raw;
  unsigned char *base = smem_raw + pad;
  unsigned char *stages = base;
  unsigned char *stg_all = base + (size_t)NST * stage_bytes;
  uint64_t *bars = (uint64_t *)(stg_all + C::STG_BYTES);
  uint32_t *tmem_slot = (uint32_t *)(bars + 2 * NST + 5);
  volatile int *abort_flag = (volatile int *)(tmem_slot + 1);
  int *prefix = (int *)(stg_all + C::STG_BYTES + 256);
  int *scan_tmp = prefix + G + 1;

  auto full_bar = [&](int s) { return smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return smem_u32(bars + NST + s); };
  auto accf_bar = [&](int b) { return smem_u32(bars + 2 * NST + b); };
  auto acce_bar = [&](int b) { return smem_u32(bars + 2 * NST + 2 + b); };
  const uint32_t drain_bar = smem_u32(bars + 2 * NST + 4);

  if (tid == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(accf_bar(b), 1);
      mbar_init(acce_bar(b), 2 * TC_EPI_WARPS);
    }
    mbar_init(drain_bar, 1);
    if (MODE == MODE_SWIGLU_BWD)
      for (int w = 0; w < TC_EPI_WARPS; ++w)
        mbar_init(smem_u32(stg_all + TC_EPI_WARPS * C::STG_WARP + 8 * w), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"((uint32_t)C::TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  const KernelStamp stamp(p.kind);
  griddep_wait();
  stamp.started();
  griddep_launch();
  const int total = build_tile_prefix(p, TC2_BM, BN, prefix, scan_tmp);
  tc_fence_before();
  cluster_sync_all();  // barriers of both CTAs initialised, TMEM allocated in both
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint64_t limit = g_wait_limit_ns;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int issued_parity[C::MAX_STAGES];
      bool issued[C::MAX_STAGES];
      for (int s = 0; s < C::MAX_STAGES; ++s) { issued[s] = false; issued_parity[s] = 0; }
      for (int tile = pair; tile < total && ok; tile += npairs) {
        const TileInfo ti = decode_tile(p, tile, prefix, TC2_BM, BN);
        const bool routed = ti.g < p.E;
        const CUtensorMap *ma = routed ? &P.maps.a_r : &P.maps.a_s;
        const CUtensorMap *mb = (tc2_two_b(MODE) && rank == 1)
                                    ? (routed ? &P.maps.b1_r : &P.maps.b1_s)
                                    : (routed ? &P.maps.b0_r : &P.maps.b0_s);
        const int a_row = ti.a_row0 + ti.m0 + (int)rank * 128;
        // CTA 1's half of a group's last tile can hold no row of the group (an expert's tail of
        // at most 128 rows): its A rows are never stored, so they are not loaded. The MMA reads
        // what that stage last held there and the epilogue masks those rows; the leader expects
        // the smaller byte count. Both CTAs decide it from the same tile record.
        const bool a1_void = ti.m0 + 128 >= ti.rows;
        const uint32_t stage_tx = KPB * (2 * C::STAGE_BYTES - (a1_void ? C::A_BYTES : 0));
        const int n_off = tc2_two_b(MODE) ? 0 : (int)rank * 128;
        // with two K-blocks per stage an odd count leaves the last stage half used: its second
        // tile (the next group's columns, or the map's zero fill) is loaded and not multiplied.
        // MN-major: each segment's nbg K-blocks start a stage (nbg rounded up to KPB)
        int nbg_pad = 0, nk;
        if (p.mn) {
          nbg_pad = (ti.K / (p.kseg * C::BK) + KPB - 1) / KPB * KPB;
          nk = p.kseg * nbg_pad;
        } else {
          nk = (ti.K + C::BK - 1) / C::BK;
        }
        for (int kb = 0; kb < nk; kb += KPB) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, abort_flag, limit, INFO_WAIT_MMA_EMPTY)) {
            ok = false;
            break;
          }
          const uint32_t sA = smem_u32(stages + (size_t)stage * stage_bytes);
          const uint32_t sB = sA + C::A_BYTES * KPB;
          if (rank == 0) mbar_expect_tx(full_bar(stage), stage_tx);
          const int kk = kb * C::BK;
          int b_row, b_col;
          if (p.kgroup) {  // one A and one B for all groups, each group its own K columns
            b_row = ti.n0 + n_off;
            b_col = ti.kofs + kk;
          } else if (routed) {
            b_row = ti.g * ti.N + ti.n0 + n_off;
            b_col = p.kb_r ? kk % p.kb_r : kk;
          } else {
            const int piece = kk / p.piece_k;
            b_row = piece * p.piece_rows + ti.n0 + n_off;
            b_col = kk - piece * p.piece_k;
          }
          if (p.mn) {  // MN-major: 64 KPB rows of K, two 64-column blocks of M (N) per operand
            const int seg = kb / nbg_pad, j0 = kb - seg * nbg_pad;
            const int acb = (ti.m0 + (int)rank * 128 + p.mn_col_a[seg]) >> 6;
            const int bcb = (ti.n0 + n_off + p.mn_col_b[seg]) >> 6;
            if (rank == 0 || !a1_void)
              tma_load_3d_pair(sA, ma, 0, p.mn_row_a[ti.g] + j0 * C::BK, acb, full_bar(stage));
            tma_load_3d_pair(sB, mb, 0, p.mn_row_b[ti.g] + j0 * C::BK, bcb, full_bar(stage));
          } else if (KPB == 2) {  // boxes of two K-blocks: coordinates {column, row, K-block}
            if (rank == 0 || !a1_void)
              tma_load_3d_pair(sA, ma, 0, a_row, (ti.kofs + kk) / C::BK, full_bar(stage));
            tma_load_3d_pair(sB, mb, 0, b_row, b_col / C::BK, full_bar(stage));
          } else {
            if (rank == 0 || !a1_void) tma_load_2d_pair(sA, ma, ti.kofs + kk, a_row, full_bar(stage));
            tma_load_2d_pair(sB, mb, b_col, b_row, full_bar(stage));
          }
          issued[stage] = true;
          issued_parity[stage] = (int)phase;
          if (++stage == NST) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok && rank == 0) {
        for (int s = 0; s < NST; ++s)
          if (issued[s]) {
            volatile int never = 0;
            mbar_wait(full_bar(s), (uint32_t)issued_parity[s], &never, limit, INFO_WAIT_DRAIN);
          }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader only)
    if (rank == 0 && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true, any = false;
      for (int tile = pair; tile < total && ok; tile += npairs) {
        const TileInfo ti = decode_tile(p, tile, prefix, TC2_BM, BN);
        int nbg = 0, nbg_pad = 0, nk;  // as in the producer
        if (p.mn) {
          nbg = ti.K / (p.kseg * C::BK);
          nbg_pad = (nbg + KPB - 1) / KPB * KPB;
          nk = p.kseg * nbg_pad;
        } else {
          nk = (ti.K + C::BK - 1) / C::BK;
        }
        if (!mbar_wait(acce_bar(acc), acc_phase ^ 1u, abort_flag, limit, INFO_WAIT_ACC_EMPTY)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d0 = tmem_base + (uint32_t)(acc * C::ACC_COLS);
        for (int kb = 0; kb < nk; kb += KPB) {
          if (!mbar_wait(full_bar(stage), phase, abort_flag, limit, INFO_WAIT_TMA_FULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sA0 = smem_u32(stages + (size_t)stage * stage_bytes);
          const uint32_t sB0 = sA0 + C::A_BYTES * KPB;
          if (!mode_fp8(MODE) && p.mn) {
            // MN-major: each operand two 64-column blocks of 64 KPB rows; the stage's K-blocks
            // that lie in the segment (nbg >= 1 for every listed tile), 16 rows of K (2 KB)
            // per instruction
            const int j0 = kb % nbg_pad;
            const uint32_t lbo = 8192u * KPB;
            for (int j = 0; j < KPB && j0 + j < nbg; ++j) {
#pragma unroll
              for (int k16 = 0; k16 < 4; ++k16)
                tc2_mma(d0, make_sdesc_mn(sA0 + j * 8192 + k16 * 2048, lbo),
                        make_sdesc_mn(sB0 + j * 8192 + k16 * 2048, lbo), C::IDESC | IDESC_MN_MAJOR,
                        (kb > 0 || j > 0 || k16 > 0) ? 1u : 0u);
            }
          } else {
            for (int j = 0; j < KPB && kb + j < nk; ++j) {  // the stage's K-blocks, 16 KB tiles
              const uint32_t sA = sA0 + j * C::A_BYTES, sB = sB0 + j * C::B_BYTES;
#pragma unroll
              for (int k16 = 0; k16 < 4; ++k16) {  // 32 bytes of K per instruction
                const uint32_t accum = (kb > 0 || j > 0 || k16 > 0) ? 1u : 0u;
                if (mode_fp8(MODE))
                  tc2_mma_f8(d0, make_sdesc(sA + k16 * 32), make_sdesc(sB + k16 * 32), C::IDESC, accum);
                else
                  tc2_mma(d0, make_sdesc(sA + k16 * 32), make_sdesc(sB + k16 * 32), C::IDESC, accum);
              }
            }
          }
          any = true;
          tc2_commit_both(empty_bar(stage));
          if (++stage == NST) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc2_commit_both(accf_bar(acc));
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      if (!ok && any) {
        tc2_commit_both(drain_bar);
        volatile int never = 0;
        mbar_wait(drain_bar, 0u, &never, limit, INFO_WAIT_DRAIN);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..9)
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    const int cbeg = half * (BN / 2), cend = cbeg + BN / 2;
    int acc = 0;
    uint32_t acc_phase = 0;
    GuFeed feed;  // SWIGLU_BWD: this warp's g, u blocks
    feed.buf = smem_u32(stg_all + (warp - 2) * C::STG_WARP);
    feed.bar = smem_u32(stg_all + TC_EPI_WARPS * C::STG_WARP + 8 * (warp - 2));
    feed.phase = 0;
    feed.pending = false;
    for (int tile = pair; tile < total; tile += npairs) {
      const TileInfo ti = decode_tile(p, tile, prefix, TC2_BM, BN);
      const bool routed = ti.g < p.E;
      const int rbase = ti.m0 + (int)rank * 128 + q * 32;  // first row of this warp's block
      const int row = rbase + lane;
      const bool row_ok = row < ti.rows;
      // SWIGLU_BWD with padded outputs: the group's rows up to the next multiple of 64 are
      // written, row i < rows at aux_row0[g+1] - rows + i and the padding ones (as zeros) in
      // front of them
      const bool pad = MODE == MODE_SWIGLU_BWD && p.pad_out && routed;
      const int rows_w = pad ? ((ti.rows + 63) & ~63) : ti.rows;
      // a warp of padding rows only, or columns past the group's width: nothing to store
      const int cstop = rbase < rows_w ? min(cend, ti.N - ti.n0) : cbeg;
      if (MODE == MODE_SWIGLU_BWD && cstop > cbeg)
        feed.issue(gu_pair_block(p, ti, routed, routed ? p.aux_r : p.aux_s, rbase, ti.n0 + cbeg),
                   lane);
      // PLAIN_FP8: the row's scale, read before the accumulator is ready
      const float rs8 = (MODE == MODE_PLAIN_FP8 && routed && row_ok)
                            ? __ldg(p.row_scale + ti.a_row0 + row) : 0.0f;
      bool ok = true;
      if (lane == 0)
        ok = mbar_wait(accf_bar(acc), acc_phase, abort_flag, limit, INFO_WAIT_ACC_FULL);
      ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
      if (!ok) break;
      tc_fence_after();
      void *out = routed ? p.out_r : p.out_s;
      const int ldo = routed ? p.ldo_r : p.ldo_s;
      const uint32_t tbase = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * C::ACC_COLS);
      unsigned char *stg = stg_all + (warp - 2) * C::STG_WARP;
#pragma unroll 1
      for (int c = cbeg; c < cstop; c += 32) {
        if (MODE == MODE_GATEUP_RAW) {
          uint32_t r0[32], r1[32];
          tmem_ld32(tbase + c, r0);
          tmem_ld32(tbase + BN + c, r1);
          tmem_wait_ld();
          gateup_raw_chunk(r0, r1, stg, gu_pair_block(p, ti, routed, out, rbase, ti.n0 + c), lane);
          continue;
        }
        if (MODE == MODE_SWIGLU_BWD) {
          const int col = ti.n0 + c;
          const int hf = routed ? p.half_r : p.half_s;
          uint32_t r0[32];
          tmem_ld32(tbase + c, r0);
          tmem_wait_ld();
          if (!feed.wait(abort_flag, limit)) { ok = false; break; }
          const size_t arow = pad ? (size_t)(p.aux_row0[ti.g] + (row_ok ? row + rows_w - ti.rows
                                                                         : row - ti.rows))
                                  : (size_t)(ti.out_row0 + row);
          __nv_bfloat16 *o = (__nv_bfloat16 *)out + arow * ldo + col;
          __nv_bfloat16 *o2 = (__nv_bfloat16 *)(routed ? p.out2_r : p.out2_s) +
                              arow * (routed ? p.ld2_r : p.ld2_s) + col;
          swiglu_bwd_chunk(r0, stg, lane, row_ok, !row_ok && row < rows_w, o, o2, hf, [&] {
            if (c + 32 < cstop)
              feed.issue(gu_pair_block(p, ti, routed, routed ? p.aux_r : p.aux_s, rbase, col + 32),
                         lane);
          });
          continue;
        }
        if (MODE == MODE_GATEUP_F32) {
          // silu(gate) * up in fp32 (IEEE exp and division), 32 columns (128 bytes of each row)
          // at a time, staged per warp and written as 32 coalesced 128-byte row stores
          uint32_t r0[32], r1[32];
          tmem_ld32(tbase + c, r0);
          tmem_ld32(tbase + BN + c, r1);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float g = __uint_as_float(r0[i]);
            r0[i] = __float_as_uint(g / (1.0f + expf(-g)) * __uint_as_float(r1[i]));
          }
#pragma unroll
          for (int i = 0; i < 8; ++i)
            *(uint4 *)(stg + lane * 128 + ((i ^ (lane & 7)) << 4)) =
                make_uint4(r0[4 * i], r0[4 * i + 1], r0[4 * i + 2], r0[4 * i + 3]);
          __syncwarp();
          const int col = ti.n0 + c;
          const int nrows = min(32, ti.rows - rbase);
          unsigned char *obase = (unsigned char *)out + ((size_t)(ti.out_row0 + rbase) * ldo + col) * 4;
          const size_t row_bytes = (size_t)ldo * 4;
          for (int rr = 0; rr < nrows; ++rr) {
            const uint32_t v = *(const uint32_t *)(stg + rr * 128 +
                                                   (((lane >> 2) ^ (rr & 7)) << 4) + ((lane & 3) << 2));
            *(uint32_t *)(obase + rr * row_bytes + lane * 4) = v;
          }
          __syncwarp();
          continue;
        }
        if (MODE == MODE_GATEUP) {
          // silu(gate) * up in bf16, 64 columns (128 bytes of each row) at a time: both 32-column
          // halves are packed, staged per warp and written as 32 coalesced 128-byte row stores
          if ((c - cbeg) & 32) continue;  // the odd 32-column steps were taken with the even ones
          uint32_t pk[32];
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            uint32_t r0[32], r1[32];
            tmem_ld32(tbase + c + 32 * hh, r0);
            tmem_ld32(tbase + BN + c + 32 * hh, r1);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float g0 = __uint_as_float(r0[2 * i]), g1 = __uint_as_float(r0[2 * i + 1]);
              __nv_bfloat162 h = __floats2bfloat162_rn(
                  __fdividef(g0, 1.0f + __expf(-g0)) * __uint_as_float(r1[2 * i]),
                  __fdividef(g1, 1.0f + __expf(-g1)) * __uint_as_float(r1[2 * i + 1]));
              pk[16 * hh + i] = *(uint32_t *)&h;
            }
          }
#pragma unroll
          for (int i = 0; i < 8; ++i)
            *(uint4 *)(stg + lane * 128 + ((i ^ (lane & 7)) << 4)) =
                make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
          __syncwarp();
          const int col = ti.n0 + c;
          if (col < ti.N) {
            const int nrows = min(32, ti.rows - rbase);
            unsigned char *obase = (unsigned char *)out + ((size_t)(ti.out_row0 + rbase) * ldo + col) * 2;
            const size_t row_bytes = (size_t)ldo * 2;
            for (int rr = 0; rr < nrows; ++rr) {
              const uint32_t v = *(const uint32_t *)(stg + rr * 128 +
                                                     (((lane >> 2) ^ (rr & 7)) << 4) + ((lane & 3) << 2));
              *(uint32_t *)(obase + rr * row_bytes + lane * 4) = v;
            }
          }
          __syncwarp();
        } else if (routed && p.out_r_bf16) {
          // routed expert outputs in bf16, 64 columns (128 bytes of each row) at a time: staged
          // per warp like the fp32 path and written as 32 coalesced 128-byte row stores
          if ((c - cbeg) & 32) continue;  // the odd 32-column steps were taken with the even ones
          uint32_t r0[32], r1[32];
          tmem_ld32(tbase + c, r0);
          tmem_ld32(tbase + c + 32, r1);
          tmem_wait_ld();
          uint32_t pk[32];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            __nv_bfloat162 a = __floats2bfloat162_rn(__uint_as_float(r0[2 * i]), __uint_as_float(r0[2 * i + 1]));
            __nv_bfloat162 b = __floats2bfloat162_rn(__uint_as_float(r1[2 * i]), __uint_as_float(r1[2 * i + 1]));
            pk[i] = *(uint32_t *)&a;
            pk[16 + i] = *(uint32_t *)&b;
          }
#pragma unroll
          for (int i = 0; i < 8; ++i)
            *(uint4 *)(stg + lane * 128 + ((i ^ (lane & 7)) << 4)) =
                make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
          __syncwarp();
          const int col = ti.n0 + c;
          if (col < ti.N) {
            const int nrows = min(32, ti.rows - rbase);
            unsigned char *obase = (unsigned char *)out + ((size_t)(ti.out_row0 + rbase) * ldo + col) * 2;
            const size_t row_bytes = (size_t)ldo * 2;
            for (int rr = 0; rr < nrows; ++rr) {
              const uint32_t v = *(const uint32_t *)(stg + rr * 128 +
                                                     (((lane >> 2) ^ (rr & 7)) << 4) + ((lane & 3) << 2));
              *(uint32_t *)(obase + rr * row_bytes + lane * 4) = v;
            }
          }
          __syncwarp();
        } else {
          // fp32 output, staged per warp and written as 128-byte rows
          float4 cs8[8];  // PLAIN_FP8: the U rows' scales of columns col .. col + 31
          if (MODE == MODE_PLAIN_FP8 && routed) {
            const float4 *cs = (const float4 *)(p.col_scale + (size_t)ti.g * ti.N + ti.n0 + c);
#pragma unroll
            for (int i = 0; i < 8; ++i) cs8[i] = __ldg(cs + i);
          }
          uint32_t r0[32];
          tmem_ld32(tbase + c, r0);
          tmem_wait_ld();
          if (MODE == MODE_PLAIN_FP8 && routed) {
            // y = sum * (row scale) * (U row scale)
#pragma unroll
            for (int i = 0; i < 8; ++i) {
              r0[4 * i] = __float_as_uint(__uint_as_float(r0[4 * i]) * rs8 * cs8[i].x);
              r0[4 * i + 1] = __float_as_uint(__uint_as_float(r0[4 * i + 1]) * rs8 * cs8[i].y);
              r0[4 * i + 2] = __float_as_uint(__uint_as_float(r0[4 * i + 2]) * rs8 * cs8[i].z);
              r0[4 * i + 3] = __float_as_uint(__uint_as_float(r0[4 * i + 3]) * rs8 * cs8[i].w);
            }
          }
#pragma unroll
          for (int i = 0; i < 8; ++i)
            *(uint4 *)(stg + lane * 128 + ((i ^ (lane & 7)) << 4)) =
                make_uint4(r0[4 * i], r0[4 * i + 1], r0[4 * i + 2], r0[4 * i + 3]);
          __syncwarp();
          const int col = ti.n0 + c;
          if (col < ti.N) {
            const int nrows = min(32, ti.rows - rbase);
            unsigned char *obase = (unsigned char *)out + ((size_t)(ti.out_row0 + rbase) * ldo + col) * 4;
            const size_t row_bytes = (size_t)ldo * 4;
            for (int rr = 0; rr < nrows; ++rr) {
              const uint32_t v = *(const uint32_t *)(stg + rr * 128 +
                                                     (((lane >> 2) ^ (rr & 7)) << 4) + ((lane & 3) << 2));
              *(uint32_t *)(obase + rr * row_bytes + lane * 4) = v;
            }
          }
          __syncwarp();
        }
      }
      if (!ok) break;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cta0(acce_bar(acc));
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
    if (MODE == MODE_SWIGLU_BWD) feed.drain(limit);
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // no CTA leaves while its peer may still read its smem or TMEM
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                 "r"((uint32_t)C::TMEM_COLS)
                 : "memory");
  }
}

}  // namespace moe

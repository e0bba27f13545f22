// C ABI of the MoE FFN layer: argument checks, workspace layout, tensor maps and launches.
// All kernels live in this one translation unit (the .cuh files), so the device error word and
// the debug switches are single symbols without relocatable device code.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>

#include "../../include/moe.h"
#include "backward.cuh"
#include "combine.cuh"
#include "common.cuh"
#include "f32split.cuh"
#include "fp8.cuh"
#include "gemm_tc.cuh"
#include "gemm_tc2.cuh"
#include "permute.cuh"
#include "router.cuh"
#include "stats.cuh"

using namespace moe;

static_assert(RT_TM == PM_CHUNK, "the router CTA is the permutation chunk");

namespace {

// ------------------------------------------------------------------ validation
bool cfg_supported(const moe_config_t *c) {
  if (!c) return false;
  if (c->T < 0 || c->d <= 0 || c->E <= 0 || c->top_k <= 0 || c->n_shared < 0) return false;
  if (c->E > 1024 || c->top_k > 8 || c->top_k > c->E || c->n_shared > 8) return false;
  if (c->d % 64) return false;
  if (c->score != MOE_SCORE_SOFTMAX && c->score != MOE_SCORE_SIGMOID) return false;
  if (c->dtype != MOE_DTYPE_F32 && c->dtype != MOE_DTYPE_BF16) return false;
  if (c->expert == MOE_EXPERT_SWIGLU) {
    if (c->ffn <= 0 || c->ffn % 64) return false;
  } else if (c->expert == MOE_EXPERT_LOWRANK) {
    if (c->rank <= 0 || c->rank % 64 || c->rank > 256) return false;
  } else {
    return false;
  }
  if (c->n_shared > 0 && (c->ffn_shared <= 0 || c->ffn_shared % 64)) return false;
  if (c->expert_storage != MOE_STORAGE_DTYPE && c->expert_storage != MOE_STORAGE_FP8_E4M3)
    return false;
  // fp8 storage: bf16 low-rank layers; the quantising scatter holds a row in registers
  if (c->expert_storage == MOE_STORAGE_FP8_E4M3 &&
      (c->expert != MOE_EXPERT_LOWRANK || c->dtype != MOE_DTYPE_BF16 ||
       c->d > 32 * PM_VEC * 8))
    return false;
  if (!std::isfinite(c->capacity_factor) || !std::isfinite(c->aux_alpha)) return false;
  // the router stages its 16 token rows and the logits in shared memory (227 KB per CTA)
  const bool sig = c->score == MOE_SCORE_SIGMOID;
  const int es = c->dtype == MOE_DTYPE_BF16 ? 2 : 4;
  if (router_smem(c->E, sig, c->d, es, router_ept(c->E, sig, c->d, es)).total > 227 * 1024)
    return false;
  // 32-bit row indices inside the kernels
  if ((long long)c->T * c->top_k * std::max(c->d, 256) >= (1ll << 31) * 64ll) return false;
  if ((long long)c->T * c->top_k >= (1ll << 31)) return false;
  return true;
}

inline bool aligned16(const void *p) { return p && ((uintptr_t)p & 15u) == 0; }
// token-sized buffers may be NULL in an empty call (T == 0)
inline bool tok16(const moe_config_t *c, const void *p) {
  return (c->T == 0 && p == nullptr) || aligned16(p);
}
inline size_t esize(const moe_config_t *c) { return c->dtype == MOE_DTYPE_BF16 ? 2 : 4; }
inline int ceil_div(long long a, long long b) { return (int)((a + b - 1) / b); }
inline size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

// exact ceil(cf * T * k / E) on the fp32 value of cf (cf = m * 2^ex, m a 24-bit integer)
int32_t capacity_of(const moe_config_t *c) {
  const float cf = c->capacity_factor;
  if (!(cf > 0.0f)) return -1;
  int ex;
  const float fr = std::frexp(cf, &ex);                 // cf = fr * 2^ex, 0.5 <= fr < 1
  const long long m = (long long)std::ldexp(fr, 24);    // exact 24-bit integer
  ex -= 24;                                            // cf = m * 2^ex
  __int128 num = (__int128)m * c->T * c->top_k;        // cf*T*k = num * 2^ex
  __int128 den = c->E;
  if (ex >= 0) {
    if (ex > 60) return 0x7fffffff;
    num <<= ex;
  } else {
    if (-ex > 100) return num > 0 ? 1 : 0;
    den <<= -ex;
  }
  __int128 q = num / den;
  if (q * den < num) q += 1;
  if (q > 0x7fffffff) return 0x7fffffff;
  return (int32_t)q;
}

// ------------------------------------------------------------------ workspace layout
// Routed expert outputs are stored in bf16 for bf16 SwiGLU layers (each enters y through a
// weighted sum of top_k rows plus the fp32 shared output, which averages their rounding) and in
// fp32 otherwise: a low-rank layer's y is a weighted sum of as few as two rows and no shared
// output, where one bf16 rounding of the rows exceeds the layer's error budget on its own.
inline bool yperm_bf16(const moe_config_t *c) {
  return c->dtype == MOE_DTYPE_BF16 && c->expert == MOE_EXPERT_SWIGLU;
}

struct Layout {
  size_t part_cnt, part_prob, chunk_base, kept;                 // route / statistics
  size_t chunk_count;                                           // moe_permute's own histogram
  size_t lrank;                                                 // within-chunk ranks [T, k] u8
  size_t hidden, hidden_sh;                                     // experts
  size_t idx, wts, count, prob, offsets, slot_pos, src, x_perm, y_perm, y_shared, aux;  // layer
  size_t sx_perm, zq, sz;  // fp8 storage: scales of the E4M3 token rows, z rows and scales
  // fp32 layers: operands as six bf16 K segments (f32split.cuh): token rows, hidden rows, the
  // routed weights of both products, and the shared experts' counterparts
  size_t s6_x, s6_h, s6_w1, s6_w1b, s6_w2, s6_xs, s6_hs, s6_sg, s6_su, s6_sd;
  size_t total;
};
inline bool fp8_experts(const moe_config_t *c) { return c->expert_storage == MOE_STORAGE_FP8_E4M3; }

Layout layout_of(const moe_config_t *c) {
  Layout L;
  const size_t T = c->T, d = c->d, E = c->E, k = c->top_k, es = esize(c);
  const size_t nch = std::max<size_t>(1, ceil_div(c->T, RT_TM));
  // hidden rows: the SwiGLU activations, or the low-rank projection (bf16: hi and lo terms;
  // fp8 storage: none, its E4M3 rows are `zq`)
  const size_t width = c->expert == MOE_EXPERT_SWIGLU ? (size_t)c->ffn
                       : fp8_experts(c)               ? 0
                       : (size_t)c->rank * (c->dtype == MOE_DTYPE_BF16 ? 2 : 1);
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t at = o; o = align256(o + std::max<size_t>(bytes, 1)); return at; };
  L.part_cnt = take(nch * E * 4);
  L.part_prob = take(nch * E * 4);
  L.chunk_base = take(nch * E * 4);
  L.kept = take(E * 4);
  L.chunk_count = take(nch * E * 4);
  L.lrank = take(T * k);
  L.hidden = take(T * k * width * es);
  L.hidden_sh = take(T * (size_t)c->n_shared * (size_t)c->ffn_shared * es);
  L.idx = take(T * k * 4);
  L.wts = take(T * k * 4);
  L.count = take(E * 4);
  L.prob = take(E * 4);
  L.offsets = take((E + 1) * 4);
  L.slot_pos = take(T * k * 4);
  L.src = take(T * k * 4);
  L.x_perm = take(T * k * d * es);
  L.y_perm = take(T * k * d * (yperm_bf16(c) ? 2 : 4));
  L.y_shared = take(T * d * 4);
  L.aux = take(16);
  // fp8 storage: the x_perm region holds the rows' E4M3 codes
  const bool f8 = fp8_experts(c);
  L.sx_perm = take(f8 ? T * k * 4 : 0);
  L.zq = take(f8 ? T * k * (size_t)c->rank : 0);
  L.sz = take(f8 ? T * k * 4 : 0);
  const bool f32 = c->dtype == MOE_DTYPE_F32;
  const size_t hw = c->expert == MOE_EXPERT_SWIGLU ? (size_t)c->ffn : (size_t)c->rank;
  const size_t sfs = (size_t)c->n_shared * c->ffn_shared;
  L.s6_x = take(f32 ? T * k * 6 * d * 2 : 0);
  L.s6_h = take(f32 ? T * k * 6 * hw * 2 : 0);
  L.s6_w1 = take(f32 ? E * hw * 6 * d * 2 : 0);
  L.s6_w1b = take(f32 && c->expert == MOE_EXPERT_SWIGLU ? E * hw * 6 * d * 2 : 0);
  L.s6_w2 = take(f32 ? E * d * 6 * hw * 2 : 0);
  L.s6_xs = take(f32 ? T * 6 * d * 2 * (sfs > 0) : 0);
  L.s6_hs = take(f32 ? T * 6 * sfs * 2 : 0);
  L.s6_sg = take(f32 ? sfs * 6 * d * 2 : 0);
  L.s6_su = take(f32 ? sfs * 6 * d * 2 : 0);
  L.s6_sd = take(f32 ? d * 6 * sfs * 2 : 0);
  L.total = o;
  return L;
}

template <typename T> T *at(void *ws, size_t off) { return (T *)((char *)ws + off); }

// ------------------------------------------------------------------ device properties
struct DevInfo {
  int sms = 0;
  bool tc_attr[8] = {};
};
DevInfo g_dev[64];

int current_device() {
  int dev = 0;
  cudaGetDevice(&dev);
  return dev;
}
int num_sms() {
  const int dev = current_device();
  if (dev >= 0 && dev < 64) {
    if (!g_dev[dev].sms) cudaDeviceGetAttribute(&g_dev[dev].sms, cudaDevAttrMultiProcessorCount, dev);
    return g_dev[dev].sms;
  }
  int s = 0;
  cudaDeviceGetAttribute(&s, cudaDevAttrMultiProcessorCount, dev);
  return s;
}

// ------------------------------------------------------------------ profiling (debug)
const char *kKindName[K_COUNT] = {"router", "stats", "perm_hist", "perm_scatter", "gemm_gateup",
                                  "gemm_down", "gemm_lowrank_v", "gemm_lowrank_u", "combine",
                                  "aux_loss", "backward_gemm", "quantize_fp8",
                                  "split_f32"};
constexpr int PROF_SLOTS = 8192;
struct Prof {
  bool on = false;
  cudaEvent_t ev[2 * PROF_SLOTS];
  int kind[PROF_SLOTS];
  int n = 0;
  bool created = false;
} g_prof;
std::mutex g_prof_mu;

struct ProfScope {
  int slot = -1;
  cudaStream_t st;
  ProfScope(int kind, cudaStream_t s) : st(s) {
    if (!g_prof.on) return;
    std::lock_guard<std::mutex> lk(g_prof_mu);
    if (g_prof.n >= PROF_SLOTS) return;
    slot = g_prof.n++;
    g_prof.kind[slot] = kind;
    cudaEventRecord(g_prof.ev[2 * slot], st);
  }
  ~ProfScope() {
    if (slot >= 0) cudaEventRecord(g_prof.ev[2 * slot + 1], st);
  }
};

// Sets every in-step stamp slot to (no start, no end).
moe_status_t stamp_reset() {
  static unsigned long long h[K_COUNT][STAMP_SLOTS][2];
  for (int k = 0; k < K_COUNT; ++k)
    for (int sl = 0; sl < STAMP_SLOTS; ++sl) {
      h[k][sl][0] = ~0ull;
      h[k][sl][1] = 0ull;
    }
  return cudaMemcpyToSymbol(g_stamp, h, sizeof(h)) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

moe_status_t last_launch_status() {
  const cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

// Every layer kernel is launched with programmatic stream serialisation, so its CTAs may be
// scheduled (and set up shared memory, barriers and TMEM) while the previous kernel finishes;
// each kernel's griddep_wait() orders its memory accesses after that kernel (common.cuh).
template <typename... KArgs, typename... Args>
moe_status_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                        cudaStream_t st, Args... args) {
  cudaLaunchConfig_t cfg;
  std::memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
  return e == cudaSuccess ? last_launch_status() : MOE_ERR_CUDA;
}

// ------------------------------------------------------------------ tensor maps
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void *f = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (PFN_cuTensorMapEncodeTiled_v12000)f;
  });
  return fn;
}

// 2-D map over a row-major [rows, cols] matrix of bf16 (esz 2) or E4M3 bytes (esz 1); box
// [box_rows, 128 bytes of columns], 128B swizzle. Columns past `cols` in a box read as zeros
// (an E4M3 K of 64 fills half a box).
bool make_map(CUtensorMap *m, const void *ptr, uint64_t rows, uint64_t cols, uint32_t box_rows,
              int esz = 2) {
  auto fn = encode_fn();
  if (!fn) return false;
  if (rows == 0 || ptr == nullptr) {  // never dereferenced: map a dummy 1-row extent
    rows = 1;
  }
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * (cuuint64_t)esz};
  cuuint32_t box[2] = {(cuuint32_t)(128 / esz), box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, esz == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                        2, const_cast<void *>(ptr), dims, strides,
                        box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3-D bf16 map over a row-major [rows, cols] matrix seen as {64 columns, rows, cols / 64 K-blocks}
// (strides: the row, then 128 bytes); box {64, box_rows, 2}: two K-blocks' [box_rows, 64] tiles,
// one after the other, 128B swizzle. cols a multiple of 64; a box's K-block past the last reads
// as zeros.
bool make_map3(CUtensorMap *m, const void *ptr, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  if (rows == 0 || ptr == nullptr) rows = 1;
  cuuint64_t dims[3] = {64, rows, cols / 64};
  cuuint64_t strides[2] = {cols * 2, 128};
  cuuint32_t box[3] = {64, box_rows, 2};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// MN-major operand: the same 3-D view of a row-major [rows, cols] matrix (cols a multiple of
// 64), box {64, box_rows, 2}: box_rows rows (K) of two consecutive 64-column blocks (M or N),
// block after block; rows before 0 or past the end read as zeros.
bool make_map_mn(CUtensorMap *m, const void *ptr, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  if (rows == 0 || ptr == nullptr) rows = 1;
  cuuint64_t dims[3] = {64, rows, cols / 64};
  cuuint64_t strides[2] = {cols * 2, 128};
  cuuint32_t box[3] = {64, box_rows, 2};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(ptr), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// ------------------------------------------------------------------ grouped GEMM launches
long long tile_bound(const GroupedGemm &g, int BM, int BN) {
  if (g.kgroup) return (long long)g.E * ceil_div(g.rows_r, BM) * ceil_div(g.N_r, BN);
  long long t = 0;
  if (g.E > 0) t += ((long long)ceil_div(g.rows_r, BM) + g.E) * ceil_div(g.N_r, BN);
  if (g.has_shared) t += (long long)ceil_div(g.T, BM) * ceil_div(g.N_s, BN);
  return t;
}

// Tensor maps of one grouped launch: A boxes of 128 rows, B boxes of `b_box` rows.
// routed operands: A [rows_r, K_r], B [E*N_r, K_r]; shared: A [T, K_s], B [b_rows_s, piece_k]
bool build_maps(const GroupedGemm &g, bool two_b, uint32_t b_box, TcMaps *m, int esz = 2,
                bool kb2 = false) {
  const void *any = g.E > 0 ? g.A_r : g.A_s;
  if (g.mn) {  // groups along K, both operands MN-major (the other maps are unused)
    const uint32_t box_rows = kb2 ? 128 : 64;
    bool ok = make_map_mn(&m->a_r, g.A_r, g.mn_rows_a, g.mn_lda, box_rows);
    ok &= make_map_mn(&m->b0_r, g.B0_r, g.mn_rows_b, g.mn_ldb, box_rows);
    m->b1_r = m->b0_r;
    m->a_s = m->a_r;
    m->b0_s = m->b1_s = m->b0_r;
    return ok;
  }
  if (kb2) {  // bf16; the same extents as the 2-D maps below
    const int kb = g.kb_r ? g.kb_r : g.K_r;
    const uint64_t b_rows = g.kgroup ? (uint64_t)g.N_r : (uint64_t)g.E * g.N_r;
    bool ok = true;
    ok &= make_map3(&m->a_r, g.E > 0 ? g.A_r : any, g.E > 0 ? g.rows_r : 1, g.E > 0 ? g.K_r : 128, 128);
    ok &= make_map3(&m->b0_r, g.E > 0 ? g.B0_r : any, g.E > 0 ? b_rows : 1, g.E > 0 ? kb : 128, b_box);
    ok &= make_map3(&m->b1_r, (g.E > 0 && two_b) ? g.B1_r : any, (g.E > 0 && two_b) ? b_rows : 1,
                    g.E > 0 ? kb : 128, b_box);
    ok &= make_map3(&m->a_s, g.has_shared ? g.A_s : any, g.has_shared ? g.T : 1,
                    g.has_shared ? g.K_s : 128, 128);
    ok &= make_map3(&m->b0_s, g.has_shared ? g.B0_s : any, g.has_shared ? g.b_rows_s : 1,
                    g.has_shared ? g.piece_k : 128, b_box);
    ok &= make_map3(&m->b1_s, (g.has_shared && two_b) ? g.B1_s : any,
                    (g.has_shared && two_b) ? g.b_rows_s : 1, g.has_shared ? g.piece_k : 128, b_box);
    return ok;
  }
  bool ok = true;
  ok &= make_map(&m->a_r, g.E > 0 ? g.A_r : any, g.E > 0 ? g.rows_r : 1, g.E > 0 ? g.K_r : 64, 128,
                 esz);
  const int kb = g.kb_r ? g.kb_r : g.K_r;  // row length of the routed weights
  // routed weights: E stacked [N_r, kb] matrices; groups along K: one [N_r, K_r] for all groups
  const uint64_t b_rows = g.kgroup ? (uint64_t)g.N_r : (uint64_t)g.E * g.N_r;
  ok &= make_map(&m->b0_r, g.E > 0 ? g.B0_r : any, g.E > 0 ? b_rows : 1, g.E > 0 ? kb : 64, b_box,
                 esz);
  ok &= make_map(&m->b1_r, (g.E > 0 && two_b) ? g.B1_r : any, (g.E > 0 && two_b) ? b_rows : 1,
                 g.E > 0 ? kb : 64, b_box, esz);
  ok &= make_map(&m->a_s, g.has_shared ? g.A_s : any, g.has_shared ? g.T : 1,
                 g.has_shared ? g.K_s : 64, 128);
  ok &= make_map(&m->b0_s, g.has_shared ? g.B0_s : any, g.has_shared ? g.b_rows_s : 1,
                 g.has_shared ? g.piece_k : 64, b_box);
  ok &= make_map(&m->b1_s, (g.has_shared && two_b) ? g.B1_s : any,
                 (g.has_shared && two_b) ? g.b_rows_s : 1, g.has_shared ? g.piece_k : 64, b_box);
  return ok;
}

template <int MODE, int BN>
moe_status_t launch_tc(const GroupedGemm &g, cudaStream_t st, int kind) {
  TcParams P;
  std::memset(&P, 0, sizeof(P));
  P.p = g;
  P.p.kind = kind;
  if (!build_maps(g, MODE == MODE_GATEUP, BN, &P.maps, mode_fp8(MODE) ? 1 : 2)) return MOE_ERR_CUDA;
  const int G = g.E + g.has_shared;
  const size_t smem = tc_smem_bytes<MODE, BN>(G);
  auto kern = gemm_tc_kernel<MODE, BN>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return MOE_ERR_CUDA;
  const long long bound = tile_bound(g, TC_BM, BN);
  if (bound == 0) return MOE_OK;
  const int grid = (int)std::min<long long>(num_sms(), bound);
  ProfScope ps(kind, st);
  return launch_pdl(kern, dim3(grid), dim3(TC_THREADS), smem, st, P);
}

// CTA-pair form (two SMs per 256-row tile); each CTA loads 128-row halves of A and B.
template <int MODE>
moe_status_t launch_tc2(const GroupedGemm &g, cudaStream_t st, int kind) {
  using C = Tc2Cfg<MODE>;
  TcParams P;
  std::memset(&P, 0, sizeof(P));
  P.p = g;
  P.p.kind = kind;
  const int G = g.E + g.has_shared;
  // two K-blocks per stage (3-D boxes) for the bf16 products, when no stage can cross a wrap
  // point of B's columns or a shared-expert piece, and the ring keeps at least 2 stages of 2
  // (MN-major operands: every segment's K-blocks start a stage, so no stage crosses one)
  const bool kb2 = !mode_fp8(MODE) && tc2_stages<MODE>(G, 2) >= 2 &&
                   (g.mn || ((g.kb_r == 0 || g.kb_r % 128 == 0) &&
                             (!g.has_shared || g.piece_k % 128 == 0)));
  if (g.mn && (mode_fp8(MODE) || !g.kgroup || g.kseg < 1 || g.kseg > 3)) return MOE_ERR_UNSUPPORTED;
  P.kpb = kb2 ? 2 : 1;
  if (!build_maps(g, tc2_two_b(MODE), 128, &P.maps, mode_fp8(MODE) ? 1 : 2, kb2)) return MOE_ERR_CUDA;
  static_assert(tc2_stages<MODE>(1024 + 1) >= 2, "tile list of 1024 experts leaves no room");
  P.stages = tc2_stages<MODE>(G, P.kpb);
  if (P.stages < 2) return MOE_ERR_UNSUPPORTED;
  const size_t smem = tc2_smem_bytes<MODE>(G, P.kpb);
  auto kern = gemm_tc2_kernel<MODE>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
    return MOE_ERR_CUDA;
  const long long bound = tile_bound(g, TC2_BM, C::BN);
  if (bound == 0) return MOE_OK;
  const int pairs = (int)std::min<long long>(num_sms() / 2, bound);
  ProfScope ps(kind, st);
  return launch_pdl(kern, dim3(2 * pairs), dim3(TC_THREADS), smem, st, P);
}

// gate/up and plain products on CTA pairs (256 x 256 tiles; an output width that is not a
// multiple of 256 leaves the last column tile partly outside the expert, whose columns the
// epilogue does not store), the low-rank projection on single SMs (N = rank).
template <int MODE>
moe_status_t launch_gemm(const moe_config_t *c, const GroupedGemm &g, cudaStream_t st,
                         int kind) {
  if (MODE == MODE_SCALE) return launch_tc<MODE_SCALE, 64>(g, st, kind);
  return launch_tc2<MODE == MODE_GATEUP ? MODE_GATEUP : MODE_PLAIN>(g, st, kind);
}

// ------------------------------------------------------------------ steps
#define MOE_TRY(expr)                   \
  do {                                  \
    const moe_status_t _s = (expr);     \
    if (_s != MOE_OK) return _s;        \
  } while (0)

template <typename Tin, int EPT>
moe_status_t launch_router_ept(const RouterArgs &a, cudaStream_t st) {
  const size_t smem =
      router_smem(a.E, a.score == MOE_SCORE_SIGMOID, a.d, (int)sizeof(Tin), EPT).total;
  if (smem > 227 * 1024) return MOE_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(router_kernel<Tin, EPT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return MOE_ERR_CUDA;
  return launch_pdl(router_kernel<Tin, EPT>, dim3(ceil_div(a.T, RT_TM)), dim3(RT_THREADS), smem,
                    st, a);
}

template <typename Tin>
moe_status_t launch_router(const RouterArgs &a, cudaStream_t st) {
  ProfScope ps(K_ROUTER, st);
  if (router_ept(a.E, a.score == MOE_SCORE_SIGMOID, a.d, (int)sizeof(Tin)) == RT_EPT_WIDE)
    return launch_router_ept<Tin, RT_EPT_WIDE>(a, st);
  return launch_router_ept<Tin, RT_EPT>(a, st);
}

moe_status_t launch_stats(const StatsArgs &sa, cudaStream_t st) {
  ProfScope ps(K_STATS, st);
  return launch_pdl(moe_stats_kernel, dim3(sa.E), dim3(ST_THREADS), 0, st, sa);
}

template <typename Tin>
moe_status_t router_only(const moe_config_t *c, const void *x, const moe_weights_t *w,
                         int32_t *idx, float *wts, int32_t *part_cnt, float *part_prob,
                         uint8_t *lrank, cudaStream_t st) {
  RouterArgs a;
  a.x = x;
  a.w = w->w_router;
  a.off = w->logit_offset;
  a.bias = c->score == MOE_SCORE_SIGMOID ? w->select_bias : nullptr;
  a.T = c->T; a.d = c->d; a.E = c->E; a.k = c->top_k; a.score = c->score; a.norm = c->norm_topk;
  a.idx = idx; a.wts = wts;
  a.part_cnt = part_cnt;
  a.part_prob = part_prob;
  a.lrank = lrank;
  return launch_router<Tin>(a, st);
}

StatsArgs stats_args(const moe_config_t *c, const int32_t *chunk_cnt, const float *chunk_prob) {
  StatsArgs sa;
  std::memset(&sa, 0, sizeof(sa));
  sa.chunk_cnt = chunk_cnt;
  sa.chunk_prob = chunk_prob;
  sa.nchunk = ceil_div(c->T, RT_TM);
  sa.E = c->E;
  sa.C = capacity_of(c);
  return sa;
}

template <typename Tin>
moe_status_t route_impl(const moe_config_t *c, const void *x, const moe_weights_t *w,
                        int32_t *idx, float *wts, int32_t *count, float *prob, void *ws,
                        cudaStream_t st) {
  const Layout L = layout_of(c);
  if (c->T == 0) {
    if (cudaMemsetAsync(count, 0, (size_t)c->E * 4, st) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaMemsetAsync(prob, 0, (size_t)c->E * 4, st) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
  }
  int32_t *pc = at<int32_t>(ws, L.part_cnt);
  float *pp = at<float>(ws, L.part_prob);
  MOE_TRY(router_only<Tin>(c, x, w, idx, wts, pc, pp, nullptr, st));
  StatsArgs sa = stats_args(c, pc, pp);
  sa.count_out = count;
  sa.prob_out = prob;
  return launch_stats(sa, st);
}

template <typename Tin>
moe_status_t scatter_impl(const moe_config_t *c, const void *x, const int32_t *idx,
                          const uint8_t *lrank, const int32_t *chunk_base, const int32_t *kept,
                          int32_t *offsets, int32_t *slot_pos, int32_t *src, void *x_perm,
                          const int32_t *count, const float *prob, float *aux, cudaStream_t st) {
  ProfScope ps(K_PERM_SCATTER, st);
  const size_t smem = (size_t)c->E * sizeof(int);  // the expert offsets
  const int grid = std::max(1, std::min(ceil_div(c->T, PM_THREADS / 32),
                                        num_sms() * PM_CTAS_PER_SM));
  return launch_pdl(perm_scatter_kernel<Tin>, dim3(grid), dim3(PM_THREADS), smem, st, idx, lrank,
                    c->T, c->top_k, c->E, capacity_of(c), chunk_base, kept, offsets, slot_pos,
                    src, (const Tin *)x, (Tin *)x_perm, c->d, count, prob, c->aux_alpha, aux);
}

// The scatter of a layer with E4M3 experts: bf16 token rows in, their codes and scales out.
moe_status_t scatter_q8_impl(const moe_config_t *c, const void *x, const int32_t *idx,
                             const uint8_t *lrank, const int32_t *chunk_base, const int32_t *kept,
                             int32_t *offsets, int32_t *slot_pos, int32_t *src, uint8_t *xq_perm,
                             float *sx_perm, const int32_t *count, const float *prob, float *aux,
                             cudaStream_t st) {
  ProfScope ps(K_PERM_SCATTER, st);
  const size_t smem = (size_t)c->E * sizeof(int);
  const int grid = std::max(1, std::min(ceil_div(c->T, PM_THREADS / 32),
                                        num_sms() * PM_CTAS_PER_SM));
  return launch_pdl(perm_scatter_q8_kernel, dim3(grid), dim3(PM_THREADS), smem, st, idx, lrank,
                    c->T, c->top_k, c->E, capacity_of(c), chunk_base, kept, offsets, slot_pos,
                    src, (const __nv_bfloat16 *)x, xq_perm, sx_perm, c->d, count, prob,
                    c->aux_alpha, aux);
}

// Per-row E4M3 quantisation (fp8.cuh) of `rows` rows of `cols` elements.
template <typename Tin>
moe_status_t launch_quantize(const void *in, long long rows, int cols, uint8_t *q, float *scale,
                             cudaStream_t st) {
  if (rows == 0) return MOE_OK;
  const int grid = (int)std::min<long long>((rows + 7) / 8, (long long)num_sms() * 16);
  ProfScope ps(K_QUANT, st);
  return launch_pdl(quantize_rows_kernel<Tin>, dim3(grid), dim3(256), 0, st, (const Tin *)in,
                    rows, cols, q, scale);
}

template <typename Tin>
moe_status_t permute_impl(const moe_config_t *c, const void *x, const int32_t *idx,
                          int32_t *offsets, int32_t *slot_pos, int32_t *src, void *x_perm,
                          void *ws, cudaStream_t st) {
  const Layout L = layout_of(c);
  if (c->T == 0) {
    return cudaMemsetAsync(offsets, 0, (size_t)(c->E + 1) * 4, st) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
  }
  const int nch = ceil_div(c->T, PM_CHUNK);
  int32_t *cc = at<int32_t>(ws, L.chunk_count), *cb = at<int32_t>(ws, L.chunk_base);
  uint8_t *lr = at<uint8_t>(ws, L.lrank);
  {
    const size_t smem = (size_t)8 * c->E * 4;
    if (cudaFuncSetAttribute(perm_hist_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
      return MOE_ERR_CUDA;
    ProfScope ps(K_PERM_HIST, st);
    MOE_TRY(launch_pdl(perm_hist_kernel, dim3(ceil_div(nch, 8)), dim3(256), smem, st, idx, c->T,
                       c->top_k, c->E, cc, lr, nch));
  }
  StatsArgs sa = stats_args(c, cc, nullptr);
  sa.chunk_base = cb;
  sa.kept = at<int32_t>(ws, L.kept);
  MOE_TRY(launch_stats(sa, st));
  return scatter_impl<Tin>(c, x, idx, lr, cb, sa.kept, offsets, slot_pos, src, x_perm, nullptr,
                           nullptr, nullptr, st);
}

// The shared experts of a low-rank layer: SwiGLU gate/up then down over every token.
moe_status_t lowrank_shared_impl(const moe_config_t *c, const GroupedGemm &g, const void *x,
                                 const moe_weights_t *w, void *Hs, void *y_shared,
                                 cudaStream_t st) {
  const int d = c->d, S = c->n_shared, fs = c->ffn_shared;
  GroupedGemm g3 = g;
  g3.E = 0; g3.has_shared = 1;
  g3.A_s = x; g3.lda_s = d; g3.B0_s = w->ws_gate; g3.B1_s = w->ws_up;
  g3.N_s = S * fs; g3.K_s = d; g3.piece_k = d; g3.piece_rows = 0; g3.b_rows_s = S * fs;
  g3.out_s = Hs; g3.ldo_s = S * fs;
  MOE_TRY(launch_gemm<MODE_GATEUP>(c, g3, st, K_GEMM_GATEUP));
  GroupedGemm g4 = g;
  g4.E = 0; g4.has_shared = 1;
  g4.A_s = Hs; g4.lda_s = S * fs; g4.B0_s = w->ws_down; g4.N_s = d; g4.K_s = S * fs;
  g4.piece_k = fs; g4.piece_rows = d; g4.b_rows_s = S * d; g4.out_s = y_shared; g4.ldo_s = d;
  return launch_gemm<MODE_PLAIN>(c, g4, st, K_GEMM_DOWN);
}

// Low-rank experts stored in E4M3 on their grouped rows (codes xq_perm, scales sx_perm):
// z = (xq V8^T) * sx * V_scale * s (fp32 sums on the fp8 tensor cores), quantised per row in the
// same kernel's epilogue (its tile is the whole row: BN = rank) -> zq, sz;
// y_perm = (zq U8^T) * sz * U_scale (fp32). The rank K = r of the second product is completed to
// a 128-element stage by the tensor map's zero fill.
moe_status_t experts_fp8_impl(const moe_config_t *c, const uint8_t *xq_perm, const float *sx_perm,
                              const int32_t *offsets, const void *x, const moe_weights_t *w,
                              void *y_perm, void *y_shared, void *ws, cudaStream_t st) {
  const Layout L = layout_of(c);
  const int T = c->T, d = c->d, E = c->E, k = c->top_k, r = c->rank;
  uint8_t *zq = at<uint8_t>(ws, L.zq);
  float *sz = at<float>(ws, L.sz);
  GroupedGemm g;
  std::memset(&g, 0, sizeof(g));
  g.offsets = offsets;
  g.T = T;
  g.rows_r = T * k;
  GroupedGemm g1 = g;
  g1.E = E; g1.A_r = xq_perm; g1.lda_r = d; g1.B0_r = w->lr_V8; g1.N_r = r; g1.K_r = d;
  g1.out_r = zq; g1.ldo_r = r; g1.out2_r = sz; g1.scale = w->lr_s; g1.row_scale = sx_perm;
  g1.col_scale = w->lr_V_scale;
  switch (r) {  // rank: a multiple of 64 up to 256
    case 64: MOE_TRY((launch_tc<MODE_SCALE_FP8, 64>(g1, st, K_GEMM_LR1))); break;
    case 128: MOE_TRY((launch_tc<MODE_SCALE_FP8, 128>(g1, st, K_GEMM_LR1))); break;
    case 192: MOE_TRY((launch_tc<MODE_SCALE_FP8, 192>(g1, st, K_GEMM_LR1))); break;
    case 256: MOE_TRY((launch_tc<MODE_SCALE_FP8, 256>(g1, st, K_GEMM_LR1))); break;
    default: return MOE_ERR_UNSUPPORTED;
  }
  GroupedGemm g2 = g;
  g2.E = E; g2.A_r = zq; g2.lda_r = r; g2.B0_r = w->lr_U8; g2.N_r = d; g2.K_r = r;
  g2.out_r = y_perm; g2.ldo_r = d; g2.row_scale = sz; g2.col_scale = w->lr_U_scale;
  MOE_TRY(launch_tc2<MODE_PLAIN_FP8>(g2, st, K_GEMM_LR2));
  if (c->n_shared > 0)
    MOE_TRY(lowrank_shared_impl(c, g, x, w, at<char>(ws, L.hidden_sh), y_shared, st));
  return MOE_OK;
}

// fp32 operands as six bf16 K segments (f32split.cuh): rows x cols in, [rows, 6 cols] out.
moe_status_t launch_split6(const void *in, long long rows, int cols, int piece, bool b_operand,
                           void *out, cudaStream_t st) {
  const long long n = rows * cols;
  if (n == 0) return MOE_OK;
  const int grid = (int)std::min<long long>((n + 255) / 256, (long long)num_sms() * 16);
  ProfScope ps(K_SPLIT, st);
  return launch_pdl(split6_bf16_kernel, dim3(grid), dim3(256), 0, st, (const float *)in, rows,
                    cols, piece, b_operand ? 1 : 0, (__nv_bfloat16 *)out);
}

// The fp32 configuration on the tensor cores: every product's operands split into six bf16 K
// segments (x_perm and x, the hidden rows, the weights, each call), the products run over
// K' = 6 K on the bf16 kernels with fp32 hidden rows (gate/up) or z (low-rank) and fp32 outputs.
moe_status_t experts_f32_impl(const moe_config_t *c, const void *x_perm, const int32_t *offsets,
                              const void *x, const moe_weights_t *w, void *y_perm,
                              void *y_shared, void *ws, cudaStream_t st) {
  const Layout L = layout_of(c);
  const int T = c->T, d = c->d, E = c->E, k = c->top_k, S = c->n_shared, fs = c->ffn_shared;
  const int sf = S * fs;
  const bool swi = c->expert == MOE_EXPERT_SWIGLU, sh = S > 0;
  const int hw = swi ? c->ffn : c->rank;  // hidden width: ffn or rank
  void *H = at<char>(ws, L.hidden), *Hs = at<char>(ws, L.hidden_sh);
  void *x6 = at<char>(ws, L.s6_x), *h6 = at<char>(ws, L.s6_h), *w1 = at<char>(ws, L.s6_w1),
       *w1b = at<char>(ws, L.s6_w1b), *w2 = at<char>(ws, L.s6_w2), *xs6 = at<char>(ws, L.s6_xs),
       *hs6 = at<char>(ws, L.s6_hs), *sg6 = at<char>(ws, L.s6_sg), *su6 = at<char>(ws, L.s6_su),
       *sd6 = at<char>(ws, L.s6_sd);
  const long long N = (long long)T * k;
  MOE_TRY(launch_split6(x_perm, N, d, d, false, x6, st));
  if (swi) {
    MOE_TRY(launch_split6(w->w_gate, (long long)E * hw, d, d, true, w1, st));
    MOE_TRY(launch_split6(w->w_up, (long long)E * hw, d, d, true, w1b, st));
    MOE_TRY(launch_split6(w->w_down, (long long)E * d, hw, hw, true, w2, st));
  } else {
    MOE_TRY(launch_split6(w->lr_V, (long long)E * hw, d, d, true, w1, st));
    MOE_TRY(launch_split6(w->lr_U, (long long)E * d, hw, hw, true, w2, st));
  }
  if (sh) {
    MOE_TRY(launch_split6(x, T, d, d, false, xs6, st));
    MOE_TRY(launch_split6(w->ws_gate, sf, d, d, true, sg6, st));
    MOE_TRY(launch_split6(w->ws_up, sf, d, d, true, su6, st));
    MOE_TRY(launch_split6(w->ws_down, (long long)S * d, fs, fs, true, sd6, st));
  }
  GroupedGemm g;
  std::memset(&g, 0, sizeof(g));
  g.offsets = offsets;
  g.T = T;
  g.rows_r = T * k;
  // first products: gate/up (h fp32) with the shared experts' in the same launch, or z = x V^T s
  GroupedGemm g1 = g;
  g1.E = E; g1.A_r = x6; g1.lda_r = 6 * d; g1.K_r = 6 * d; g1.B0_r = w1; g1.N_r = hw;
  g1.out_r = H; g1.ldo_r = hw;
  if (swi) {
    g1.B1_r = w1b;
    g1.has_shared = sh;
    if (sh) {
      g1.A_s = xs6; g1.lda_s = 6 * d; g1.B0_s = sg6; g1.B1_s = su6; g1.N_s = sf; g1.K_s = 6 * d;
      g1.piece_k = 6 * d; g1.piece_rows = 0; g1.b_rows_s = sf; g1.out_s = Hs; g1.ldo_s = sf;
    }
    MOE_TRY(launch_tc2<MODE_GATEUP_F32>(g1, st, K_GEMM_GATEUP));
  } else {
    g1.scale = w->lr_s;
    g1.out_f32 = 1;
    MOE_TRY((launch_tc<MODE_SCALE, 64>(g1, st, K_GEMM_LR1)));
    if (sh) {  // the shared experts' gate/up alone
      GroupedGemm g3 = g;
      g3.E = 0; g3.has_shared = 1;
      g3.A_s = xs6; g3.lda_s = 6 * d; g3.B0_s = sg6; g3.B1_s = su6; g3.N_s = sf; g3.K_s = 6 * d;
      g3.piece_k = 6 * d; g3.piece_rows = 0; g3.b_rows_s = sf; g3.out_s = Hs; g3.ldo_s = sf;
      MOE_TRY(launch_tc2<MODE_GATEUP_F32>(g3, st, K_GEMM_GATEUP));
    }
  }
  // second products: down (or U) over the split hidden rows, the shared down in the same launch
  MOE_TRY(launch_split6(H, N, hw, hw, false, h6, st));
  if (sh) MOE_TRY(launch_split6(Hs, T, sf, fs, false, hs6, st));
  GroupedGemm g2 = g;
  g2.E = E; g2.A_r = h6; g2.lda_r = 6 * hw; g2.K_r = 6 * hw; g2.B0_r = w2; g2.N_r = d;
  g2.out_r = y_perm; g2.ldo_r = d; g2.out_r_bf16 = 0;
  g2.has_shared = sh;
  if (sh) {
    g2.A_s = hs6; g2.lda_s = 6 * sf; g2.B0_s = sd6; g2.N_s = d; g2.K_s = 6 * sf;
    g2.piece_k = 6 * fs; g2.piece_rows = d; g2.b_rows_s = S * d; g2.out_s = y_shared;
    g2.ldo_s = d;
  }
  return launch_tc2<MODE_PLAIN>(g2, st, swi ? K_GEMM_DOWN : K_GEMM_LR2);
}

moe_status_t experts_impl(const moe_config_t *c, const void *x_perm, const int32_t *offsets,
                          const void *x, const moe_weights_t *w, void *y_perm, void *y_shared,
                          void *ws, cudaStream_t st) {
  if (c->T == 0) return MOE_OK;
  if (c->dtype == MOE_DTYPE_F32)
    return experts_f32_impl(c, x_perm, offsets, x, w, y_perm, y_shared, ws, st);
  if (fp8_experts(c)) {  // the bf16 rows quantised first, as the layer quantises its tokens
    const Layout L = layout_of(c);
    uint8_t *xq = at<uint8_t>(ws, L.x_perm);
    float *sxp = at<float>(ws, L.sx_perm);
    MOE_TRY(launch_quantize<__nv_bfloat16>(x_perm, (long long)c->T * c->top_k, c->d, xq, sxp, st));
    return experts_fp8_impl(c, xq, sxp, offsets, x, w, y_perm, y_shared, ws, st);
  }
  const Layout L = layout_of(c);
  const int T = c->T, d = c->d, E = c->E, k = c->top_k, S = c->n_shared, fs = c->ffn_shared;
  void *H = at<char>(ws, L.hidden);
  void *Hs = at<char>(ws, L.hidden_sh);
  GroupedGemm g;
  std::memset(&g, 0, sizeof(g));
  g.offsets = offsets;
  g.T = T;
  g.rows_r = T * k;
  const bool sh = S > 0;
  if (c->expert == MOE_EXPERT_SWIGLU) {
    const int f = c->ffn;
    GroupedGemm g1 = g;
    g1.E = E; g1.A_r = x_perm; g1.lda_r = d; g1.B0_r = w->w_gate; g1.B1_r = w->w_up;
    g1.N_r = f; g1.K_r = d; g1.out_r = H; g1.ldo_r = f;
    g1.has_shared = sh;
    if (sh) {
      g1.A_s = x; g1.lda_s = d; g1.B0_s = w->ws_gate; g1.B1_s = w->ws_up;
      g1.N_s = S * fs; g1.K_s = d; g1.piece_k = d; g1.piece_rows = 0; g1.b_rows_s = S * fs;
      g1.out_s = Hs; g1.ldo_s = S * fs;
    }
    MOE_TRY(launch_gemm<MODE_GATEUP>(c, g1, st, K_GEMM_GATEUP));
    GroupedGemm g2 = g;
    g2.E = E; g2.A_r = H; g2.lda_r = f; g2.B0_r = w->w_down; g2.N_r = d; g2.K_r = f;
    g2.out_r = y_perm; g2.ldo_r = d; g2.out_r_bf16 = yperm_bf16(c) ? 1 : 0;
    g2.has_shared = sh;
    if (sh) {
      g2.A_s = Hs; g2.lda_s = S * fs; g2.B0_s = w->ws_down; g2.N_s = d; g2.K_s = S * fs;
      g2.piece_k = fs; g2.piece_rows = d; g2.b_rows_s = S * d; g2.out_s = y_shared; g2.ldo_s = d;
    }
    return launch_gemm<MODE_PLAIN>(c, g2, st, K_GEMM_DOWN);
  }
  // low-rank experts: Z = (X V^T) * s, then Y = Z U^T. In bf16, Z is kept as two bf16 terms
  // [Z_hi | Z_lo] (Z_lo = the rounding residual), and the second product runs over K = 2r with
  // the k loop wrapping over U's r columns: Y = Z_hi U^T + Z_lo U^T, i.e. Z at ~2^-17 relative
  // precision for twice the (small) flops of that product.
  const int r = c->rank;
  const bool split = c->dtype == MOE_DTYPE_BF16;
  GroupedGemm g1 = g;
  g1.E = E; g1.A_r = x_perm; g1.lda_r = d; g1.B0_r = w->lr_V; g1.N_r = r; g1.K_r = d;
  g1.out_r = H; g1.ldo_r = split ? 2 * r : r; g1.scale = w->lr_s; g1.lo_split = split ? r : 0;
  MOE_TRY(launch_gemm<MODE_SCALE>(c, g1, st, K_GEMM_LR1));
  GroupedGemm g2 = g;
  g2.E = E; g2.A_r = H; g2.lda_r = split ? 2 * r : r; g2.B0_r = w->lr_U; g2.N_r = d;
  g2.K_r = split ? 2 * r : r; g2.kb_r = split ? r : 0;
  g2.out_r = y_perm; g2.ldo_r = d; g2.out_r_bf16 = yperm_bf16(c) ? 1 : 0;
  MOE_TRY(launch_gemm<MODE_PLAIN>(c, g2, st, K_GEMM_LR2));
  if (sh) MOE_TRY(lowrank_shared_impl(c, g, x, w, Hs, y_shared, st));
  return MOE_OK;
}

// early: slot_pos and wts were written at least two kernels back in the stream (combine.cuh).
moe_status_t combine_impl(const moe_config_t *c, const void *y_perm, const void *y_shared,
                          const int32_t *slot_pos, const float *wts, void *y, cudaStream_t st,
                          bool early) {
  if (c->T == 0) return MOE_OK;
  ProfScope ps(K_COMBINE, st);
  const float *ysh = c->n_shared > 0 ? (const float *)y_shared : nullptr;
  if (yperm_bf16(c))
    return launch_pdl(combine_kernel<__nv_bfloat16>, dim3(ceil_div(c->T, 8)), dim3(256), 0, st,
                      (const __nv_bfloat16 *)y_perm, ysh, slot_pos, wts, (float *)y, c->T,
                      c->top_k, c->d, early);
  return launch_pdl(combine_kernel<float>, dim3(ceil_div(c->T, 8)), dim3(256), 0, st,
                    (const float *)y_perm, ysh, slot_pos, wts, (float *)y, c->T, c->top_k, c->d,
                    early);
}

moe_status_t aux_impl(const moe_config_t *c, const int32_t *count, const float *prob, float *loss,
                      cudaStream_t st) {
  ProfScope ps(K_AUX, st);
  return launch_pdl(aux_loss_kernel, dim3(1), dim3(32), 0, st, count, prob, c->E, c->T, c->top_k,
                    c->aux_alpha, loss);
}

#include "backward_lib.cuh"

// ------------------------------------------------------------------ argument checks
moe_status_t check_cfg(const moe_config_t *c) {
  if (!c) return MOE_ERR_INVALID_ARG;
  return cfg_supported(c) ? MOE_OK : MOE_ERR_UNSUPPORTED;
}
moe_status_t check_ws(const moe_config_t *c, void *ws, size_t bytes) {
  if (!aligned16(ws)) return MOE_ERR_INVALID_ARG;
  return bytes >= layout_of(c).total ? MOE_OK : MOE_ERR_WORKSPACE;
}
inline bool aligned4_or_null(const void *p) { return ((uintptr_t)p & 3u) == 0; }
moe_status_t check_weights(const moe_config_t *c, const moe_weights_t *w, bool router,
                           bool experts) {
  if (!w) return MOE_ERR_INVALID_ARG;
  if (router && !aligned16(w->w_router)) return MOE_ERR_INVALID_ARG;
  if (router && (!aligned4_or_null(w->logit_offset) || !aligned4_or_null(w->select_bias)))
    return MOE_ERR_INVALID_ARG;
  if (experts) {
    if (c->expert == MOE_EXPERT_SWIGLU) {
      if (!aligned16(w->w_gate) || !aligned16(w->w_up) || !aligned16(w->w_down)) return MOE_ERR_INVALID_ARG;
    } else if (fp8_experts(c)) {
      if (!aligned16(w->lr_V8) || !aligned16(w->lr_U8) || !aligned16(w->lr_s) ||
          !aligned16(w->lr_V_scale) || !aligned16(w->lr_U_scale))
        return MOE_ERR_INVALID_ARG;
    } else {
      if (!aligned16(w->lr_V) || !aligned16(w->lr_U) || !aligned16(w->lr_s)) return MOE_ERR_INVALID_ARG;
    }
    if (c->n_shared > 0 && (!aligned16(w->ws_gate) || !aligned16(w->ws_up) || !aligned16(w->ws_down)))
      return MOE_ERR_INVALID_ARG;
  }
  return MOE_OK;
}

#define MOE_REQUIRE(cond) \
  do {                    \
    if (!(cond)) return MOE_ERR_INVALID_ARG; \
  } while (0)

}  // namespace

// ================================================================== C ABI
extern "C" {

size_t moe_workspace_size(const moe_config_t *cfg) {
  if (check_cfg(cfg) != MOE_OK) return 0;
  return layout_of(cfg).total;
}

int32_t moe_capacity(const moe_config_t *cfg) {
  if (check_cfg(cfg) != MOE_OK) return -2;
  return capacity_of(cfg);
}

moe_status_t moe_route(const moe_config_t *cfg, const void *x, const moe_weights_t *w,
                       int32_t *topk_idx, float *topk_w, int32_t *expert_count, float *prob_sum,
                       void *ws, size_t ws_bytes, void *stream) {
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(check_weights(cfg, w, true, false));
  MOE_REQUIRE(tok16(cfg, x) && tok16(cfg, topk_idx) && tok16(cfg, topk_w) &&
              aligned16(expert_count) && aligned16(prob_sum));
  MOE_TRY(check_ws(cfg, ws, ws_bytes));
  cudaStream_t st = (cudaStream_t)stream;
  if (cfg->dtype == MOE_DTYPE_BF16)
    return route_impl<__nv_bfloat16>(cfg, x, w, topk_idx, topk_w, expert_count, prob_sum, ws, st);
  return route_impl<float>(cfg, x, w, topk_idx, topk_w, expert_count, prob_sum, ws, st);
}

moe_status_t moe_permute(const moe_config_t *cfg, const void *x, const int32_t *topk_idx,
                         int32_t *offsets, int32_t *slot_pos, int32_t *src_token, void *x_perm,
                         void *ws, size_t ws_bytes, void *stream) {
  MOE_TRY(check_cfg(cfg));
  MOE_REQUIRE(tok16(cfg, x) && tok16(cfg, topk_idx) && aligned16(offsets) && tok16(cfg, slot_pos) &&
              tok16(cfg, src_token) && (x_perm == nullptr || aligned16(x_perm)));
  MOE_TRY(check_ws(cfg, ws, ws_bytes));
  cudaStream_t st = (cudaStream_t)stream;
  if (cfg->dtype == MOE_DTYPE_BF16)
    return permute_impl<__nv_bfloat16>(cfg, x, topk_idx, offsets, slot_pos, src_token, x_perm, ws, st);
  return permute_impl<float>(cfg, x, topk_idx, offsets, slot_pos, src_token, x_perm, ws, st);
}

moe_status_t moe_expert_forward(const moe_config_t *cfg, const void *x_perm,
                                const int32_t *offsets, const void *x, const moe_weights_t *w,
                                void *y_perm, void *y_shared, void *ws, size_t ws_bytes,
                                void *stream) {
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(check_weights(cfg, w, false, true));
  MOE_REQUIRE(tok16(cfg, x_perm) && aligned16(offsets) && tok16(cfg, x) && tok16(cfg, y_perm));
  MOE_REQUIRE(cfg->n_shared == 0 || tok16(cfg, y_shared));
  MOE_TRY(check_ws(cfg, ws, ws_bytes));
  return experts_impl(cfg, x_perm, offsets, x, w, y_perm, y_shared, ws, (cudaStream_t)stream);
}

moe_status_t moe_combine(const moe_config_t *cfg, const void *y_perm, const void *y_shared,
                         const int32_t *slot_pos, const float *topk_w, void *y, void *stream) {
  MOE_TRY(check_cfg(cfg));
  MOE_REQUIRE(tok16(cfg, y_perm) && tok16(cfg, slot_pos) && tok16(cfg, topk_w) && tok16(cfg, y));
  MOE_REQUIRE(cfg->n_shared == 0 || tok16(cfg, y_shared));
  return combine_impl(cfg, y_perm, y_shared, slot_pos, topk_w, y, (cudaStream_t)stream, false);
}

#include "backward_api.cuh"

moe_status_t moe_aux_loss(const moe_config_t *cfg, const int32_t *expert_count,
                          const float *prob_sum, float *loss, void *stream) {
  MOE_TRY(check_cfg(cfg));
  MOE_REQUIRE(aligned16(expert_count) && aligned16(prob_sum) && loss != nullptr);
  return aux_impl(cfg, expert_count, prob_sum, loss, (cudaStream_t)stream);
}

moe_status_t moe_bias_update(const moe_config_t *cfg, const int32_t *expert_count,
                             float *select_bias, float u, void *stream) {
  MOE_TRY(check_cfg(cfg));
  MOE_REQUIRE(aligned16(expert_count) && aligned16(select_bias) && std::isfinite(u));
  return launch_pdl(bias_update_kernel, dim3(1), dim3(256), 0, (cudaStream_t)stream,
                    expert_count, select_bias, cfg->E, u);
}

moe_status_t moe_layer_forward(const moe_config_t *cfg, const void *x, const moe_weights_t *w,
                               void *y, float *aux_loss, int32_t *expert_count, void *ws,
                               size_t ws_bytes, void *stream) {
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(check_weights(cfg, w, true, true));
  MOE_REQUIRE(tok16(cfg, x) && tok16(cfg, y));
  MOE_REQUIRE(expert_count == nullptr || aligned16(expert_count));
  MOE_TRY(check_ws(cfg, ws, ws_bytes));
  const Layout L = layout_of(cfg);
  cudaStream_t st = (cudaStream_t)stream;
  int32_t *idx = at<int32_t>(ws, L.idx);
  float *wts = at<float>(ws, L.wts);
  int32_t *cnt = expert_count ? expert_count : at<int32_t>(ws, L.count);
  float *prob = at<float>(ws, L.prob);
  int32_t *offsets = at<int32_t>(ws, L.offsets);
  int32_t *slot_pos = at<int32_t>(ws, L.slot_pos);
  int32_t *src = at<int32_t>(ws, L.src);
  void *x_perm = at<char>(ws, L.x_perm);
  void *y_perm = at<char>(ws, L.y_perm);
  void *y_sh = at<char>(ws, L.y_shared);
  float *aux = aux_loss ? aux_loss : at<float>(ws, L.aux);
  if (cfg->T == 0) {
    if (cudaMemsetAsync(cnt, 0, (size_t)cfg->E * 4, st) != cudaSuccess) return MOE_ERR_CUDA;
    return cudaMemsetAsync(aux, 0, 4, st) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
  }
  // route -> statistics (counts, probability sums, chunk scans, kept counts) -> scatter
  // (offsets, loss, positions, rows)
  int32_t *pc = at<int32_t>(ws, L.part_cnt);
  float *pp = at<float>(ws, L.part_prob);
  int32_t *cb = at<int32_t>(ws, L.chunk_base);
  uint8_t *lr = at<uint8_t>(ws, L.lrank);
  const bool f8 = fp8_experts(cfg);
  float *sxp = at<float>(ws, L.sx_perm);
  if (cfg->dtype == MOE_DTYPE_BF16)
    MOE_TRY(router_only<__nv_bfloat16>(cfg, x, w, idx, wts, pc, pp, lr, st));
  else
    MOE_TRY(router_only<float>(cfg, x, w, idx, wts, pc, pp, lr, st));
  StatsArgs sa = stats_args(cfg, pc, pp);
  sa.count_out = cnt;
  sa.prob_out = prob;
  sa.chunk_base = cb;
  sa.kept = at<int32_t>(ws, L.kept);
  MOE_TRY(launch_stats(sa, st));
  if (f8)  // the token rows quantised on their way to the experts' rows
    MOE_TRY(scatter_q8_impl(cfg, x, idx, lr, cb, sa.kept, offsets, slot_pos, src,
                            (uint8_t *)x_perm, sxp, cnt, prob, aux, st));
  else if (cfg->dtype == MOE_DTYPE_BF16)
    MOE_TRY(scatter_impl<__nv_bfloat16>(cfg, x, idx, lr, cb, sa.kept, offsets, slot_pos, src,
                                        x_perm, cnt, prob, aux, st));
  else
    MOE_TRY(scatter_impl<float>(cfg, x, idx, lr, cb, sa.kept, offsets, slot_pos, src, x_perm,
                                cnt, prob, aux, st));
  // T > 0 here: the expert forward launched at least two kernels after the scatter
  if (f8)
    MOE_TRY(experts_fp8_impl(cfg, (const uint8_t *)x_perm, sxp, offsets, x, w, y_perm, y_sh, ws,
                             st));
  else
    MOE_TRY(experts_impl(cfg, x_perm, offsets, x, w, y_perm, y_sh, ws, st));
  return combine_impl(cfg, y_perm, y_sh, slot_pos, wts, y, st, true);
}

moe_status_t moe_quantize_fp8(const void *in, int32_t in_dtype, int64_t rows, int32_t cols,
                              uint8_t *q, float *scale, void *stream) {
  if (rows < 0 || cols <= 0) return MOE_ERR_INVALID_ARG;
  if (cols % 16 || (in_dtype != MOE_DTYPE_BF16 && in_dtype != MOE_DTYPE_F32) ||
      rows * (long long)cols >= (1ll << 40))
    return MOE_ERR_UNSUPPORTED;
  if (rows == 0) return MOE_OK;
  MOE_REQUIRE(aligned16(in) && aligned16(q) && aligned16(scale));
  cudaStream_t st = (cudaStream_t)stream;
  if (in_dtype == MOE_DTYPE_BF16) return launch_quantize<__nv_bfloat16>(in, rows, cols, q, scale, st);
  return launch_quantize<float>(in, rows, cols, q, scale, st);
}

const char *moe_status_str(moe_status_t s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_INVALID_ARG: return "MOE_ERR_INVALID_ARG: null or misaligned pointer";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED: shape or option outside the supported set";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE: workspace smaller than moe_workspace_size()";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA: a CUDA runtime call failed";
    case MOE_ERR_TIMEOUT: return "MOE_ERR_TIMEOUT: a bounded device-side wait ran out";
    case MOE_ERR_DEVICE_CHECK: return "MOE_ERR_DEVICE_CHECK: a device-side check failed";
  }
  return "unknown moe_status_t";
}

moe_status_t moe_get_device_error(void *stream, int64_t *info) {
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return MOE_ERR_CUDA;
  int code = 0;
  long long inf = 0;
  if (cudaMemcpyFromSymbol(&code, g_err_code, sizeof(int)) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaMemcpyFromSymbol(&inf, g_err_info, sizeof(long long)) != cudaSuccess) return MOE_ERR_CUDA;
  const int zero = 0;
  const long long zero64 = 0;
  cudaMemcpyToSymbol(g_err_code, &zero, sizeof(int));
  cudaMemcpyToSymbol(g_err_info, &zero64, sizeof(long long));
  if (info) *info = inf;
  return (moe_status_t)code;
}

moe_status_t moe_debug_set(int32_t what, int64_t value) {
  switch (what) {
    case MOE_DEBUG_FORCE_EXACT: {
      if (value < 0 || value > 2) return MOE_ERR_INVALID_ARG;
      const int v = (int)value;
      return cudaMemcpyToSymbol(g_force_exact, &v, sizeof(int)) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
    }
    case MOE_DEBUG_WAIT_LIMIT_NS: {
      if (value <= 0) return MOE_ERR_INVALID_ARG;
      const unsigned long long v = (unsigned long long)value;
      return cudaMemcpyToSymbol(g_wait_limit_ns, &v, sizeof(v)) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
    }
    case MOE_DEBUG_STAMP: {
      const int v = value != 0;
      if (stamp_reset() != MOE_OK) return MOE_ERR_CUDA;
      return cudaMemcpyToSymbol(g_stamp_on, &v, sizeof(int)) == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
    }
    case MOE_DEBUG_PROFILE: {
      std::lock_guard<std::mutex> lk(g_prof_mu);
      if (value && !g_prof.created) {
        for (int i = 0; i < 2 * PROF_SLOTS; ++i)
          if (cudaEventCreate(&g_prof.ev[i]) != cudaSuccess) return MOE_ERR_CUDA;
        g_prof.created = true;
      }
      g_prof.on = value != 0;
      g_prof.n = 0;
      return MOE_OK;
    }
  }
  return MOE_ERR_INVALID_ARG;
}

int32_t moe_stamp_read(const char **names, double *us, int32_t max) {
  if (cudaDeviceSynchronize() != cudaSuccess) return -1;
  static unsigned long long h[K_COUNT][STAMP_SLOTS][2];
  if (cudaMemcpyFromSymbol(h, g_stamp, sizeof(h)) != cudaSuccess) return -1;
  if (stamp_reset() != MOE_OK) return -1;
  int out = 0;
  for (int k = 0; k < K_COUNT; ++k) {
    unsigned long long t0 = ~0ull, t1 = 0ull;
    for (int sl = 0; sl < STAMP_SLOTS; ++sl) {
      t0 = std::min(t0, h[k][sl][0]);
      t1 = std::max(t1, h[k][sl][1]);
    }
    if (t0 == ~0ull || t1 <= t0) continue;
    if (out < max) {
      if (names) names[out] = kKindName[k];
      if (us) us[out] = (double)(t1 - t0) * 1e-3;
    }
    ++out;
  }
  return out;
}

int32_t moe_profile_read(const char **names, double *total_ms, int64_t *launches, int32_t max) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  if (!g_prof.created) return 0;
  cudaDeviceSynchronize();
  double ms[K_COUNT] = {0};
  long long n[K_COUNT] = {0};
  for (int i = 0; i < g_prof.n; ++i) {
    float t = 0.0f;
    if (cudaEventElapsedTime(&t, g_prof.ev[2 * i], g_prof.ev[2 * i + 1]) == cudaSuccess) {
      ms[g_prof.kind[i]] += t;
      n[g_prof.kind[i]] += 1;
    }
  }
  g_prof.n = 0;
  int out = 0;
  for (int k = 0; k < K_COUNT; ++k) {
    if (!n[k]) continue;
    if (out < max) {
      if (names) names[out] = kKindName[k];
      if (total_ms) total_ms[out] = ms[k];
      if (launches) launches[out] = n[k];
    }
    ++out;
  }
  return out;
}

}  // extern "C"

namespace moe {
__global__ void wait_probe_kernel() {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  // nothing ever arrives on `bar`: the bounded wait must expire and record MOE_ERR_TIMEOUT
  if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0u, &abort_flag, g_wait_limit_ns, INFO_WAIT_PROBE);
}
}  // namespace moe

extern "C" moe_status_t moe_debug_wait_timeout_probe(void *stream) {
  moe::wait_probe_kernel<<<1, 32, 0, (cudaStream_t)stream>>>();
  return last_launch_status();
}

// ================================================================== moe_route_noalloc
// The router's scratch (the per-CTA partial statistics) placed in a fixed array of the library's
// own device memory instead of a caller workspace. Host code must not use the array's name as a
// device pointer: it is a host stand-in for the symbol, so its device address is looked up per
// device (and per context of that device) below.
namespace {

static __device__ __align__(256) unsigned char g_route_scratch[MOE_ROUTE_NOALLOC_SCRATCH_BYTES];

// Per device: the array's address and the id of the context it was looked up in. A context
// made anew on the device (after cudaDeviceReset, for example) may load the module at another
// address, so the address is looked up again whenever the current context's id differs.
struct ScratchAddr {
  void *ptr = nullptr;
  unsigned long long ctx_id = 0;
};
ScratchAddr g_route_scratch_dev[64];
std::mutex g_route_scratch_mu;

// Unique id of the calling thread's current context (driver entry points, looked up once).
moe_status_t current_context_id(unsigned long long *id) {
  using GetCurrent = CUresult (*)(CUcontext *);
  using GetId = CUresult (*)(CUcontext, unsigned long long *);
  static GetCurrent get_current = nullptr;
  static GetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void *f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = (GetCurrent)f;
    f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = (GetId)f;
  });
  if (!get_current || !get_id) return MOE_ERR_CUDA;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return MOE_ERR_CUDA;
  return get_id(ctx, id) == CUDA_SUCCESS ? MOE_OK : MOE_ERR_CUDA;
}

// Device address of g_route_scratch on the current device, looked up (with that device current)
// on the first call there and again when the device's context has been made anew.
moe_status_t route_scratch_address(void **out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (dev < 0 || dev >= 64) return MOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_route_scratch_mu);
  ScratchAddr &a = g_route_scratch_dev[dev];
  unsigned long long ctx_id = 0;
  const bool have_id = current_context_id(&ctx_id) == MOE_OK;  // false: no context yet
  if (a.ptr == nullptr || !have_id || a.ctx_id != ctx_id) {
    void *p = nullptr;
    // initialises the device's primary context when none is current on this thread
    const cudaError_t e = cudaGetSymbolAddress(&p, g_route_scratch);
    if (e != cudaSuccess || p == nullptr) return MOE_ERR_CUDA;
    if (!have_id) MOE_TRY(current_context_id(&ctx_id));
    a.ptr = p;
    a.ctx_id = ctx_id;
  }
  *out = a.ptr;
  return MOE_OK;
}

struct RouteScratch {
  size_t part_cnt, part_prob, total;
};

RouteScratch route_scratch_layout(const moe_config_t *c) {
  RouteScratch L;
  const size_t E = c->E;
  const size_t nblk = std::max<size_t>(1, ceil_div(c->T, RT_TM));
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t at = o; o = align256(o + std::max<size_t>(bytes, 1)); return at; };
  L.part_cnt = take(nblk * E * 4);
  L.part_prob = take(nblk * E * 4);
  L.total = o;
  return L;
}

template <typename Tin>
moe_status_t route_noalloc_impl(const moe_config_t *c, const void *x, const moe_weights_t *w,
                                int32_t *idx, float *wts, int32_t *count, float *prob,
                                char *scratch, cudaStream_t st) {
  const RouteScratch L = route_scratch_layout(c);
  if (c->T == 0) {
    if (cudaMemsetAsync(count, 0, (size_t)c->E * 4, st) != cudaSuccess) return MOE_ERR_CUDA;
    if (cudaMemsetAsync(prob, 0, (size_t)c->E * 4, st) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
  }
  // every call rewrites the per-CTA partials before reading them, so nothing left in the
  // array by an earlier call is read
  int32_t *pc = (int32_t *)(scratch + L.part_cnt);
  float *pp = (float *)(scratch + L.part_prob);
  MOE_TRY(router_only<Tin>(c, x, w, idx, wts, pc, pp, nullptr, st));
  StatsArgs sa = stats_args(c, pc, pp);
  sa.count_out = count;
  sa.prob_out = prob;
  return launch_stats(sa, st);
}

}  // namespace

extern "C" moe_status_t moe_route_noalloc(const moe_config_t *cfg, const void *x,
                                          const moe_weights_t *w, int32_t *topk_idx,
                                          float *topk_w, int32_t *expert_count, float *prob_sum,
                                          void *stream) {
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(check_weights(cfg, w, true, false));
  MOE_REQUIRE(tok16(cfg, x) && tok16(cfg, topk_idx) && tok16(cfg, topk_w) &&
              aligned16(expert_count) && aligned16(prob_sum));
  if (route_scratch_layout(cfg).total > MOE_ROUTE_NOALLOC_SCRATCH_BYTES) return MOE_ERR_WORKSPACE;
  void *scratch = nullptr;
  MOE_TRY(route_scratch_address(&scratch));
  cudaStream_t st = (cudaStream_t)stream;
  if (cfg->dtype == MOE_DTYPE_BF16)
    return route_noalloc_impl<__nv_bfloat16>(cfg, x, w, topk_idx, topk_w, expert_count, prob_sum,
                                             (char *)scratch, st);
  return route_noalloc_impl<float>(cfg, x, w, topk_idx, topk_w, expert_count, prob_sum,
                                   (char *)scratch, st);
}

// Shared device-side helpers of the MoE library (one translation unit: moe_lib.cu).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/moe.h"

namespace moe {

// ------------------------------------------------------------------ device error word
// First error wins; the host reads and clears it with moe_get_device_error().
__device__ int g_err_code = 0;
__device__ long long g_err_info = 0;
__device__ int g_force_exact = 0;  // 0 off; 1 every logit/key via the exact paths; 2 also skip the integer path
__device__ unsigned long long g_wait_limit_ns = 2000000000ull;

// detail codes stored in g_err_info
enum : long long {
  INFO_SIGMOID_UNRESOLVED = 1,
  INFO_EXPANSION_OVERFLOW = 2,
  INFO_WAIT_TMA_FULL = 10,
  INFO_WAIT_MMA_EMPTY = 11,
  INFO_WAIT_ACC_FULL = 12,
  INFO_WAIT_ACC_EMPTY = 13,
  INFO_WAIT_DRAIN = 14,
  INFO_WAIT_ROUTER_X = 15,
  INFO_WAIT_SCATTER = 16,
  INFO_WAIT_PROBE = 20,
};

__device__ __forceinline__ void set_device_error(int code, long long info) {
  if (atomicCAS(&g_err_code, 0, code) == 0) g_err_info = info;
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ------------------------------------------------------------------ kernel kinds and stamps
// Kinds of the library's forward kernels (the host's profiler and the device stamps share them).
enum KernelKind {
  K_ROUTER, K_STATS, K_PERM_HIST, K_PERM_SCATTER, K_GEMM_GATEUP, K_GEMM_DOWN, K_GEMM_LR1,
  K_GEMM_LR2, K_COMBINE, K_AUX, K_BWD_GEMM, K_QUANT, K_SPLIT, K_COUNT
};

// In-step timestamps. With stamping on (moe_debug_set(MOE_DEBUG_STAMP, 1)) a kernel records, per
// kind, the global-timer time at which its first CTA passed griddep_wait (its inputs final) and
// the time its last warp finished, as a min / max over 32 slots (CTA index mod 32) to spread the
// atomics. Unlike CUDA events around each launch, this leaves programmatic dependent launch in
// place, so a kernel is measured as it runs inside the layer call.
constexpr int STAMP_SLOTS = 32;
__device__ int g_stamp_on = 0;
__device__ unsigned long long g_stamp[K_COUNT][STAMP_SLOTS][2];

struct KernelStamp {
  int kind;
  bool on;
  __device__ __forceinline__ explicit KernelStamp(int k) : kind(k), on(g_stamp_on != 0) {}
  __device__ __forceinline__ void started() const {
    if (on && threadIdx.x == 0)
      atomicMin(&g_stamp[kind][blockIdx.x & (STAMP_SLOTS - 1)][0], globaltimer_ns());
  }
  __device__ __forceinline__ ~KernelStamp() {
    if (on && (threadIdx.x & 31) == 0)
      atomicMax(&g_stamp[kind][blockIdx.x & (STAMP_SLOTS - 1)][1], globaltimer_ns());
  }
};

// ------------------------------------------------------------------ element conversion
template <typename T> struct Elem;
template <> struct Elem<float> {
  static __device__ __forceinline__ float to_f(float v) { return v; }
  static __device__ __forceinline__ float from_f(float v) { return v; }
};
template <> struct Elem<__nv_bfloat16> {
  static __device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
  static __device__ __forceinline__ __nv_bfloat16 from_f(float v) { return __float2bfloat16_rn(v); }
};

// ------------------------------------------------------------------ warp helpers
__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

__device__ __forceinline__ float warp_sum_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max_f(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Inclusive warp scan of ints.
__device__ __forceinline__ int warp_incl_scan(int v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int n = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += n;
  }
  return v;
}

// Exclusive scan of `n` ints in shared memory `a` (in place) by the whole block; returns total.
// blockDim.x must be a multiple of 32. `tmp` needs blockDim.x/32 + 1 ints.
__device__ int block_excl_scan_inplace(int *a, int n, int *tmp) {
  const int tid = threadIdx.x, nt = blockDim.x;
  const int per = (n + nt - 1) / nt;
  const int lo = min(n, tid * per), hi = min(n, lo + per);
  int s = 0;
  for (int i = lo; i < hi; ++i) s += a[i];
  int incl = warp_incl_scan(s);
  const int warp = tid >> 5, lane = tid & 31;
  if (lane == 31) tmp[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int nw = nt >> 5;
    int v = lane < nw ? tmp[lane] : 0;
    int vi = warp_incl_scan(v);
    if (lane < nw) tmp[lane] = vi - v;
    if (lane == 31) tmp[nw] = vi;
  }
  __syncthreads();
  int run = tmp[warp] + incl - s;
  for (int i = lo; i < hi; ++i) {
    int v = a[i];
    a[i] = run;
    run += v;
  }
  int total = tmp[nt >> 5];
  __syncthreads();
  return total;
}

// ---------------------------------------------------------------- clusters
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// All threads of every CTA in the cluster; release / acquire ordering of shared-memory writes.
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.aligned;\n\tbarrier.cluster.wait.aligned;" ::: "memory");
}
// Generic address of the same shared-memory object in CTA `rank` of this cluster.
template <typename T> __device__ __forceinline__ T *cluster_map(T *p, uint32_t rank) {
  uint64_t out;
  asm volatile("mapa.u64 %0, %1, %2;" : "=l"(out) : "l"((uint64_t)p), "r"(rank));
  return (T *)out;
}

// ---------------------------------------------------------------- programmatic dependent launch
// The library launches its kernels with programmatic stream serialisation: a kernel may be
// scheduled while the previous kernel of the stream is still finishing. griddep_wait() returns
// once that kernel has completed and its memory operations are visible; every kernel calls it
// before its first access to global memory that an earlier kernel may write or read (set-up of
// shared memory, barriers and TMEM may precede it). griddep_launch() allows the next kernel to
// be scheduled. Both are no-ops for a kernel launched without the attribute.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// 32 contiguous bytes to global memory in one store (dst 32-byte aligned): a whole L2 sector, so
// the sector is never written in halves.
__device__ __forceinline__ void st_global_32B(void *dst, const uint32_t (&v)[8]) {
  asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(dst), "r"(v[0]),
               "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7])
               : "memory");
}

// ---------------------------------------------------------------- mbarriers (shared memory)
// 1-D bulk copy shared -> global, tracked by the issuing thread's bulk group. src, dst 16-byte
// aligned; bytes a multiple of 16. bulk_store_commit_wait_read() returns when every store the
// thread issued has finished reading shared memory (the buffer may then be reused).
__device__ __forceinline__ void bulk_store_1d(void *dst, uint32_t src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(src),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_store_commit_wait_read() {
  asm volatile("cp.async.bulk.commit_group;\n\tcp.async.bulk.wait_group.read 0;" ::: "memory");
}
// 1-D bulk copy global -> this CTA's shared memory, counted on an mbarrier (complete_tx).
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_load_1d(uint32_t dst, const void *src, uint32_t bytes,
                                             uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(dst), "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// 16-byte asynchronous copy global -> shared through L2 (bypassing L1), in commit groups that a
// thread waits for itself.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N> __device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
// Bounded wait: true when the phase of `parity` completed; false on timeout or abort.
__device__ __noinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                       uint64_t limit_ns, long long info) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (globaltimer_ns() - t0 > limit_ns) {
      set_device_error(MOE_ERR_TIMEOUT, info);
      *abort_flag = 1;
      return false;
    }
  }
}

}  // namespace moe

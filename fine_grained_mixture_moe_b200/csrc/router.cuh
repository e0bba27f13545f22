// Router: logits, selection keys, top-k, combine weights and per-expert statistics.
//
// What it computes (Quartz: softmax router, 6 of 24 experts; Moonfrost expert card: top-3
// routing; Sutra-1.3B: top-4 by sigmoid score plus a per-expert balancing bias):
//   l[t,e]  = RN32(exact sum_i x[t,i] W[e,i] + off[e])              (fp32, canonical)
//   key     = l  (softmax)  |  RN32(exact sigmoid(l) + b[e])  (sigmoid + selection bias)
//   top-k by key, ties -> lower expert index, slot order = descending key
//   weights = softmax over all E (or sigmoid) of the selected experts, optional renormalise
//
// How. The integer results (which experts, in which slot order) depend only on the order of the
// k+1 largest canonical keys, so the kernel computes every logit approximately and proves the
// order, falling back to exact arithmetic only where the proof fails:
//   1. screen: fp32 dot products on the CUDA cores with packed two-lane fused multiply-adds.
//      A product is exact inside its FMA, so each term passes through at most
//      m = 4 ceil(d/128) + 10 roundings and |l~ - l| <= gamma_m (|x_t|_2 max_e |W_e|_2 + max|off|)
//      =: B_t for every expert of token t (norms from fp32 sums of squares, bounded above);
//   2. proof: if each of the k gaps between consecutive keys of the approximate top k+1 exceeds
//      twice the key bound plus two fp32 steps, the canonical keys of those k+1 experts lie in
//      the same strict order and above every other expert's, so the approximate selection is
//      the exact one;
//   3. otherwise (about 1% of Quartz tokens) every expert whose key could still reach the top k
//      (within that margin of the (k+1)-th key) gets its canonical logit: an fp64 sum of the exact
//      products (error <= (d+16) 2^-52 (|x||W_e| + |off|)) rounded directly when no fp32 rounding
//      boundary lies inside the error, else decided by an exact integer comparison with the
//      boundaries (or, for exponent spans beyond 50 bits, a floating-point expansion). The other
//      experts provably stay below the k-th canonical key, and selection reruns on the mix.
// Sigmoid keys are screened from the approximate logit (sigmoid is 1/4-Lipschitz) and, for the
// candidates of step 3, resolved exactly in double-double. Combine weights and probability sums
// use the logits as computed: within B_t of canonical, far inside their tolerance.
#pragma once
#include "common.cuh"

namespace moe {

constexpr int RT_TM = 16;          // tokens per CTA
constexpr int RT_WARPS = 8;        // each takes every 8th slice of the d dimension
constexpr int RT_THREADS = 32 * RT_WARPS;
// Screen tiling. Lane = ks + 2 (eg + 8 tg): tg in {0,1} picks tokens tg, tg+2, ..., tg+14;
// eg in 0..7 picks experts eg, eg+8, ... of the round; ks in {0,1} halves the warp's d slice.
constexpr int RT_TPT = 8;          // tokens per thread
constexpr int RT_EPT = 3;          // experts per thread (6 in the wide form for many experts)
constexpr int RT_EPT_WIDE = 6;
constexpr int RT_WIDE_MIN_E = 97;  // the wide form from this many experts, when it fits
constexpr int RT_SEL_THREAD_MAX_E = 64;  // ranking: up to this many experts a thread counts the
                                         // rank of one (token, expert) pair; above, a warp per
                                         // token takes the largest keys in turn
constexpr int EXPANSION_MAX = 40;

struct RouterArgs {
  const void *x;
  const void *w;        // [E, d] router weight in the input dtype
  const float *off;     // [E] or null
  const float *bias;    // [E] or null
  int T, d, E, k, score, norm;
  int32_t *idx;
  float *wts;
  int32_t *part_cnt;    // [nblk, E]
  float *part_prob;     // [nblk, E]
  int32_t *count_out;   // [E]
  float *prob_out;      // [E]
  uint8_t *lrank;       // [T, k] or null: rank of pair (t, j) among the CTA's tokens routed to
                        // the same expert (the permutation's within-chunk rank)
};

// Eight consecutive elements (bf16: 16 bytes; fp32: 32 bytes) and their pairs as fp32.
template <typename Tin> struct Chunk8;
template <> struct Chunk8<__nv_bfloat16> {
  static constexpr int PARTS = 1;  // 16-byte parts
  uint4 q;
  __device__ __forceinline__ void ld_s(const __nv_bfloat16 *p) { q = *(const uint4 *)p; }
  __device__ __forceinline__ void ld(const __nv_bfloat16 *p) { q = *(const uint4 *)p; }  // any space
  __device__ __forceinline__ void ld_g(const __nv_bfloat16 *p) { q = __ldg((const uint4 *)p); }
  __device__ __forceinline__ void zero() { q = make_uint4(0u, 0u, 0u, 0u); }
  // parts `stride` uint4s apart (the ring layout)
  __device__ __forceinline__ void ld_ring(const uint4 *p, int) { q = *p; }
  // elements 2i and 2i+1, widened exactly (a bf16 is the upper half of an fp32)
  __device__ __forceinline__ float2 pair(int i) const {
    const uint32_t w = i == 0 ? q.x : (i == 1 ? q.y : (i == 2 ? q.z : q.w));
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
  }
};
template <> struct Chunk8<float> {
  static constexpr int PARTS = 2;
  float4 a, b;
  __device__ __forceinline__ void ld_s(const float *p) {
    a = ((const float4 *)p)[0];
    b = ((const float4 *)p)[1];
  }
  __device__ __forceinline__ void ld(const float *p) { ld_s(p); }  // any space
  __device__ __forceinline__ void ld_g(const float *p) {
    a = __ldg((const float4 *)p);
    b = __ldg((const float4 *)p + 1);
  }
  __device__ __forceinline__ void zero() { a = b = make_float4(0.f, 0.f, 0.f, 0.f); }
  __device__ __forceinline__ void ld_ring(const uint4 *p, int stride) {
    a = *(const float4 *)p;
    b = *(const float4 *)(p + stride);
  }
  __device__ __forceinline__ float2 pair(int i) const {
    return i == 0 ? make_float2(a.x, a.y)
                  : (i == 1 ? make_float2(a.z, a.w) : (i == 2 ? make_float2(b.x, b.y) : make_float2(b.z, b.w)));
  }
};

// ------------------------------------------------------------------ exact expansion sums
struct Expansion {
  double h[EXPANSION_MAX];
  int n;
  bool overflow;
};

// Adds b exactly (Grow-Expansion with zero elimination; components non-overlapping,
// increasing magnitude). Round-to-nearest intrinsics keep the compiler from contracting.
__device__ __noinline__ void expansion_add(Expansion &X, double b) {
  double q = b;
  int m = 0;
  for (int i = 0; i < X.n; ++i) {
    const double hi = X.h[i];
    const double s = __dadd_rn(q, hi);
    const double bv = __dsub_rn(s, q);
    const double av = __dsub_rn(s, bv);
    const double err = __dadd_rn(__dsub_rn(q, av), __dsub_rn(hi, bv));
    q = s;
    if (err != 0.0) X.h[m++] = err;
  }
  if (q != 0.0) {
    if (m < EXPANSION_MAX) X.h[m++] = q;
    else X.overflow = true;
  }
  X.n = m;
}

__device__ __forceinline__ int expansion_sign(const Expansion &X) {
  if (X.n == 0) return 0;
  return X.h[X.n - 1] > 0.0 ? 1 : -1;
}

__device__ __forceinline__ bool f32_is_even(float v) { return (__float_as_uint(v) & 1u) == 0u; }

// Decide RN32 of the exact value S given: r = RN32(approx), S - mid_hi sign and S - mid_lo sign.
__device__ __forceinline__ float rn32_from_signs(float r, float up, float dn, int c_hi, int c_lo) {
  if (c_hi > 0) return up;
  if (c_hi == 0) return f32_is_even(r) ? r : up;
  if (c_lo < 0) return dn;
  if (c_lo == 0) return f32_is_even(r) ? r : dn;
  return r;
}

// True when RN32 of every value in [v - B, v + B] equals RN32(v).
__device__ __forceinline__ bool rn32_certain(double v, double B, float &r, float &up, float &dn,
                                             double &mid_hi, double &mid_lo) {
  r = __double2float_rn(v);
  up = nextafterf(r, INFINITY);
  dn = nextafterf(r, -INFINITY);
  mid_hi = 0.5 * ((double)r + (double)up);
  mid_lo = 0.5 * ((double)r + (double)dn);
  return (v + B < mid_hi) && (v - B > mid_lo) && fabs((double)r) < 0x1p126;
}

// RN32 of S = sum_i x_i W_i + off by one thread: S as an exact non-overlapping expansion; its top
// component is within an fp64 step of S, so RN32(S) is the fp32 value r nearest to it or a
// neighbour, and the signs of S minus the two rounding midpoints around r decide which.
template <typename Tin>
__device__ __noinline__ float exact_logit(const Tin *xrow, const Tin *wrow, int d, double off) {
  Expansion X;
  X.n = 0;
  X.overflow = false;
  for (int i = 0; i < d; ++i) {
    const double p = __dmul_rn((double)Elem<Tin>::to_f(xrow[i]), (double)Elem<Tin>::to_f(wrow[i]));  // exact
    if (p != 0.0) expansion_add(X, p);
  }
  if (off != 0.0) expansion_add(X, off);
  if (X.overflow) set_device_error(MOE_ERR_DEVICE_CHECK, INFO_EXPANSION_OVERFLOW);
  if (X.n == 0) return 0.0f;
  float r, up, dn;
  double mh, ml;
  rn32_certain(X.h[X.n - 1], 0.0, r, up, dn, mh, ml);
  expansion_add(X, -mh);                    // X = S - mid_hi
  const int c_hi = expansion_sign(X);
  expansion_add(X, mh - ml);                // X = S - mid_lo (difference exact)
  const int c_lo = expansion_sign(X);
  return rn32_from_signs(r, up, dn, c_hi, c_lo);
}

// ------------------------------------------------------------------ double-double sigmoid
struct dd {
  double hi, lo;
};
__device__ __forceinline__ dd two_sum(double a, double b) {
  const double s = __dadd_rn(a, b);
  const double bv = __dsub_rn(s, a);
  const double av = __dsub_rn(s, bv);
  return {s, __dadd_rn(__dsub_rn(a, av), __dsub_rn(b, bv))};
}
__device__ __forceinline__ dd quick_two_sum(double a, double b) {
  const double s = __dadd_rn(a, b);
  return {s, __dsub_rn(b, __dsub_rn(s, a))};
}
__device__ __forceinline__ dd two_prod(double a, double b) {
  const double p = __dmul_rn(a, b);
  return {p, __fma_rn(a, b, -p)};
}
__device__ __forceinline__ dd dd_add(dd a, dd b) {
  dd s = two_sum(a.hi, b.hi);
  dd t = two_sum(a.lo, b.lo);
  s.lo = __dadd_rn(s.lo, t.hi);
  s = quick_two_sum(s.hi, s.lo);
  s.lo = __dadd_rn(s.lo, t.lo);
  return quick_two_sum(s.hi, s.lo);
}
__device__ __forceinline__ dd dd_mul(dd a, dd b) {
  dd p = two_prod(a.hi, b.hi);
  p.lo = __dadd_rn(p.lo, __dadd_rn(__dmul_rn(a.hi, b.lo), __dmul_rn(a.lo, b.hi)));
  return quick_two_sum(p.hi, p.lo);
}
__device__ __forceinline__ dd dd_div(dd a, dd b) {
  const double q1 = __ddiv_rn(a.hi, b.hi);
  dd r = dd_add(a, dd_mul({-q1, 0.0}, b));
  const double q2 = __ddiv_rn(r.hi, b.hi);
  r = dd_add(r, dd_mul({-q2, 0.0}, b));
  const double q3 = __ddiv_rn(r.hi, b.hi);
  dd q = quick_two_sum(q1, q2);
  return dd_add(q, {q3, 0.0});
}

// Exponent of the leading bit and of the lowest set bit of a nonzero, normal double.
__device__ __forceinline__ void dbl_bit_range(double v, int &lead, int &lsb) {
  const unsigned long long b = (unsigned long long)__double_as_longlong(v);
  const int ef = (int)((b >> 52) & 0x7ff);
  const unsigned long long M = (b & 0xFFFFFFFFFFFFFull) | (1ull << 52);
  lead = ef - 1075 + 52;
  lsb = ef - 1075 + (__ffsll((long long)M) - 1);
}

// RN32(a 2^q), exactly: round to nearest even on the integer at the fp32 quantum of the value's
// binade (2^(E-23), or 2^-149 below 2^-126), then scale by a power of two, which is exact.
__device__ __forceinline__ float rn32_scaled_int(long long a, int q) {
  if (a == 0) return 0.0f;
  const bool neg = a < 0;
  const unsigned long long m = neg ? 0ull - (unsigned long long)a : (unsigned long long)a;
  const int E = (63 - __clzll((long long)m)) + q;  // 2^E <= |a 2^q| < 2^(E+1)
  if (E > 127) return neg ? -INFINITY : INFINITY;
  const int qexp = E >= -126 ? E - 23 : -149;
  const int sh = qexp - q;  // bits of m below the quantum
  unsigned long long t;
  if (sh <= 0) {
    t = m << (-sh);  // already a multiple of the quantum: t < 2^24
  } else if (sh >= 64) {
    t = 0ull;        // m < 2^63 <= half a quantum
  } else {
    t = m >> sh;
    const unsigned long long rem = m & ((1ull << sh) - 1ull), half = 1ull << (sh - 1);
    if (rem > half || (rem == half && (t & 1ull))) ++t;
  }
  const float r = ldexpf((float)t, qexp);  // t <= 2^24: exact, or the correct overflow to infinity
  return neg ? -r : r;
}

// Warp-cooperative exact rounding of S = sum_i x_i W_i + off. Every product is exact in fp64 and
// so is a multiple of 2^lsb(p); with q the smallest such exponent over all terms, every term is
// an integer multiple of 2^q below 2^(span+1), span = top exponent - q. When span + 1 +
// ceil(log2(d + 3)) <= 62 the integer sum of the terms is exact in int64, and S is that integer
// times 2^q. Returns false (caller falls back) when the span is wider or a term is subnormal.
template <typename Tin>
__device__ bool warp_exact_round(const Tin *xrow, const Tin *wrow, int d, double off, float &out) {
  const int lane = threadIdx.x & 31;
  int qmin = 0x7fffffff, emax = -0x7fffffff;
  bool bad = false;
  auto scan = [&](double v) {
    if (v == 0.0) return;
    if (fabs(v) < 0x1p-1020) { bad = true; return; }
    int lead, lsb;
    dbl_bit_range(v, lead, lsb);
    qmin = min(qmin, lsb);
    emax = max(emax, lead);
  };
  // lane covers elements [8*lane + 256*j, +8): d is a multiple of 64, so a chunk never straddles
  // d. Four chunks of each row are requested together; the products of bf16 or fp32 values are
  // exact in fp64.
  auto for_products = [&](auto &&fn) {
    for (int i0 = 8 * lane; i0 < d; i0 += 4 * 256) {
      Chunk8<Tin> xq[4], wq[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (i0 + 256 * u < d) {
          xq[u].ld(xrow + i0 + 256 * u);
          wq[u].ld(wrow + i0 + 256 * u);
        } else {
          xq[u].zero();
          wq[u].zero();
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          const float2 xf = xq[u].pair(p), wf = wq[u].pair(p);
          fn(__dmul_rn((double)xf.x, (double)wf.x));
          fn(__dmul_rn((double)xf.y, (double)wf.y));
        }
    }
  };
  for_products(scan);
  if (lane == 0) scan(off);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    qmin = min(qmin, __shfl_xor_sync(0xffffffffu, qmin, o));
    emax = max(emax, __shfl_xor_sync(0xffffffffu, emax, o));
  }
  bad = __any_sync(0xffffffffu, bad);
  const int span_max = 61 - (32 - __clz(d + 2));  // 61 - ceil(log2(d + 3))
  if (bad || emax - qmin > span_max) return false;
  long long acc = 0;
  for_products([&](double v) { acc += (long long)ldexp(v, -qmin); });
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  acc += (long long)ldexp(off, -qmin);
  out = rn32_scaled_int(acc, qmin);
  return true;
}

// Warp-cooperative exact RN32 of one logit whose fp64 evaluation could not settle it (or every
// logit in the forced test modes). Every lane calls it with the same arguments and gets the same
// result: the exact integer sum when the terms' exponent span allows, else the single-thread
// expansion. Neither depends on the fp64 sum, so a sum that cancels below its own error bound is
// rounded exactly too. force_level 2 skips the integer path, to test the expansion as well.
template <typename Tin>
__device__ __noinline__ float resolve_logit(const Tin *xrow, const Tin *wrow, int d, double off,
                                            int force_level) {
  const int lane = threadIdx.x & 31;
  float l;
  if (force_level < 2 && warp_exact_round<Tin>(xrow, wrow, d, off, l)) return l;
  l = 0.0f;
  if (lane == 0) l = exact_logit<Tin>(xrow, wrow, d, off);
  return __shfl_sync(0xffffffffu, l, 0);
}

// e^y in double-double: y = n ln2 + r, e^r by its Taylor series on r/2^10, squared 10 times.
// ln 2 to 106 bits as a double-double (hi = ln 2 rounded to double, lo = the remainder).
__device__ dd dd_exp(double y) {
  if (y > 709.0) return {INFINITY, 0.0};
  if (y < -745.0) return {0.0, 0.0};
  const double LN2_HI = 6.93147180559945286227e-01;
  const double LN2_LO = 2.31904681384629955842e-17;
  const double n = rint(y / LN2_HI);
  dd p = two_prod(n, LN2_HI);
  dd r = dd_add({y, 0.0}, {-p.hi, -p.lo});
  r = dd_add(r, {-n * LN2_LO, 0.0});
  r = {r.hi * 0x1p-10, r.lo * 0x1p-10};
  // Horner: sum_{i=0}^{12} r^i / i!
  double fact = 1.0;
  for (int i = 1; i <= 12; ++i) fact *= i;
  dd s = dd_div({1.0, 0.0}, {fact, 0.0});
  for (int i = 12; i >= 1; --i) {
    fact /= i;  // (i-1)!
    s = dd_add(dd_mul(s, r), dd_div({1.0, 0.0}, {fact, 0.0}));
  }
  for (int i = 0; i < 10; ++i) s = dd_mul(s, s);
  const int ni = (int)n;
  return {ldexp(s.hi, ni), ldexp(s.lo, ni)};
}

// The exact decision for a sigmoid key the fp64 screen could not settle (rare, kept out of line
// so it does not occupy the instruction cache of the hot loop): double-double sigmoid, compared
// with the fp32 rounding midpoints mh / ml around the candidate r.
__device__ __noinline__ float sigmoid_key_exact(float l, float b, float r, float up, float dn,
                                                double mh, double ml) {
  int c_hi, c_lo;
  if (l == 0.0f) {  // sigmoid(0) = 1/2 exactly
    const dd vv = two_sum(0.5, (double)b);
    const dd a = dd_add(vv, {-mh, 0.0}), c = dd_add(vv, {-ml, 0.0});
    c_hi = a.hi > 0 ? 1 : (a.hi < 0 ? -1 : 0);
    c_lo = c.hi > 0 ? 1 : (c.hi < 0 ? -1 : 0);
    return rn32_from_signs(r, up, dn, c_hi, c_lo);
  }
  const dd e = dd_exp(-(double)l);
  dd sig;
  if (isinf(e.hi)) sig = {0.0, 0.0};
  else sig = dd_div({1.0, 0.0}, dd_add({1.0, 0.0}, e));
  const dd vv = dd_add(sig, {(double)b, 0.0});
  const dd a = dd_add(vv, {-mh, 0.0}), c = dd_add(vv, {-ml, 0.0});
  const double tol = 1e-26 * fabs(vv.hi) + 1e-300;
  if (fabs(a.hi) <= tol || fabs(c.hi) <= tol)
    set_device_error(MOE_ERR_DEVICE_CHECK, INFO_SIGMOID_UNRESOLVED);
  c_hi = a.hi > 0 ? 1 : (a.hi < 0 ? -1 : 0);
  c_lo = c.hi > 0 ? 1 : (c.hi < 0 ? -1 : 0);
  return rn32_from_signs(r, up, dn, c_hi, c_lo);
}

// RN32(sigmoid(l) + b), exact. fp64 screen first unless forced.
__device__ __forceinline__ float sigmoid_key(float l, float b, bool force) {
  const double s = 1.0 / (1.0 + exp(-(double)l));
  const double v = s + (double)b;
  const double B = 0x1p-48 * s + 0x1p-52 * fabs(v) + 1e-300;
  float r, up, dn;
  double mh, ml;
  if (rn32_certain(v, B, r, up, dn, mh, ml) && !force) return r;
  return sigmoid_key_exact(l, b, r, up, dn, mh, ml);
}

// ------------------------------------------------------------------ kernel
constexpr int RT_WD = 4;  // W chunks in flight per lane pair (cp.async ring)

// The kernel's scalars in shared memory, kept in the dynamic allocation so that the host's size
// check covers every byte the kernel uses.
struct RouterMisc {
  uint64_t xbar;                 // token-row copies
  unsigned long long wnmax;      // max_e |W_e| bound (bits of a nonnegative double)
  int nflag, offmax, bmax;       // listed tokens; max |offset|, max |bias| (bits of floats)
  int xabort;
  unsigned badtok, proven;       // bit tt: a non-finite logit; the order is proven
  int flag[RT_TM];               // listed tokens
  unsigned lmax[RT_TM];          // max |l| per token (bits of a nonnegative float)
};
constexpr int RT_MISC_BYTES = 256;
static_assert(sizeof(RouterMisc) <= RT_MISC_BYTES, "router scalars");

// Shared-memory layout of the router kernel (byte offsets), shared by host and device.
struct RouterSmem {
  size_t xs, xs_stride, ring, part, wsq, wn, off, lg, keys, cnt, xnorm, cmask, misc, total;
};
__host__ __device__ inline RouterSmem router_smem(int E, bool sigmoid, int d, int esize, int ept) {
  RouterSmem L;
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t at = o; o = (o + bytes + 15) & ~(size_t)15; return at; };
  // the CTA's token rows, each padded by 32 bytes: the rows tg, tg+2, ... that a warp reads in
  // one instruction then start 32 bytes apart in the banks
  L.xs_stride = (size_t)d * esize + 32;
  L.xs = take((size_t)RT_TM * L.xs_stride);
  // rings of W chunks, one per lane pair (lanes tg = 0, 1 use the same chunks):
  // [slot][expert][16-byte part][pair]
  L.ring = take((size_t)RT_WD * ept * (RT_THREADS / 2) * 8 * esize);
  L.part = take((size_t)RT_WARPS * RT_TM * 8 * ept * sizeof(float));  // per-warp partial logits
  L.wsq = take((size_t)RT_WARPS * 8 * ept * sizeof(float));           // per-warp W sums of squares
  L.wn = take((size_t)E * sizeof(double));
  L.off = take((size_t)E * sizeof(float));
  L.lg = take((size_t)RT_TM * E * sizeof(float));
  L.keys = take(sigmoid ? (size_t)RT_TM * E * sizeof(float) : 0);
  L.cnt = take((size_t)E * sizeof(int));
  L.xnorm = take(RT_TM * sizeof(double));
  L.cmask = take((size_t)RT_TM * ((E + 31) / 32) * sizeof(unsigned));  // candidates per listed token
  L.misc = take(RT_MISC_BYTES);  // barrier and per-CTA scalars (RouterMisc)
  L.total = o;
  return L;
}

// Experts per thread of a launch: the wide tile from RT_WIDE_MIN_E experts when its shared memory
// fits, else the narrow one.
__host__ __device__ inline int router_ept(int E, bool sigmoid, int d, int esize) {
  if (E >= RT_WIDE_MIN_E && router_smem(E, sigmoid, d, esize, RT_EPT_WIDE).total <= 227 * 1024)
    return RT_EPT_WIDE;
  return RT_EPT;
}

// Upper bound on sqrt(sum of squares) from an fp32 accumulation of at most n = d + 16 fused
// multiply-adds and additions: each step rounds with relative error <= 2^-24 or, in the
// subnormal range, absolute error <= 2^-150, so the exact sum is at most
// (computed + n 2^-149) (1 + n 2^-23) while n 2^-24 is small. Infinite or NaN input stays so.
__device__ __forceinline__ double norm_upper(double computed, int d) {
  const double n = (double)(d + 16);
  return sqrt((computed + n * 0x1p-149) * (1.0 + n * 0x1p-23));
}

__device__ __forceinline__ double sigmoid64(float l) { return 1.0 / (1.0 + exp(-(double)l)); }

// The n largest keys of a row (NaN as -infinity; equal keys: lower index first) into sel[0..n).
__device__ __forceinline__ void warp_topn(const float *krow, int E, int n, int (&sel)[9]) {
  const int lane = threadIdx.x & 31;
  unsigned selmask = 0u;
#pragma unroll
  for (int j = 0; j < 9; ++j) {
    sel[j] = 0;
    if (j < n) {
      float bk = -INFINITY;
      int be = 0x7fffffff;
      for (int i = 0, e = lane; e < E; ++i, e += 32) {
        if ((selmask >> i) & 1u) continue;
        float kv = krow[e];
        if (kv != kv) kv = -INFINITY;
        if (be == 0x7fffffff || kv > bk) { bk = kv; be = e; }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ok = __shfl_xor_sync(0xffffffffu, bk, o);
        const int oe = __shfl_xor_sync(0xffffffffu, be, o);
        if (oe != 0x7fffffff && (be == 0x7fffffff || ok > bk || (ok == bk && oe < be))) {
          bk = ok;
          be = oe;
        }
      }
      sel[j] = be;
      if ((be & 31) == lane) selmask |= 1u << (be >> 5);
    }
  }
}

// Canonical logit from the fp64 sum s of the exact products plus the offset (every lane holds
// the same s): |s - S| <= gamma_{d+16} (sum |x_i W_i| + |off|) <= (d+16) 2^-52 (|x||W_e| + |off|).
// When no fp32 rounding boundary lies within that distance, RN32(s) is the canonical logit;
// otherwise resolve_logit decides exactly (warp-cooperative).
template <typename Tin>
__device__ float finish_logit(double s, const Tin *xrow, const Tin *wrow, int d, double off,
                              double xn, double wne, int force_level) {
  if (!isfinite(s)) return (float)s;  // an infinite or NaN input: the sum is that, exactly
  const double B = (double)(d + 16) * 0x1p-52 * (xn * wne + fabs(off));
  float r, up, dn;
  double mh, ml;
  if (force_level == 0 && rn32_certain(s, B, r, up, dn, mh, ml)) return r;
  return resolve_logit<Tin>(xrow, wrow, d, off, force_level);
}

// EPT experts per thread (a round covers 8 EPT experts): 3 for up to 96 experts (two CTAs per SM),
// 6 above, where the logit rows already hold one CTA per SM and the wider tile halves the rounds.
template <typename Tin, int EPT>
__global__ void __launch_bounds__(RT_THREADS, EPT == RT_EPT ? 2 : 1) router_kernel(RouterArgs a) {
  constexpr int EB = 8 * EPT;  // experts per round
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  using CH = Chunk8<Tin>;
  const int E = a.E, d = a.d, k = a.k;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t0 = blockIdx.x * RT_TM;
  const int ntok = min(RT_TM, a.T - t0);
  const Tin *__restrict__ x = (const Tin *)a.x;
  const Tin *__restrict__ wr = (const Tin *)a.w;
  const int force_level = g_force_exact;
  const bool force = force_level != 0;
  const bool sigmoid = a.score == MOE_SCORE_SIGMOID;
  const RouterSmem SL = router_smem(E, sigmoid, d, (int)sizeof(Tin), EPT);
  uint4 *ring = (uint4 *)(smem_raw + SL.ring);   // [RT_WD][EPT][PARTS][RT_THREADS / 2]
  float *off_s = (float *)(smem_raw + SL.off);   // [E] logit offsets (zeros without)
  float *part = (float *)(smem_raw + SL.part);   // [RT_WARPS][RT_TM][EB]
  float *wsq_s = (float *)(smem_raw + SL.wsq);   // [RT_WARPS][EB]
  double *wn = (double *)(smem_raw + SL.wn);     // [E] upper bounds of |W_e|_2
  float *lg = (float *)(smem_raw + SL.lg);       // [RT_TM][E] logits, then probabilities
  float *keys = (float *)(smem_raw + SL.keys);   // [RT_TM][E] sigmoid keys
  int *cnt = (int *)(smem_raw + SL.cnt);
  double *xnorm = (double *)(smem_raw + SL.xnorm);
  unsigned *cmask = (unsigned *)(smem_raw + SL.cmask);  // [listed token][E/32]
  RouterMisc &M = *(RouterMisc *)(smem_raw + SL.misc);
  int &s_nflag = M.nflag, *s_flag = M.flag;
  unsigned long long &s_wnmax = M.wnmax;  // bits of nonnegative doubles / floats order as integers
  int &s_offmax = M.offmax, &s_bmax = M.bmax;
  unsigned &s_badtok = M.badtok, &s_proven = M.proven, *s_lmax = M.lmax;
  // after the screen the per-warp partials are free: the selection's records live there
  int *s_sel = (int *)(smem_raw + SL.part);                   // [RT_TM][8] final selections
  int *s_by = s_sel + RT_TM * 8;                               // [RT_TM][9] experts by rank
  double *s_bk = (double *)(smem_raw + SL.part + 1280);        // [RT_TM] key bounds

  const KernelStamp stamp(K_ROUTER);
  griddep_wait();
  stamp.started();
  griddep_launch();
  // ---- the CTA's token rows -> shared memory: one bulk copy per row, all in flight at once
  unsigned char *xs = smem_raw + SL.xs;
  const size_t xs_stride = SL.xs_stride;
  const uint32_t row_bytes = (uint32_t)d * (uint32_t)sizeof(Tin);
  volatile int &s_xabort = M.xabort;
  const uint32_t xbar = smem_u32(&M.xbar);
  if (tid == 0) {
    mbar_init(xbar, 1);
    s_xabort = 0;
    s_wnmax = 0ull;
    s_offmax = 0;
    s_bmax = 0;
    s_nflag = 0;
    s_badtok = 0u;
    s_proven = 0u;
  }
  if (tid < RT_TM) {
    s_lmax[tid] = 0u;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (tid == 0) {
    mbar_expect_tx(xbar, (uint32_t)ntok * row_bytes);
    for (int r = 0; r < ntok; ++r)
      bulk_load_1d(smem_u32(xs + (size_t)r * xs_stride), x + (size_t)(t0 + r) * d, row_bytes, xbar);
  }

  // ---- screen tiling (see the header): this lane's chunks of d and its W ring
  const int nch = d >> 3;  // 8-element chunks per row (d is a multiple of 64)
  const int ks = lane & 1, eg = (lane >> 1) & 7, tg = lane >> 4;
  const int c0 = 2 * warp + ks;
  const int nmine = c0 < nch ? (nch - c0 + 2 * RT_WARPS - 1) / (2 * RT_WARPS) : 0;
  const int pr = warp * 16 + (lane & 15);  // the lane pair
  constexpr int NP = RT_THREADS / 2;
  auto slot_ptr = [&](int s, int j) { return ring + ((size_t)(s * EPT + j) * CH::PARTS) * NP + pr; };
  // copies of chunk n of the pair's expert rows of the round at eb into slot n % RT_WD, the
  // 16-byte parts q = j PARTS + u dealt to the two lanes by q % 2 = tg; one commit group per
  // call, empty or not, so that the group count stays uniform
  auto ring_issue = [&](int eb, int n) {
    if (n < nmine) {
      const int c = c0 + 2 * RT_WARPS * n;
#pragma unroll
      for (int j = 0; j < EPT; ++j) {
        const int e = eb + eg + 8 * j;
#pragma unroll
        for (int u = 0; u < CH::PARTS; ++u)
          if (((j * CH::PARTS + u) & 1) == tg && e < E)
            cp_async16(smem_u32(slot_ptr(n % RT_WD, j) + u * NP),
                       (const unsigned char *)(wr + (size_t)e * d + 8 * c) + 16 * u);
      }
    }
    cp_async_commit();
  };
  // the first chunks of a round; parts of experts past E are zeroed (never copied into)
  auto ring_prologue = [&](int eb) {
#pragma unroll
    for (int j = 0; j < EPT; ++j)
#pragma unroll
      for (int u = 0; u < CH::PARTS; ++u)
        if (((j * CH::PARTS + u) & 1) == tg && eb + eg + 8 * j >= E)
          for (int s = 0; s < RT_WD; ++s) slot_ptr(s, j)[u * NP] = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int n = 0; n < RT_WD; ++n) ring_issue(eb, n);
  };
  ring_prologue(0);  // W does not depend on x: its first chunks travel with the token rows

  for (int r = ntok; r < RT_TM; ++r)  // rows past the last token read as zeros
    for (uint32_t i = tid; i < row_bytes / 16; i += RT_THREADS)
      ((uint4 *)(xs + (size_t)r * xs_stride))[i] = make_uint4(0u, 0u, 0u, 0u);
  for (int e = tid; e < E; e += RT_THREADS) {
    cnt[e] = 0;
    const float o = a.off ? a.off[e] : 0.0f;
    off_s[e] = o;
    // largest |offset| and |bias| (NaN orders above infinity and poisons the bound, as it should)
    atomicMax(&s_offmax, __float_as_int(fabsf(o)));
    if (a.bias) atomicMax(&s_bmax, __float_as_int(fabsf(a.bias[e])));
  }
  mbar_wait(xbar, 0u, (volatile int *)&s_xabort, g_wait_limit_ns, INFO_WAIT_ROUTER_X);
  __syncthreads();
  if (s_xabort) {  // the copies did not land in time: error recorded; let them drain, then leave
    if (tid == 0) {
      volatile int never = 0;
      mbar_wait(xbar, 0u, &never, g_wait_limit_ns, INFO_WAIT_DRAIN);
    }
    cp_async_wait<0>();
    __syncthreads();
    return;
  }

  // ---- |x_t|_2 bounds: 16 threads per row, fp32 sums of squares, fixed tree
  {
    const int tt = tid >> 4, q16 = tid & 15;
    const Tin *row = (const Tin *)(xs + (size_t)tt * xs_stride);
    float s = 0.0f;
    for (int c = q16; c < nch; c += 16) {
      CH q;
      q.ld_s(row + 8 * c);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 p = q.pair(i);
        s = fmaf(p.x, p.x, s);
        s = fmaf(p.y, p.y, s);
      }
    }
#pragma unroll
    for (int o = 8; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (q16 == 0) xnorm[tt] = norm_upper((double)s, d);
  }

  // ---- screen: approximate logits in fp32, EB experts per round. Warp w takes the chunks
  // 2w + ks + 16n of d; per chunk a thread takes its EPT expert chunks from its ring (filled
  // RT_WD chunks ahead) and its 8 token chunks from the staged rows, and accumulates 8 EPT
  // (token, expert) pairs as two-lane packed FMAs (even and odd elements in the two lanes).
  // The sums of squares of the W rows ride along: lane tg squares pairs 2tg, 2tg+1 of a chunk.
  const size_t xs_es = xs_stride / sizeof(Tin);  // row stride in elements
  const Tin *xrow0 = (const Tin *)(xs + (size_t)tg * xs_stride);
  for (int eb = 0; eb < E; eb += EB) {
    float2 acc[RT_TPT][EPT], wsq[EPT];
#pragma unroll
    for (int j = 0; j < EPT; ++j) {
      wsq[j] = make_float2(0.f, 0.f);
#pragma unroll
      for (int tj = 0; tj < RT_TPT; ++tj) acc[tj][j] = make_float2(0.f, 0.f);
    }
    for (int n = 0; n < nmine; ++n) {
      const int c = c0 + 2 * RT_WARPS * n;
      // both lanes of the pair are done with slot (n-1) % RT_WD: it refills with chunk
      // n-1+RT_WD; then chunk n (RT_WD groups back) is complete in both lanes and visible
      __syncwarp();
      if (n > 0) ring_issue(eb, n - 1 + RT_WD);
      else cp_async_commit();
      cp_async_wait<RT_WD>();
      __syncwarp();
      float2 w2[EPT][4];
#pragma unroll
      for (int j = 0; j < EPT; ++j) {
        CH wc;
        wc.ld_ring(slot_ptr(n % RT_WD, j), NP);
#pragma unroll
        for (int i = 0; i < 4; ++i) w2[j][i] = wc.pair(i);
        const float2 p0 = tg ? w2[j][2] : w2[j][0], p1 = tg ? w2[j][3] : w2[j][1];
        wsq[j] = __ffma2_rn(p0, p0, wsq[j]);
        wsq[j] = __ffma2_rn(p1, p1, wsq[j]);
      }
#pragma unroll
      for (int tj = 0; tj < RT_TPT; ++tj) {
        CH xc;
        xc.ld_s(xrow0 + (size_t)(2 * tj) * xs_es + 8 * c);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 x2 = xc.pair(i);
#pragma unroll
          for (int j = 0; j < EPT; ++j) acc[tj][j] = __ffma2_rn(x2, w2[j][i], acc[tj][j]);
        }
      }
    }
    cp_async_wait<0>();
    __syncwarp();  // both lanes done with the ring before the next round's copies
    if (eb + EB < E) ring_prologue(eb + EB);  // the next round's W, during this reduction
    // fold the two lanes of each pair, then the two k halves (lanes ks = 0, 1); lane ks = 0
    // stores tokens tg + 2tj for tj < 4, lane ks = 1 the rest
    float *pw = part + (size_t)warp * RT_TM * EB;
#pragma unroll
    for (int tj = 0; tj < RT_TPT; ++tj)
#pragma unroll
      for (int j = 0; j < EPT; ++j) {
        float v = __fadd_rn(acc[tj][j].x, acc[tj][j].y);
        v = __fadd_rn(v, __shfl_xor_sync(0xffffffffu, v, 1));
        if ((tj >> 2) == ks) pw[(tg + 2 * tj) * EB + eg + 8 * j] = v;
      }
#pragma unroll
    for (int j = 0; j < EPT; ++j) {
      float s = __fadd_rn(wsq[j].x, wsq[j].y);
      s = __fadd_rn(s, __shfl_xor_sync(0xffffffffu, s, 16));
      s = __fadd_rn(s, __shfl_xor_sync(0xffffffffu, s, 1));
      if (tg == 0 && ks == 0) wsq_s[warp * EB + eg + 8 * j] = s;
    }
    __syncthreads();
    // per-warp partials added in warp order, then the offset: every product passes through at
    // most 4 ceil(d/128) (its chain) + 1 + 1 + 7 + 1 roundings
    for (int q = tid; q < RT_TM * EB; q += RT_THREADS) {
      const int tt = q / EB, el = q - tt * EB, e = eb + el;
      if (tt < ntok && e < E) {
        float s = part[tt * EB + el];
#pragma unroll
        for (int w = 1; w < RT_WARPS; ++w) s = __fadd_rn(s, part[(w * RT_TM + tt) * EB + el]);
        if (a.off) s = __fadd_rn(s, off_s[e]);
        lg[tt * E + e] = s;
      }
    }
    if (tid < EB && eb + tid < E) {
      float s = wsq_s[tid];
#pragma unroll
      for (int w = 1; w < RT_WARPS; ++w) s = __fadd_rn(s, wsq_s[w * EB + tid]);
      const double nrm = norm_upper((double)s, d);
      wn[eb + tid] = nrm;
      atomicMax(&s_wnmax, (unsigned long long)__double_as_longlong(nrm));
    }
    __syncthreads();  // part and wsq_s are rewritten by the next round
  }

  // key of expert e of token tt as the screen sees it (fp64, before any fp32 rounding)
  auto key_of = [&](int tt, int e) -> double {
    const float l = lg[tt * E + e];
    if (!sigmoid) return (double)l;
    return sigmoid64(l) + (a.bias ? (double)a.bias[e] : 0.0);
  };
  // Experts of rank 0..n-1 (descending key, NaN as -infinity, ties to the lower index) of the
  // tokens in `tmask` into s_by[tt][0..n). Up to 64 experts a thread counts the rank of one
  // (token, expert) pair; above, a warp per token takes the n largest in turn.
  auto rank_tokens = [&](unsigned tmask, int n) {
    const float *kb = sigmoid ? keys : lg;
    if (E <= RT_SEL_THREAD_MAX_E) {
      for (int q = tid; q < ntok * E; q += RT_THREADS) {
        const int tt = q / E, e = q - tt * E;
        if (!((tmask >> tt) & 1u)) continue;
        const float *krow = kb + tt * E;
        float v = krow[e];
        if (v != v) v = -INFINITY;
        int rank = 0;
        for (int e2 = 0; e2 < E; ++e2) {
          float v2 = krow[e2];
          if (v2 != v2) v2 = -INFINITY;
          rank += (v2 > v || (v2 == v && e2 < e)) ? 1 : 0;
        }
        if (rank < n) s_by[tt * 9 + rank] = e;
      }
    } else {
      for (int tt = warp; tt < ntok; tt += RT_WARPS) {
        if (!((tmask >> tt) & 1u)) continue;
        int sel[9];
        warp_topn(kb + tt * E, E, n, sel);
#pragma unroll
        for (int j = 0; j < 9; ++j)
          if (j < n && lane == 0) s_by[tt * 9 + j] = sel[j];
      }
    }
  };
  // Probabilities, combine weights and outputs of every token, fixed-order trees; the logits row
  // becomes the probability basis of the load-balancing statistics. Up to 64 experts 16 threads
  // (a half-warp) take a token, all 16 tokens at once; above, a warp per token.
  auto finish_tokens = [&]() {
    const int G = E <= RT_SEL_THREAD_MAX_E ? 16 : 32;  // threads per token
    const unsigned gmask = G == 16 ? 0xFFFFu << (lane & 16) : 0xFFFFFFFFu;
    const int sub = tid & (G - 1);
    for (int tt = tid / G; tt < ntok; tt += RT_THREADS / G) {  // whole groups
      float *lrow = lg + tt * E;
      float m = -INFINITY, sum = 0.0f;
      if (!sigmoid) {
        for (int e = sub; e < E; e += G) m = fmaxf(m, lrow[e]);
        for (int o = G / 2; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(gmask, m, o));
        for (int e = sub; e < E; e += G) sum += expf(lrow[e] - m);
      } else {
        for (int e = sub; e < E; e += G) sum += 1.0f / (1.0f + expf(-lrow[e]));
      }
      for (int o = G / 2; o > 0; o >>= 1) sum += __shfl_xor_sync(gmask, sum, o);
      int ej = 0;
      float pj = 0.0f;
      if (sub < k) {
        ej = s_by[tt * 9 + sub];
        pj = !sigmoid ? expf(lrow[ej] - m) / sum : 1.0f / (1.0f + expf(-lrow[ej]));
      }
      float psel = pj;
      for (int o = G / 2; o > 0; o >>= 1) psel += __shfl_xor_sync(gmask, psel, o);
      __syncwarp(gmask);  // every read of the logits row precedes its overwrite
      for (int e = sub; e < E; e += G)
        lrow[e] = !sigmoid ? expf(lrow[e] - m) / sum : (1.0f / (1.0f + expf(-lrow[e]))) / sum;
      if (sub < k) {
        const size_t o = (size_t)(t0 + tt) * k + sub;
        a.idx[o] = ej;
        a.wts[o] = a.norm ? pj / psel : pj;
        atomicAdd(&cnt[ej], 1);
        s_sel[tt * 8 + sub] = ej;
      }
    }
  };
  // ---- selection in block-wide phases over the CTA's tokens (a token's order is proven from
  // the screen, or its candidate experts are listed and settled exactly by the whole CTA below)
  const double mg = (double)(4 * ((nch + 15) / 16) + 10);  // roundings per term of the screen
  const double gam = mg * 0x1p-24 / (1.0 - mg * 0x1p-24);
  const double wmax = __longlong_as_double((long long)s_wnmax);
  const double omax = (double)__int_as_float(s_offmax), bmax = (double)__int_as_float(s_bmax);
  const int nmw = (E + 31) >> 5;  // candidate mask words per token
  // (a) sigmoid keys from the screened logits; per token: any non-finite logit, max |l|
  for (int q = tid; q < ntok * E; q += RT_THREADS) {
    const int tt = q / E, e = q - tt * E;
    const float l = lg[q];
    if (!isfinite(l)) atomicOr(&s_badtok, 1u << tt);
    if (sigmoid) {
      keys[q] = (float)key_of(tt, e);
      atomicMax(&s_lmax[tt], __float_as_uint(fabsf(l)));
    }
  }
  __syncthreads();
  // (b) experts of approximate ranks 0..k of every token
  rank_tokens((1u << ntok) - 1u, min(k + 1, E));
  __syncthreads();
  // (c) the proof, 8 threads per token: each of the J gaps between consecutive approximate ranks
  // must exceed twice the key bound plus two fp32 steps at that magnitude (thread j checks gap j)
  if (tid < RT_TM * 8) {  // warps 0-3, whole
    const int tt = tid >> 3, j = tid & 7;
    bool ok = true;
    double Bk = 0.0;
    if (tt < ntok) {
      // Bound of the token's keys. Screen: |l~ - S| <= gamma_m (|x_t| max_e |W_e| + max |off|)
      // for the exact sum S of every expert (m roundings per term, plus m 2^-149 for
      // underflow). Sigmoid: the key comes from the canonical (rounded) logit, within that plus
      // half an fp32 step of l~; sigmoid is 1/4-Lipschitz, and its fp64 evaluation plus the bias
      // add err by less than 2^-47 + 2^-51 |b|.
      Bk = gam * (xnorm[tt] * wmax + omax) * (1.0 + 0x1p-40) + mg * 0x1p-149;
      if (sigmoid) {
        const double lmax = (double)__uint_as_float(s_lmax[tt]);
        Bk = 0.25 * (Bk + 0x1p-24 * (lmax + Bk) + 0x1p-149) + 0x1p-47 + 0x1p-51 * bmax;
      }
      if (j < min(k, E - 1)) {
        const int *br = s_by + tt * 9;
        const double prev = key_of(tt, br[j]), cur = key_of(tt, br[j + 1]);
        ok = prev - cur > 2.0 * Bk + 0x1p-22 * (fmax(fabs(prev), fabs(cur)) + Bk) + 0x1p-148;
      }
    }
    const unsigned fails = __ballot_sync(0xffffffffu, !ok);
    if (j == 0 && tt < ntok) {
      s_bk[tt] = Bk;
      const bool bad = (s_badtok >> tt) & 1u;
      if (((fails >> (lane & 24)) & 0xFFu) == 0u && !bad && !force && Bk < INFINITY)
        atomicOr(&s_proven, 1u << tt);
    }
  }
  __syncthreads();
  // (d) the unproven tokens' candidates: every expert whose key is not provably below the
  // (k+1)-th approximate key (all of them when the bound is unusable or k = E); a warp per token
  for (int tt = warp; tt < ntok; tt += RT_WARPS) {
    if ((s_proven >> tt) & 1u) continue;
    const double Bk = s_bk[tt];
    const bool bad = (s_badtok >> tt) & 1u;
    const bool all = force || bad || E <= k || !(Bk < INFINITY);
    double cut = -INFINITY;
    if (!all) {
      const double vk = key_of(tt, s_by[tt * 9 + k]);
      cut = vk - 2.0 * Bk - 0x1p-22 * (fabs(vk) + Bk) - 0x1p-148;
    }
    int f = 0;
    if (lane == 0) f = atomicAdd(&s_nflag, 1);
    f = __shfl_sync(0xffffffffu, f, 0);
    if (lane == 0) s_flag[f] = tt;
    for (int w0 = 0; w0 < nmw; ++w0) {
      const int e = 32 * w0 + lane;
      const unsigned m = __ballot_sync(0xffffffffu, e < E && (all || key_of(tt, e) >= cut));
      if (lane == 0) cmask[f * nmw + w0] = m;
    }
    __syncwarp();
  }
  __syncthreads();

  // ---- exact settlement of the listed tokens: their candidates dealt round-robin to the warps,
  // one warp per candidate (fp64 sum of the exact products, then finish_logit)
  const int nflag = s_nflag;
  if (nflag > 0) {
    int ci = 0;
    for (int f = 0; f < nflag; ++f) {
      const int tt = s_flag[f];
      const Tin *xrow = (const Tin *)(xs + (size_t)tt * xs_stride);
      for (int w0 = 0; w0 < nmw; ++w0) {
        unsigned m = cmask[f * nmw + w0];
        while (m) {
          const int ee = 32 * w0 + __ffs(m) - 1;
          m &= m - 1;
          if ((ci++ % RT_WARPS) != warp) continue;
          const Tin *wrow = wr + (size_t)ee * d;
          double acc = 0.0;
          uint32_t xmn = 0xFFFFFFFFu, wmn = 0xFFFFFFFFu, emx = 0u;  // fp32 magnitude bits
          auto note = [&](float xv, float wv) {
            const uint32_t bx = __float_as_uint(xv) & 0x7FFFFFFFu, bw = __float_as_uint(wv) & 0x7FFFFFFFu;
            xmn = min(xmn, bx ? bx : 0xFFFFFFFFu);
            wmn = min(wmn, bw ? bw : 0xFFFFFFFFu);
            emx = max(emx, max(bx, bw));
          };
          for (int i0 = 8 * lane; i0 < d; i0 += 4 * 256) {
            CH wq[4], xq[4];  // four chunks of the lane requested together
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int i = i0 + 256 * u;
              if (i < d) {
                wq[u].ld_g(wrow + i);
                xq[u].ld_s(xrow + i);
              } else {
                wq[u].zero();
                xq[u].zero();
              }
            }
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
              for (int p = 0; p < 4; ++p) {
                const float2 xf = xq[u].pair(p), wf = wq[u].pair(p);
                acc = fma((double)xf.x, (double)wf.x, acc);
                acc = fma((double)xf.y, (double)wf.y, acc);
                note(xf.x, wf.x);
                note(xf.y, wf.y);
              }
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) {
            xmn = min(xmn, __shfl_xor_sync(0xffffffffu, xmn, o));
            wmn = min(wmn, __shfl_xor_sync(0xffffffffu, wmn, o));
            emx = max(emx, __shfl_xor_sync(0xffffffffu, emx, o));
          }
          const float of = off_s[ee];
          const double o = (double)of;
          const double sum = warp_sum_d(acc) + o;
          // Exactness certificate: with all elements normal and finite (biased exponents
          // >= xe, we), every product is an integer multiple of 2^q, q = xe + we - 254 - 2 MANT
          // (MANT fraction bits of the input type), and so is the offset with its own quantum.
          // Every partial sum, in any order, is at most |x||W_e| + |off| (Cauchy-Schwarz); below
          // 2^(q+53) all of them are fp64 values, so `sum` is the exact sum and its fp32
          // rounding the canonical logit, ties to even included.
          constexpr int MANT = sizeof(Tin) == 2 ? 7 : 23;
          bool exact = false;
          if (xmn != 0xFFFFFFFFu && wmn != 0xFFFFFFFFu) {
            const int xe = (int)(xmn >> 23), we = (int)(wmn >> 23);
            int q = xe + we - 254 - 2 * MANT;
            bool okc = xe > 0 && we > 0 && (emx >> 23) < 255u;
            if (of != 0.0f) {
              const int eo = (int)((__float_as_uint(of) >> 23) & 0xFFu);
              okc = okc && eo > 0 && eo < 255;
              q = min(q, eo - 150);
            }
            const double S = (xnorm[tt] * wn[ee] + fabs(o)) * (1.0 + (double)(d + 8) * 0x1p-50);
            exact = okc && S <= ldexp(1.0, min(q + 53, 1023));
          } else if (xmn == 0xFFFFFFFFu || wmn == 0xFFFFFFFFu) {
            exact = (emx >> 23) < 255u;  // one row all zeros: the sum is the offset, exactly
          }
          const float l = exact && !force
                              ? __double2float_rn(sum)
                              : finish_logit<Tin>(sum, xrow, wrow, d, o, xnorm[tt], wn[ee], force_level);
          if (lane == 0) {
            lg[tt * E + ee] = l;
            if (sigmoid) keys[tt * E + ee] = sigmoid_key(l, a.bias ? a.bias[ee] : 0.0f, force);
          }
          __syncwarp();
        }
      }
    }
    __syncthreads();
    // the listed tokens, ranked again on their canonical candidate keys
    unsigned fm = 0u;
    for (int f = 0; f < nflag; ++f) fm |= 1u << s_flag[f];
    rank_tokens(fm, k);
  }
  __syncthreads();
  // (e) probabilities, combine weights and outputs of every token, 16 threads per token
  finish_tokens();
  __syncthreads();

  // ---- within-chunk ranks: pair (tt, j) counts the earlier tokens of the CTA that selected the
  // same expert (a token selects an expert at most once)
  if (a.lrank && tid < ntok * k) {
    const int tt = tid / k, j = tid - tt * k;
    const int e = s_sel[tt * 8 + j];
    int r = 0;
    for (int u = 0; u < tt; ++u)
      for (int jj = 0; jj < k; ++jj) r += s_sel[u * 8 + jj] == e ? 1 : 0;
    a.lrank[(size_t)(t0 + tt) * k + j] = (uint8_t)r;
  }
  // ---- per-CTA statistics (fixed token order), then the last CTA reduces in CTA order
  for (int e = tid; e < E; e += RT_THREADS) {
    float ps = 0.0f;
    for (int tt = 0; tt < ntok; ++tt) ps += lg[tt * E + e];
    a.part_cnt[(size_t)blockIdx.x * E + e] = cnt[e];
    a.part_prob[(size_t)blockIdx.x * E + e] = ps;
  }
}

}  // namespace moe

// Router: logits, selection keys, top-k, combine weights and per-expert statistics.
//
// What it computes (Quartz: softmax router, 6 of 24 experts; Moonfrost expert card: top-3
// routing; Sutra-1.3B: top-4 by sigmoid score plus a per-expert balancing bias):
//   l[t,e]  = RN32(exact sum_i x[t,i] W[e,i] + off[e])              (fp32, canonical)
//   key     = l  (softmax)  |  RN32(exact sigmoid(l) + b[e])  (sigmoid + selection bias)
//   top-k by key, ties -> lower expert index, slot order = descending key
//   weights = softmax over all E (or sigmoid) of the selected experts, optional renormalise
//
// How: the dot products run on the fp64 tensor pipe (mma.sync m8n8k4). bf16 and fp32 inputs
// multiply exactly in fp64, so the only error is the summation. Each logit is then decided one
// of three ways, all exact:
//   1. certificate: when every product is a multiple of 2^q (from the rows' smallest exponents)
//      and the Cauchy-Schwarz bound on every partial sum is below 2^(q+53), the fp64 sum *is*
//      the exact sum and its round-to-nearest-even is the logit. This covers the exact ties that
//      bf16 data produce often (~0.8% of logits land exactly on an fp32 rounding midpoint);
//   2. enclosure: the error bound (d+16) 2^-52 (|x|_2 |W_e|_2 + |off|) leaves no fp32 rounding
//      boundary inside the interval, so RN32 of the fp64 value is the exact rounding;
//   3. otherwise (2 in 98,304 Quartz logits) a whole warp decides it after the main pass: it
//      scales every exact product to an integer multiple of the smallest power of two present,
//      sums them in int64, exactly, and compares with the boundaries. Only when the exponent span
//      exceeds 50 bits (or in a forced test mode) does one thread sum the products as a
//      non-overlapping floating-point expansion (Shewchuk's Grow-Expansion with zero
//      elimination) and decide from its sign.
// Sigmoid keys are screened the same way (fp64 exp within its documented error) and resolved
// in double-double arithmetic. So the integer routing decisions are exact, not merely tolerant.
#pragma once
#include "common.cuh"

namespace moe {

constexpr int RT_TM = 16;          // tokens per CTA
constexpr int RT_MT = RT_TM / 8;   // fp64 MMA row tiles per warp (each W fragment feeds all)
constexpr int RT_WARPS = 8;        // each a slice of the K dimension
constexpr int RT_THREADS = 32 * RT_WARPS;
constexpr int RT_KB = 16;          // k block: lane (row r, column c) of a fragment reads the 4
                                   // consecutive elements 4c..4c+3 of the block with one load
constexpr int RT_SEL_THREAD_MAX_E = 64;  // up to this many experts: one thread per (token,
                                         // expert) finds its rank; above, a warp per token
constexpr int EXPANSION_MAX = 40;
constexpr int RT_FIX_CAP = 256;   // flagged logits per CTA kept with their fp64 sums

// Expert tiles of 8 per round (a round covers 8*NT experts): the NT in {4,3,2,1} that wastes the
// fewest padded expert slots over all rounds, larger NT on ties.
inline int router_nt_for(int E) {
  int best = 4, waste = 1 << 30;
  for (int nt : {4, 3, 2, 1}) {
    const int eb = 8 * nt, w = ((E + eb - 1) / eb) * eb - E;
    if (w < waste) { waste = w; best = nt; }
  }
  return best;
}

// D(8x8) += A(8x4) B(4x8) in fp64 on the tensor cores. Fragments: lane l holds A[l/4][l%4],
// B[l%4][l/4] and D[l/4][2(l%4) + {0,1}]. Every product of bf16 or fp32 inputs is exact in fp64
// and each accumulation is an fp64 rounding, so the summation error bound below still holds.
__device__ __forceinline__ void dmma_8x8x4(double (&d)[2], double a, double b) {
  asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
               : "+d"(d[0]), "+d"(d[1])
               : "d"(a), "d"(b));
}

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
  unsigned int *counter; // completion counter of the statistics kernel, cleared here
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

template <typename Tin>
__device__ __noinline__ float exact_logit(const Tin *xrow, const Tin *wrow, int d, double off,
                                          double approx) {
  float r, up, dn;
  double mh, ml;
  rn32_certain(approx, 0.0, r, up, dn, mh, ml);
  Expansion X;
  X.n = 0;
  X.overflow = false;
  for (int i = 0; i < d; ++i) {
    const double p = __dmul_rn((double)Elem<Tin>::to_f(xrow[i]), (double)Elem<Tin>::to_f(wrow[i]));  // exact
    if (p != 0.0) expansion_add(X, p);
  }
  if (off != 0.0) expansion_add(X, off);
  expansion_add(X, -mh);                    // X = S - mid_hi
  const int c_hi = expansion_sign(X);
  expansion_add(X, mh - ml);                // X = S - mid_lo (difference exact)
  const int c_lo = expansion_sign(X);
  if (X.overflow) set_device_error(MOE_ERR_DEVICE_CHECK, INFO_EXPANSION_OVERFLOW);
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

// Warp-cooperative exact comparison of S = sum_i x_i W_i + off with two dyadic thresholds.
// Every product is exact in fp64 and so is a multiple of 2^lsb(p); with q the smallest such
// exponent over all terms and thresholds, every term is an integer multiple of 2^q and, when
// the exponent span is at most 50 bits, below 2^51, so their sum (at most d + 3 terms) is exact
// in int64. Returns false (caller falls back) when the span is wider or a term is subnormal.
// Eight consecutive elements of x (bf16 or fp32) as doubles, from a 16-byte aligned address.
__device__ __forceinline__ void load8(const __nv_bfloat16 *p, double *v) {
  const uint4 q = *(const uint4 *)p;
  const __nv_bfloat162 *h = (const __nv_bfloat162 *)&q;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}
__device__ __forceinline__ void load8(const float *p, double *v) {
  const float4 a = *(const float4 *)p, b = *(const float4 *)(p + 4);
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void load8(const double *p, double *v) {
#pragma unroll
  for (int i = 0; i < 8; i += 2) {
    const double2 q = *(const double2 *)(p + i);
    v[i] = q.x;
    v[i + 1] = q.y;
  }
}

template <typename Tin>
__device__ bool warp_exact_signs(const Tin *xrow, const Tin *wrow, int d, double off,
                                 double mh, double ml, int &c_hi, int &c_lo) {
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
  // lane covers elements [8*lane + 256*j, +8): d is a multiple of 64, so a chunk never straddles d
  for (int i = 8 * lane; i < d; i += 256) {
    double xv[8], wv[8];
    load8(xrow + i, xv);
    load8(wrow + i, wv);
#pragma unroll
    for (int u = 0; u < 8; ++u) scan(__dmul_rn(xv[u], wv[u]));
  }
  if (lane == 0) {
    scan(off);
    scan(mh);
    scan(ml);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    qmin = min(qmin, __shfl_xor_sync(0xffffffffu, qmin, o));
    emax = max(emax, __shfl_xor_sync(0xffffffffu, emax, o));
  }
  bad = __any_sync(0xffffffffu, bad);
  if (bad || emax - qmin > 50) return false;
  long long acc = 0;
  for (int i = 8 * lane; i < d; i += 256) {
    double xv[8], wv[8];
    load8(xrow + i, xv);
    load8(wrow + i, wv);
#pragma unroll
    for (int u = 0; u < 8; ++u) acc += (long long)ldexp(__dmul_rn(xv[u], wv[u]), -qmin);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  acc += (long long)ldexp(off, -qmin);
  const long long h = (long long)ldexp(mh, -qmin), l = (long long)ldexp(ml, -qmin);
  c_hi = acc > h ? 1 : (acc < h ? -1 : 0);
  c_lo = acc > l ? 1 : (acc < l ? -1 : 0);
  return true;
}

// Warp-cooperative resolution of one logit whose fp64 screen was undecided (or every logit in
// the forced test modes). Every lane calls it with the same arguments and gets the same result.
// `approx` is the fp64 sum of the main pass, within (d+16) 2^-52 |x||W_e| of the exact value -
// far below an fp32 step - so RN32 of the exact value is r = RN32(approx) or a neighbour; the
// exact integer comparison against the two rounding boundaries around r decides which, ties to
// even. force_level 2 skips the integer path and sends the logit to the single-thread
// expansion, to test that path too.
template <typename Tin>
__device__ __noinline__ float resolve_logit(const Tin *xrow, const Tin *wrow, int d, double off,
                                            double approx, int force_level) {
  const int lane = threadIdx.x & 31;
  float r, up, dn;
  double mh, ml;
  rn32_certain(approx, 0.0, r, up, dn, mh, ml);
  int c_hi, c_lo;
  if (force_level < 2 && fabs((double)r) < 0x1p126 &&
      warp_exact_signs<Tin>(xrow, wrow, d, off, mh, ml, c_hi, c_lo))
    return rn32_from_signs(r, up, dn, c_hi, c_lo);
  float l = 0.0f;
  if (lane == 0) l = exact_logit<Tin>(xrow, wrow, d, off, approx);
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

// ------------------------------------------------------------------ kernels
// Shared-memory layout of the router kernel (byte offsets), shared by host and device.
struct RouterSmem {
  size_t xs, xs_stride, part, sq, ex, lg, pb, keys, sel_e, sel_p, wn, wexp, cnt, flags, xnorm,
      xexp, fix, total;
};
__host__ __device__ inline RouterSmem router_smem(int E, int NT, bool sigmoid, int d, int esize) {
  RouterSmem L;
  const int EB = 8 * NT;
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t at = o; o = (o + bytes + 15) & ~(size_t)15; return at; };
  // the CTA's token rows, each padded by 32 bytes so that the 8 rows of an MMA fragment fall
  // on distinct bank pairs
  L.xs_stride = (size_t)d * esize + 32;
  L.xs = take((size_t)RT_TM * L.xs_stride);
  L.part = take((size_t)RT_WARPS * RT_TM * EB * sizeof(double));   // per-warp partial sums
  L.sq = take((size_t)RT_WARPS * (EB + RT_TM) * sizeof(double));   // per-warp sums of squares
  L.ex = take((size_t)RT_WARPS * (EB + RT_TM) * 2 * sizeof(int));  // per-warp exponent ranges
  L.lg = take((size_t)RT_TM * E * sizeof(float));
  const bool rank_sel = E <= RT_SEL_THREAD_MAX_E;
  L.pb = take(rank_sel ? (size_t)RT_TM * E * sizeof(float) : 0);
  L.keys = take(sigmoid ? (size_t)(rank_sel ? RT_TM : RT_WARPS) * E * sizeof(float) : 0);
  L.sel_e = take((size_t)RT_TM * 8 * sizeof(int));
  L.sel_p = take((size_t)RT_TM * 8 * sizeof(float));
  L.wn = take((size_t)EB * sizeof(double));
  L.wexp = take((size_t)EB * 2 * sizeof(int));
  L.cnt = take((size_t)E * sizeof(int));
  L.flags = take((size_t)RT_TM * ((E + 31) / 32) * sizeof(unsigned));
  L.xnorm = take(RT_TM * sizeof(double));
  L.xexp = take(RT_TM * 2 * sizeof(int));
  L.fix = take(RT_FIX_CAP * sizeof(double));
  L.total = o;
  return L;
}

// Raw 4-element fragment loads (bf16: 8 bytes; fp32: 16 bytes) and their conversion to fp64.
// Fragment digest: the four raw elements a lane loads per 16-k block become (1) fp64 MMA
// operands (a bf16 widens exactly to fp32 by a shift, then to fp64 by the conversion
// instruction), (2) an fp32 running sum of squares for the norm bound, (3) the running min / max
// magnitude key (the element's bits without the sign: key >> MANT is the biased exponent) over
// the nonzero elements, for the exactness certificate.
template <typename Tin> struct Frag4;
template <> struct Frag4<__nv_bfloat16> {
  using raw_t = uint2;
  static constexpr int MANT = 7;  // fraction bits
  static __device__ __forceinline__ raw_t load(const __nv_bfloat16 *p) { return __ldg((const uint2 *)p); }
  static __device__ __forceinline__ raw_t load_s(const __nv_bfloat16 *p) { return *(const uint2 *)p; }
  static __device__ __forceinline__ raw_t zero() { return make_uint2(0u, 0u); }
  static __device__ __forceinline__ void digest(raw_t q, double (&v)[4], float &sq, uint32_t &mn,
                                                uint32_t &mx) {
    const uint32_t w[2] = {q.x, q.y};
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t b = h ? (w[i] >> 16) : (w[i] & 0xFFFFu);
        const uint32_t m = b & 0x7FFFu;
        const float f = __uint_as_float(b << 16);
        sq = fmaf(f, f, sq);
        mn = min(mn, m ? m : 0xFFFFFFFFu);
        mx = max(mx, m);
        v[2 * i + h] = (double)f;
      }
  }
};
template <> struct Frag4<float> {
  using raw_t = float4;
  static constexpr int MANT = 23;
  static __device__ __forceinline__ raw_t load(const float *p) { return __ldg((const float4 *)p); }
  static __device__ __forceinline__ raw_t load_s(const float *p) { return *(const float4 *)p; }
  static __device__ __forceinline__ raw_t zero() { return make_float4(0.f, 0.f, 0.f, 0.f); }
  static __device__ __forceinline__ void digest(raw_t q, double (&v)[4], float &sq, uint32_t &mn,
                                                uint32_t &mx) {
    const float f[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[i] = f[i];
      sq = fmaf(f[i], f[i], sq);
      const uint32_t m = __float_as_uint(f[i]) & 0x7FFFFFFFu;
      mn = min(mn, m ? m : 0xFFFFFFFFu);
      mx = max(mx, m);
    }
  }
};

// Upper bound on sqrt(sum of squares) from an fp32 accumulation of at most n = d + 16 fused
// multiply-adds and additions: each step rounds with relative error <= 2^-24 or, in the
// subnormal range, absolute error <= 2^-150, so the exact sum is at most
// (computed + n 2^-149) (1 + n 2^-23) while n 2^-24 is small. Infinite or NaN input stays so.
__device__ __forceinline__ double norm_upper(double computed, int d) {
  const double n = (double)(d + 16);
  return sqrt((computed + n * 0x1p-149) * (1.0 + n * 0x1p-23));
}

template <typename Tin, int NT>
__global__ void __launch_bounds__(RT_THREADS, 2) router_kernel(RouterArgs a) {
  constexpr int EB = 8 * NT;  // experts per round
  using F = Frag4<Tin>;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const int E = a.E, d = a.d, k = a.k;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int fr = lane >> 2, fc = lane & 3;  // fragment row / column of this lane
  const int t0 = blockIdx.x * RT_TM;
  const int ntok = min(RT_TM, a.T - t0);
  const Tin *__restrict__ x = (const Tin *)a.x;
  const Tin *__restrict__ wr = (const Tin *)a.w;
  const int force_level = g_force_exact;
  const bool force = force_level != 0;
  const bool sigmoid = a.score == MOE_SCORE_SIGMOID;
  const RouterSmem SL = router_smem(E, NT, sigmoid, d, (int)sizeof(Tin));
  double *part = (double *)(smem_raw + SL.part);  // [RT_WARPS][RT_TM][EB]
  double *sq = (double *)(smem_raw + SL.sq);      // [RT_WARPS][EB + RT_TM]
  uint32_t *exr = (uint32_t *)(smem_raw + SL.ex);  // [RT_WARPS][EB + RT_TM][min, max] keys
  int *wexp = (int *)(smem_raw + SL.wexp);         // [EB][min, max] of the round's rows
  int *xexp = (int *)(smem_raw + SL.xexp);         // [RT_TM][min, max]
  float *lg = (float *)(smem_raw + SL.lg);
  float *keys = (float *)(smem_raw + SL.keys);
  const bool rank_sel = E <= RT_SEL_THREAD_MAX_E;
  float *pb = rank_sel ? (float *)(smem_raw + SL.pb) : lg;
  int *sel_e = (int *)(smem_raw + SL.sel_e);
  float *sel_p = (float *)(smem_raw + SL.sel_p);
  double *wn = (double *)(smem_raw + SL.wn);  // [EB] norms of the round's rows
  int *cnt = (int *)(smem_raw + SL.cnt);
  const int nfw = (E + 31) / 32;
  unsigned *flags = (unsigned *)(smem_raw + SL.flags);  // [RT_TM][nfw] undecided logits
  double *xnorm = (double *)(smem_raw + SL.xnorm);
  double *fix_s = (double *)(smem_raw + SL.fix);  // fp64 sums of the first RT_FIX_CAP flagged
  __shared__ int s_nfix;

  griddep_wait();
  griddep_launch();
  // ---- the CTA's token rows -> shared memory: one bulk copy per row, all in flight at once
  unsigned char *xs = smem_raw + SL.xs;
  const size_t xs_stride = SL.xs_stride;
  const uint32_t row_bytes = (uint32_t)d * (uint32_t)sizeof(Tin);
  __shared__ __align__(8) uint64_t s_xbar;
  __shared__ volatile int s_xabort;
  const uint32_t xbar = smem_u32(&s_xbar);
  if (tid == 0) {
    mbar_init(xbar, 1);
    s_xabort = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (tid == 0) {
    mbar_expect_tx(xbar, (uint32_t)ntok * row_bytes);
    for (int r = 0; r < ntok; ++r)
      bulk_load_1d(smem_u32(xs + (size_t)r * xs_stride), x + (size_t)(t0 + r) * d, row_bytes, xbar);
  }
  for (int r = ntok; r < RT_TM; ++r)  // rows past the last token read as zeros
    for (uint32_t i = tid; i < row_bytes / 16; i += RT_THREADS)
      ((uint4 *)(xs + (size_t)r * xs_stride))[i] = make_uint4(0u, 0u, 0u, 0u);
  for (int e = tid; e < E; e += RT_THREADS) cnt[e] = 0;
  for (int i = tid; i < RT_TM * nfw; i += RT_THREADS) flags[i] = 0u;
  if (tid == 0) s_nfix = 0;
  if (blockIdx.x == 0 && tid == 0) *a.counter = 0u;
  mbar_wait(xbar, 0u, (volatile int *)&s_xabort, g_wait_limit_ns, INFO_WAIT_ROUTER_X);
  __syncthreads();
  if (s_xabort) {  // the copies did not land in time: error recorded; let them drain, then leave
    if (tid == 0) {
      volatile int never = 0;
      mbar_wait(xbar, 0u, &never, g_wait_limit_ns, INFO_WAIT_DRAIN);
    }
    __syncthreads();
    return;
  }

  // ---- logits on the fp64 tensor cores, one round per 8*NT experts. Warp w takes the 16-k
  // blocks w, w+RT_WARPS, ... of the d dimension. For a block, the lane at fragment (row r, column c)
  // loads elements 4c..4c+3 of token rows r, r+8 (shared memory) and of expert row r of each
  // column tile (global memory, L2), and MMA step i uses element 4c+i: a permutation of k inside
  // the block, identical for both operands. Every element of the CTA's token rows and of the
  // round's expert rows is loaded exactly once per round, so the sums of squares of the loaded
  // values give |x_t| and |W_e| for the rounding bound. The per-warp partial sums are then
  // added in warp order.
  const int nkb = d / RT_KB;
  const Tin *xs_f[RT_MT];
#pragma unroll
  for (int mt = 0; mt < RT_MT; ++mt) xs_f[mt] = (const Tin *)(xs + (size_t)(fr + 8 * mt) * xs_stride) + 4 * fc;
  for (int eb = 0; eb < E; eb += EB) {
    double acc[RT_MT][NT][2];
    float xsq[RT_MT], wsq[NT];
    uint32_t xmn[RT_MT], xmx[RT_MT], wmn[NT], wmx[NT];
    const Tin *wrow_f[NT];
    bool e_ok[NT];
#pragma unroll
    for (int mt = 0; mt < RT_MT; ++mt) {
      xsq[mt] = 0.0f;
      xmn[mt] = 0xFFFFFFFFu;
      xmx[mt] = 0u;
#pragma unroll
      for (int j = 0; j < NT; ++j) acc[mt][j][0] = acc[mt][j][1] = 0.0;
    }
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      wsq[j] = 0.0f;
      wmn[j] = 0xFFFFFFFFu;
      wmx[j] = 0u;
      const int e = eb + 8 * j + fr;
      e_ok[j] = e < E;
      wrow_f[j] = wr + (size_t)(e_ok[j] ? e : 0) * d + 4 * fc;
    }
    // one-block-ahead prefetch of the raw fragments
    typename F::raw_t ra[RT_MT], rb[NT];
#pragma unroll
    for (int mt = 0; mt < RT_MT; ++mt) ra[mt] = F::zero();
#pragma unroll
    for (int j = 0; j < NT; ++j) rb[j] = F::zero();
    int kb = warp;
    if (kb < nkb) {
#pragma unroll
      for (int mt = 0; mt < RT_MT; ++mt) ra[mt] = F::load_s(xs_f[mt] + kb * RT_KB);
#pragma unroll
      for (int j = 0; j < NT; ++j) if (e_ok[j]) rb[j] = F::load(wrow_f[j] + kb * RT_KB);
    }
    for (; kb < nkb; kb += RT_WARPS) {
      double av[RT_MT][4], bv[NT][4];
#pragma unroll
      for (int mt = 0; mt < RT_MT; ++mt) F::digest(ra[mt], av[mt], xsq[mt], xmn[mt], xmx[mt]);
#pragma unroll
      for (int j = 0; j < NT; ++j) F::digest(rb[j], bv[j], wsq[j], wmn[j], wmx[j]);
      const int kn = kb + RT_WARPS;
      if (kn < nkb) {
#pragma unroll
        for (int mt = 0; mt < RT_MT; ++mt) ra[mt] = F::load_s(xs_f[mt] + kn * RT_KB);
#pragma unroll
        for (int j = 0; j < NT; ++j) rb[j] = e_ok[j] ? F::load(wrow_f[j] + kn * RT_KB) : F::zero();
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < NT; ++j)
#pragma unroll
          for (int mt = 0; mt < RT_MT; ++mt) dmma_8x8x4(acc[mt][j], av[mt][i], bv[j][i]);
    }
    // per-warp row sums of squares (lanes of one fragment row differ in fc = lane bits 0-1)
#pragma unroll
    for (int o = 1; o < 4; o <<= 1) {
#pragma unroll
      for (int mt = 0; mt < RT_MT; ++mt) {
        xsq[mt] += __shfl_xor_sync(0xffffffffu, xsq[mt], o);
        xmn[mt] = min(xmn[mt], __shfl_xor_sync(0xffffffffu, xmn[mt], o));
        xmx[mt] = max(xmx[mt], __shfl_xor_sync(0xffffffffu, xmx[mt], o));
      }
#pragma unroll
      for (int j = 0; j < NT; ++j) {
        wsq[j] += __shfl_xor_sync(0xffffffffu, wsq[j], o);
        wmn[j] = min(wmn[j], __shfl_xor_sync(0xffffffffu, wmn[j], o));
        wmx[j] = max(wmx[j], __shfl_xor_sync(0xffffffffu, wmx[j], o));
      }
    }
    if (fc == 0) {
#pragma unroll
      for (int j = 0; j < NT; ++j) {
        sq[warp * (EB + RT_TM) + 8 * j + fr] = wsq[j];
        exr[2 * (warp * (EB + RT_TM) + 8 * j + fr)] = wmn[j];
        exr[2 * (warp * (EB + RT_TM) + 8 * j + fr) + 1] = wmx[j];
      }
#pragma unroll
      for (int mt = 0; mt < RT_MT; ++mt) {
        sq[warp * (EB + RT_TM) + EB + fr + 8 * mt] = xsq[mt];
        exr[2 * (warp * (EB + RT_TM) + EB + fr + 8 * mt)] = xmn[mt];
        exr[2 * (warp * (EB + RT_TM) + EB + fr + 8 * mt) + 1] = xmx[mt];
      }
    }
#pragma unroll
    for (int mt = 0; mt < RT_MT; ++mt)
#pragma unroll
      for (int j = 0; j < NT; ++j)
#pragma unroll
        for (int h = 0; h < 2; ++h)
          part[(warp * RT_TM + fr + 8 * mt) * EB + 8 * j + 2 * fc + h] = acc[mt][j][h];
    __syncthreads();
    for (int q = tid; q < EB + RT_TM; q += RT_THREADS) {
      double t = 0.0;
      uint32_t mn = 0xFFFFFFFFu, mx = 0u;
#pragma unroll
      for (int w = 0; w < RT_WARPS; ++w) {
        t += sq[w * (EB + RT_TM) + q];
        mn = min(mn, exr[2 * (w * (EB + RT_TM) + q)]);
        mx = max(mx, exr[2 * (w * (EB + RT_TM) + q) + 1]);
      }
      // biased exponents of the smallest and largest nonzero magnitude; (255, -1): all zero
      const int emn = mx ? (int)(mn >> F::MANT) : 255, emx = mx ? (int)(mx >> F::MANT) : -1;
      if (q < EB) {
        wn[q] = norm_upper(t, d);
        wexp[2 * q] = emn;
        wexp[2 * q + 1] = emx;
      } else if (eb == 0) {
        xnorm[q - EB] = norm_upper(t, d);
        xexp[2 * (q - EB)] = emn;
        xexp[2 * (q - EB) + 1] = emx;
      }
    }
    __syncthreads();
    for (int q = tid; q < RT_TM * EB; q += RT_THREADS) {
      const int tt = q / EB, e = eb + q % EB;
      if (tt < ntok && e < E) {
        double s = 0.0;
#pragma unroll
        for (int w = 0; w < RT_WARPS; ++w) s += part[(w * RT_TM + tt) * EB + q % EB];
        const double o = a.off ? (double)a.off[e] : 0.0;
        s += o;
        // any summation order over d products plus the partials and the offset:
        // |error| <= gamma_{d+16} (sum |x_i W_i| + |off|) <= (d+16) 2^-52 (|x|_2 |W_e|_2 + |off|)
        const double B = (double)(d + 16) * 0x1p-52 * (xnorm[tt] * wn[q % EB] + fabs(o));
        // Exactness certificate. With biased exponents of at least xmin and wmin (all normal),
        // every product is an integer multiple of 2^qq, qq = xmin + wmin - 254 - 2 MANT, and so is
        // the offset when its own quantum is folded in. Every partial sum, in any order, is
        // bounded by sum |x_i W_i| + |off| <= |x|_2 |W_e|_2 + |off| (Cauchy-Schwarz); xnorm and wn
        // are upper bounds of the norms and the factor covers this line's own rounding. Below
        // 2^(qq + 53) every partial sum
        // is an fp64 value, so s is the exact sum and its round-to-nearest-even to fp32 is the
        // canonical logit, exact ties included.
        bool exact;
        {
          const int xmn_ = xexp[2 * tt], xmx_ = xexp[2 * tt + 1];
          const int wmn_ = wexp[2 * (q % EB)], wmx_ = wexp[2 * (q % EB) + 1];
          int qq = 1 << 20;
          if (xmx_ >= 0 && wmx_ >= 0) qq = xmn_ + wmn_ - 254 - 2 * F::MANT;
          bool ok = (xmx_ < 0 || wmx_ < 0 || (xmn_ > 0 && wmn_ > 0)) && xmx_ < 255 && wmx_ < 255;
          if (o != 0.0) {
            const int eo = (int)((__float_as_uint((float)o) >> 23) & 0xFFu);
            ok = ok && eo > 0 && eo < 255;
            qq = min(qq, eo - 150);
          }
          const double S = (xnorm[tt] * wn[q % EB] + fabs(o)) * (1.0 + (double)(d + 8) * 0x1p-50);
          exact = ok && S <= ldexp(1.0, min(qq + 53, 1023));
        }
        float r, up, dn;
        double mh, ml;
        float l;
        if (exact && !force) {
          l = __double2float_rn(s);
        } else if (rn32_certain(s, B, r, up, dn, mh, ml) && !force) {
          l = r;
        } else {
          // undecided: resolved exactly by the fixup pass below, which needs the fp64 sum
          const int slot = atomicAdd(&s_nfix, 1);
          if (slot < RT_FIX_CAP) {
            fix_s[slot] = s;
            l = __int_as_float(slot);  // the slot index rides in the logit until resolved
          } else {
            l = __int_as_float(-1);    // overflow (forced test modes): the fixup recomputes
          }
          atomicOr(&flags[tt * nfw + (e >> 5)], 1u << (e & 31));
        }
        lg[tt * E + e] = l;
      }
    }
    __syncthreads();  // part, sq and wn are rewritten by the next round
  }

  // ---- fixup of undecided logits: flag words dealt round-robin to the warps; one warp decides
  // one logit exactly (see resolve_logit)
  for (int wi = warp; wi < ntok * nfw; wi += RT_THREADS / 32) {
    unsigned m = flags[wi];
    const int tt = wi / nfw, e0 = (wi % nfw) * 32;
    while (m) {
      const int ee = e0 + __ffs(m) - 1;
      m &= m - 1;
      const int slot = __float_as_int(lg[tt * E + ee]);
      const Tin *xrow = x + (size_t)(t0 + tt) * d;
      const Tin *wrow = wr + (size_t)ee * d;
      const double o = a.off ? (double)a.off[ee] : 0.0;
      double approx;
      if (slot >= 0 && slot < RT_FIX_CAP) {
        approx = fix_s[slot];
      } else {
        double s = 0.0;
        for (int i = lane; i < d; i += 32)
          s = fma((double)Elem<Tin>::to_f(xrow[i]), (double)Elem<Tin>::to_f(wrow[i]), s);
        approx = warp_sum_d(s) + o;
      }
      const float l = resolve_logit<Tin>(xrow, wrow, d, o, approx, force_level);
      __syncwarp();
      if (lane == 0) lg[tt * E + ee] = l;
      __syncwarp();
    }
  }
  __syncthreads();

  // ---- selection
  if (rank_sel) {
    // up to 64 experts: every (token, expert) pair finds its own rank among the token's keys
    if (sigmoid)
      for (int q = tid; q < ntok * E; q += RT_THREADS)
        keys[q] = sigmoid_key(lg[q], a.bias ? a.bias[q % E] : 0.0f, force);
    __syncthreads();
    // the token's max logit and normaliser, once per token (one warp per token, fixed order)
    __shared__ float s_tok_m[RT_TM], s_tok_inv[RT_TM];
    for (int tt = warp; tt < ntok; tt += RT_THREADS / 32) {
      const float *lrow = lg + tt * E;
      float m = -INFINITY;
      for (int e = lane; e < E; e += 32) m = fmaxf(m, lrow[e]);
      m = warp_max_f(m);
      float ssum = 0.0f;
      if (!sigmoid)
        for (int e = lane; e < E; e += 32) ssum += expf(lrow[e] - m);
      else
        for (int e = lane; e < E; e += 32) ssum += 1.0f / (1.0f + expf(-lrow[e]));
      ssum = warp_sum_f(ssum);
      if (lane == 0) {
        s_tok_m[tt] = m;
        s_tok_inv[tt] = 1.0f / ssum;
      }
    }
    __syncthreads();
    for (int q = tid; q < ntok * E; q += RT_THREADS) {
      const int tt = q / E, e = q - tt * E;
      const float *krow = (sigmoid ? keys : lg) + tt * E;
      float v = krow[e];
      if (v != v) v = -INFINITY;
      int rank = 0;
      for (int e2 = 0; e2 < E; ++e2) {
        float v2 = krow[e2];
        if (v2 != v2) v2 = -INFINITY;
        rank += (v2 > v || (v2 == v && e2 < e)) ? 1 : 0;
      }
      const float inv = s_tok_inv[tt];
      const float l = lg[tt * E + e];
      float p, pbasis;
      if (!sigmoid) {
        p = expf(l - s_tok_m[tt]) * inv;
        pbasis = p;
      } else {
        p = 1.0f / (1.0f + expf(-l));
        pbasis = p * inv;
      }
      pb[q] = pbasis;
      if (rank < k) {
        sel_e[tt * 8 + rank] = e;
        sel_p[tt * 8 + rank] = p;
      }
    }
    __syncthreads();
    if (tid < ntok) {
      const int t = t0 + tid;
      float psel = 0.0f;
      for (int j = 0; j < k; ++j) psel += sel_p[tid * 8 + j];
      for (int j = 0; j < k; ++j) {
        const int e = sel_e[tid * 8 + j];
        const float pj = sel_p[tid * 8 + j];
        a.idx[(size_t)t * k + j] = e;
        a.wts[(size_t)t * k + j] = a.norm ? pj / psel : pj;
        atomicAdd(&cnt[e], 1);
      }
    }
    __syncthreads();
  } else {
    // one warp per token
  for (int tt = warp; tt < ntok; tt += RT_THREADS / 32) {
    const int t = t0 + tt;
    float *lrow = lg + tt * E;
    const float *krow = lrow;
    if (a.score == MOE_SCORE_SIGMOID) {
      float *kw = keys + warp * E;
      for (int e = lane; e < E; e += 32) kw[e] = sigmoid_key(lrow[e], a.bias ? a.bias[e] : 0.0f, force);
      __syncwarp();
      krow = kw;
    }
    unsigned selmask = 0u;
    int sel[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      sel[j] = 0;
      if (j < k) {
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
          if (oe != 0x7fffffff &&
              (be == 0x7fffffff || ok > bk || (ok == bk && oe < be))) { bk = ok; be = oe; }
        }
        sel[j] = be;
        if ((be & 31) == lane) selmask |= 1u << (be >> 5);
      }
    }
    // probabilities
    float pj = 0.0f;
    if (a.score == MOE_SCORE_SOFTMAX) {
      float m = -INFINITY;
      for (int e = lane; e < E; e += 32) m = fmaxf(m, lrow[e]);
      m = warp_max_f(m);
      float s = 0.0f;
      for (int e = lane; e < E; e += 32) s += expf(lrow[e] - m);
      s = warp_sum_f(s);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (j < k && lane == j) pj = expf(lrow[sel[j]] - m) / s;
      __syncwarp();
      for (int e = lane; e < E; e += 32) lrow[e] = expf(lrow[e] - m) / s;
    } else {
      float s = 0.0f;
      for (int e = lane; e < E; e += 32) s += 1.0f / (1.0f + expf(-lrow[e]));
      s = warp_sum_f(s);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (j < k && lane == j) pj = 1.0f / (1.0f + expf(-lrow[sel[j]]));
      __syncwarp();
      for (int e = lane; e < E; e += 32) lrow[e] = (1.0f / (1.0f + expf(-lrow[e]))) / s;
    }
    float psel = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float v = __shfl_sync(0xffffffffu, pj, j);
      if (j < k) psel += v;
    }
    if (lane < k) {
      int e_out = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) if (j == lane) e_out = sel[j];
      a.idx[(size_t)t * k + lane] = e_out;
      a.wts[(size_t)t * k + lane] = a.norm ? pj / psel : pj;
      atomicAdd(&cnt[e_out], 1);
    }
    __syncwarp();
  }
  __syncthreads();
  }

  // ---- per-CTA statistics (fixed token order), then the last CTA reduces in CTA order
  for (int e = tid; e < E; e += RT_THREADS) {
    float ps = 0.0f;
    for (int tt = 0; tt < ntok; ++tt) ps += pb[tt * E + e];
    a.part_cnt[(size_t)blockIdx.x * E + e] = cnt[e];
    a.part_prob[(size_t)blockIdx.x * E + e] = ps;
  }
}

}  // namespace moe

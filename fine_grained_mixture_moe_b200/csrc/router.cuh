// Router: logits, selection keys, top-k, combine weights and per-expert statistics.
//
// What it computes (Quartz "Router: top-6 of 24", Moonfrost "a router picks the top 3",
// Sutra-1.3B "top-4 routing with sigmoid scoring and bias-based load balancing"):
//   l[t,e]  = RN32(exact sum_i x[t,i] W[e,i] + off[e])              (fp32, canonical)
//   key     = l  (softmax)  |  RN32(exact sigmoid(l) + b[e])  (sigmoid + selection bias)
//   top-k by key, ties -> lower expert index, slot order = descending key
//   weights = softmax over all E (or sigmoid) of the selected experts, optional renormalise
//
// How: the dot products run on the fp64 FMA pipe. bf16 and fp32 inputs multiply exactly in
// fp64, so the only error is the summation, bounded by (d+2) 2^-52 (|x|_2 |W_e|_2 + |off|).
// When that enclosure holds no fp32 rounding boundary, RN32 of the fp64 value *is* the exact
// rounding. Otherwise the logit is marked and, after the main pass, a whole warp decides it
// exactly: bf16 products carry at most 16 significant bits, so the exact sum of a row is a
// multiple of a small power of two and lands exactly on an fp32 rounding boundary for about
// 0.4% of logits - genuine ties that no error bound can settle. The warp scales every exact
// product to an integer multiple of the smallest power of two present and sums them in int64,
// exactly, then compares with the boundaries. Only when the exponent span exceeds 50 bits (or
// in a forced test mode) does one thread sum the products as a non-overlapping floating-point
// expansion (Shewchuk's Grow-Expansion with zero elimination) and decide from its sign. Sigmoid keys are
// screened the same way (fp64 exp, documented 1-ulp) and resolved in double-double arithmetic.
// So the integer routing decisions are exact, not merely tolerant.
#pragma once
#include "common.cuh"

namespace moe {

constexpr int RT_TM = 16;          // tokens per CTA
constexpr int RT_THREADS = 256;    // 8 warps, each a slice of the K dimension
constexpr int RT_KC = 32;          // k-chunk staged (fp64) in a warp's shared-memory slot
constexpr int RT_LD = RT_KC + 2;   // padded row: 68 words = 4 (mod 32), conflict-free 16 B loads
constexpr int EXPANSION_MAX = 40;
constexpr int RT_FIX_CAP = 256;   // flagged logits per CTA kept with their fp64 sums

// Experts per thread in one round (a round covers 4*RE experts): the RE in {8,6,4,2} that wastes
// the fewest padded expert slots over all rounds, larger RE on ties.
inline int router_re_for(int E) {
  int best = 8, waste = 1 << 30;
  for (int re : {8, 6, 4, 2}) {
    const int eb = 4 * re, w = ((E + eb - 1) / eb) * eb - E;
    if (w < waste) { waste = w; best = re; }
  }
  return best;
}

struct RouterArgs {
  const void *x;
  const double *w64;    // [E, d] router weight in fp64 (prep kernel)
  const double *wnorm;  // [E] l2 norms
  const float *off;     // [E] or null
  const float *bias;    // [E] or null
  int T, d, E, k, score, norm;
  int32_t *idx;
  float *wts;
  int32_t *part_cnt;    // [nblk, E]
  float *part_prob;     // [nblk, E]
  int32_t *count_out;   // [E]
  float *prob_out;      // [E]
  unsigned int *counter;
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
__device__ __noinline__ float exact_logit(const Tin *xrow, const double *wrow, int d, double off,
                                          double approx) {
  float r, up, dn;
  double mh, ml;
  rn32_certain(approx, 0.0, r, up, dn, mh, ml);
  Expansion X;
  X.n = 0;
  X.overflow = false;
  for (int i = 0; i < d; ++i) {
    const double p = __dmul_rn((double)Elem<Tin>::to_f(xrow[i]), wrow[i]);  // exact
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
__device__ bool warp_exact_signs(const Tin *xrow, const double *wrow, int d, double off,
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
__device__ __noinline__ float resolve_logit(const Tin *xrow, const double *wrow, int d, double off,
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

// RN32(sigmoid(l) + b), exact. fp64 screen first unless forced.
__device__ float sigmoid_key(float l, float b, bool force) {
  const double s = 1.0 / (1.0 + exp(-(double)l));
  const double v = s + (double)b;
  const double B = 0x1p-48 * s + 0x1p-52 * fabs(v) + 1e-300;
  float r, up, dn;
  double mh, ml;
  if (rn32_certain(v, B, r, up, dn, mh, ml) && !force) return r;
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
  // recompute the candidate around the dd value in case the screen's r was a neighbour off
  return rn32_from_signs(r, up, dn, c_hi, c_lo);
}

// ------------------------------------------------------------------ kernels
// fp64 copy of the router weight and its row norms; also clears the completion counter.
template <typename Tin>
__global__ void __launch_bounds__(256) router_prep_kernel(const Tin *__restrict__ w, int E, int d,
                                                          double *__restrict__ w64,
                                                          double *__restrict__ wnorm,
                                                          unsigned *counter) {
  const int e = blockIdx.x;
  double s = 0.0;
  for (int i = threadIdx.x; i < d; i += blockDim.x) {
    const double v = (double)Elem<Tin>::to_f(w[(size_t)e * d + i]);
    w64[(size_t)e * d + i] = v;
    s = fma(v, v, s);
  }
  __shared__ double red[8];
  s = warp_sum_d(s);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int i = 0; i < (int)(blockDim.x >> 5); ++i) t += red[i];
    wnorm[e] = sqrt(t);
    if (e == 0) *counter = 0u;
  }
}

__host__ __device__ inline size_t router_smem_bytes(int E, int RE) {
  size_t b = (size_t)(RT_THREADS / 32) * (RT_TM + 4 * RE) * RT_LD * sizeof(double);  // staging
  b += (size_t)RT_TM * E * sizeof(float);                  // logits / probabilities
  b += (size_t)(RT_THREADS / 32) * E * sizeof(float);      // per-warp sigmoid keys
  b += (size_t)E * sizeof(int);                             // selection counts
  b += (size_t)RT_TM * ((E + 31) / 32) * sizeof(unsigned);  // undecided-logit flags
  b = (b + 15) & ~(size_t)15;
  b += RT_TM * sizeof(double);                              // token norms
  b += (size_t)RT_FIX_CAP * sizeof(double);                 // fp64 sums of flagged logits
  return b;
}

template <typename Tin, int RE>
__global__ void __launch_bounds__(RT_THREADS, 2) router_kernel(RouterArgs a) {
  constexpr int EB = 4 * RE;  // experts per round
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const int E = a.E, d = a.d, k = a.k;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int lt = lane >> 2, le = lane & 3;  // thread tile: tokens {lt, lt+8} x experts {le+4j}
  const int t0 = blockIdx.x * RT_TM;
  const int ntok = min(RT_TM, a.T - t0);
  const Tin *__restrict__ x = (const Tin *)a.x;
  const int force_level = g_force_exact;
  const bool force = force_level != 0;

  double *stage = (double *)smem_raw;
  double *xs = stage + warp * (RT_TM + EB) * RT_LD;  // this warp's [16][RT_LD] x chunk
  double *wsm = xs + RT_TM * RT_LD;                  // this warp's [EB][RT_LD] W chunk
  double *part = stage;                              // reused: [8 warps][16][EB] partial sums
  float *lg = (float *)(stage + (RT_THREADS / 32) * (RT_TM + EB) * RT_LD);
  float *keys = lg + RT_TM * E;
  int *cnt = (int *)(keys + (RT_THREADS / 32) * E);
  const int nfw = (E + 31) / 32;
  unsigned *flags = (unsigned *)(cnt + E);  // [RT_TM][nfw] undecided logits
  double *xnorm = (double *)(((uintptr_t)(flags + RT_TM * nfw) + 15) & ~(uintptr_t)15);
  double *fix_s = xnorm + RT_TM;  // fp64 sums of the first RT_FIX_CAP flagged logits
  __shared__ int s_nfix;

  for (int e = tid; e < E; e += RT_THREADS) cnt[e] = 0;
  for (int i = tid; i < RT_TM * nfw; i += RT_THREADS) flags[i] = 0u;
  if (tid == 0) s_nfix = 0;
  for (int tt = warp; tt < RT_TM; tt += RT_THREADS / 32) {
    double s = 0.0;
    if (tt < ntok) {
      const Tin *row = x + (size_t)(t0 + tt) * d;
      for (int i = lane; i < d; i += 32) {
        const double v = (double)Elem<Tin>::to_f(row[i]);
        s = fma(v, v, s);
      }
    }
    s = warp_sum_d(s);
    if (lane == 0) xnorm[tt] = sqrt(s);
  }

  // ---- logits. Warp w sums the k-chunks w, w+8, ... of every (token, expert) of the round;
  // the eight partial sums are then added in warp order. Both operands sit in shared memory
  // as fp64: one 16-byte load of x serves 4 lanes and one of W serves 8, so a warp issues one
  // wavefront per load and 2*RE fp64 FMAs per pair of loads.
  const int nchunk = d / RT_KC;
  for (int eb = 0; eb < E; eb += EB) {
    double acc[2][RE];
#pragma unroll
    for (int j = 0; j < RE; ++j) acc[0][j] = acc[1][j] = 0.0;
    for (int c = warp; c < nchunk; c += RT_THREADS / 32) {
      const int k0 = c * RT_KC;
      {  // x chunk: lane -> token lane/2, 16 consecutive k
        const int tt = lane >> 1, h = (lane & 1) * 16;
        double *dst = xs + tt * RT_LD + h;
        if (tt < ntok) {
          const Tin *src = x + (size_t)(t0 + tt) * d + k0 + h;
#pragma unroll
          for (int i = 0; i < 16; i += 2)
            *(double2 *)(dst + i) = make_double2((double)Elem<Tin>::to_f(src[i]),
                                                 (double)Elem<Tin>::to_f(src[i + 1]));
        } else {
#pragma unroll
          for (int i = 0; i < 16; i += 2) *(double2 *)(dst + i) = make_double2(0.0, 0.0);
        }
      }
      for (int i = lane; i < EB * (RT_KC / 2); i += 32) {  // W chunk from the fp64 copy
        const int e = i / (RT_KC / 2), kp = (i % (RT_KC / 2)) * 2;
        double2 wv = make_double2(0.0, 0.0);
        if (eb + e < E) wv = *(const double2 *)(a.w64 + (size_t)(eb + e) * d + k0 + kp);
        *(double2 *)(wsm + e * RT_LD + kp) = wv;
      }
      __syncwarp();
#pragma unroll 4
      for (int kk = 0; kk < RT_KC; kk += 2) {
        const double2 x0 = *(const double2 *)(xs + lt * RT_LD + kk);
        const double2 x1 = *(const double2 *)(xs + (lt + 8) * RT_LD + kk);
#pragma unroll
        for (int j = 0; j < RE; ++j) {
          const double2 wv = *(const double2 *)(wsm + (le + 4 * j) * RT_LD + kk);
          acc[0][j] = fma(x0.x, wv.x, acc[0][j]);
          acc[0][j] = fma(x0.y, wv.y, acc[0][j]);
          acc[1][j] = fma(x1.x, wv.x, acc[1][j]);
          acc[1][j] = fma(x1.y, wv.y, acc[1][j]);
        }
      }
      __syncwarp();
    }
    __syncthreads();  // staging slots become the partial-sum buffer
#pragma unroll
    for (int j = 0; j < RE; ++j) {
      part[(warp * RT_TM + lt) * EB + le + 4 * j] = acc[0][j];
      part[(warp * RT_TM + lt + 8) * EB + le + 4 * j] = acc[1][j];
    }
    __syncthreads();
    for (int q = tid; q < RT_TM * EB; q += RT_THREADS) {
      const int tt = q / EB, e = eb + q % EB;
      if (tt < ntok && e < E) {
        double s = 0.0;
#pragma unroll
        for (int w = 0; w < RT_THREADS / 32; ++w) s += part[(w * RT_TM + tt) * EB + q % EB];
        const double o = a.off ? (double)a.off[e] : 0.0;
        s += o;
        // any summation order over d products plus 8 partials and the offset:
        // |error| <= gamma_{d+16} (sum |x_i W_i| + |off|) <= (d+16) 2^-52 (|x|_2 |W_e|_2 + |off|)
        const double B = (double)(d + 16) * 0x1p-52 * (xnorm[tt] * a.wnorm[e] + fabs(o));
        float r, up, dn;
        double mh, ml;
        float l;
        if (rn32_certain(s, B, r, up, dn, mh, ml) && !force) {
          l = r;
        } else {
          // undecided: resolved exactly by the fixup pass below, which needs the fp64 sum
          const int slot = atomicAdd(&s_nfix, 1);
          if (slot < RT_FIX_CAP) {
            fix_s[slot] = s;
            l = __int_as_float(slot);  // the slot index rides in the logit until resolved
            atomicOr(&flags[tt * nfw + (e >> 5)], 1u << (e & 31));
          } else {
            // overflow (forced test modes only): the fixup recomputes the fp64 sum
            l = __int_as_float(-1);
            atomicOr(&flags[tt * nfw + (e >> 5)], 1u << (e & 31));
          }
        }
        lg[tt * E + e] = l;
      }
    }
    __syncthreads();  // the partial-sum buffer is the next round's staging area
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
      const double *wrow = a.w64 + (size_t)ee * d;
      const double o = a.off ? (double)a.off[ee] : 0.0;
      double approx;
      if (slot >= 0 && slot < RT_FIX_CAP) {
        approx = fix_s[slot];
      } else {
        double s = 0.0;
        for (int i = lane; i < d; i += 32) s = fma((double)Elem<Tin>::to_f(xrow[i]), wrow[i], s);
        approx = warp_sum_d(s) + o;
      }
      const float l = resolve_logit<Tin>(xrow, wrow, d, o, approx, force_level);
      __syncwarp();
      if (lane == 0) lg[tt * E + ee] = l;
      __syncwarp();
    }
  }
  __syncthreads();

  // ---- selection, one warp per token
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

  // ---- per-CTA statistics (fixed token order), then the last CTA reduces in CTA order
  for (int e = tid; e < E; e += RT_THREADS) {
    float ps = 0.0f;
    for (int tt = 0; tt < ntok; ++tt) ps += lg[tt * E + e];
    a.part_cnt[(size_t)blockIdx.x * E + e] = cnt[e];
    a.part_prob[(size_t)blockIdx.x * E + e] = ps;
  }
}

// Per-expert totals of the per-CTA selection counts and probability sums: one block per
// expert; thread t adds the CTAs t, t+128, ... in order, then a fixed-shape tree combines the
// 128 partial sums, so prob_sum is bitwise reproducible.
__global__ void __launch_bounds__(128) router_reduce_kernel(const int32_t *__restrict__ part_cnt,
                                                            const float *__restrict__ part_prob,
                                                            int nblk, int E,
                                                            int32_t *__restrict__ count_out,
                                                            float *__restrict__ prob_out) {
  const int e = blockIdx.x, tid = threadIdx.x;
  int c = 0;
  float p = 0.0f;
  for (int b = tid; b < nblk; b += 128) {
    c += part_cnt[(size_t)b * E + e];
    p += part_prob[(size_t)b * E + e];
  }
  __shared__ int sc[4];
  __shared__ float sp[4];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    c += __shfl_xor_sync(0xffffffffu, c, o);
    p += __shfl_xor_sync(0xffffffffu, p, o);
  }
  if ((tid & 31) == 0) {
    sc[tid >> 5] = c;
    sp[tid >> 5] = p;
  }
  __syncthreads();
  if (tid == 0) {
    count_out[e] = (sc[0] + sc[1]) + (sc[2] + sc[3]);
    prob_out[e] = (sp[0] + sp[1]) + (sp[2] + sp[3]);
  }
}

}  // namespace moe

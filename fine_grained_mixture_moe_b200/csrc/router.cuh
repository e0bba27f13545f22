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
// rounding. Otherwise (about 1 logit in 10^5 at these sizes) the thread recomputes the sum
// exactly as a non-overlapping floating-point expansion (Shewchuk's Grow-Expansion with zero
// elimination) and decides the rounding from its sign against the boundary. Sigmoid keys are
// screened the same way (fp64 exp, documented 1-ulp) and resolved in double-double arithmetic.
// So the integer routing decisions are exact, not merely tolerant.
#pragma once
#include "common.cuh"

namespace moe {

constexpr int RT_TM = 32;       // tokens per CTA (one per lane)
constexpr int RT_THREADS = 256; // 8 warps
constexpr int RT_KC = 128;      // k-chunk of x staged in fp64
constexpr int RT_EWMAX = 8;     // experts per warp per round
constexpr int EXPANSION_MAX = 40;

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

__host__ __device__ inline size_t router_smem_bytes(int E) {
  size_t b = (size_t)RT_TM * (RT_KC + 1) * sizeof(double);  // x chunk (fp64)
  b += (size_t)RT_TM * E * sizeof(float);                  // logits / probabilities
  b += (size_t)(RT_THREADS / 32) * E * sizeof(float);      // per-warp sigmoid keys
  b += (size_t)E * sizeof(int);                             // selection counts
  b = (b + 15) & ~(size_t)15;
  b += RT_TM * sizeof(double);                              // token norms
  return b;
}

template <typename Tin>
__global__ void __launch_bounds__(RT_THREADS) router_kernel(RouterArgs a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const int E = a.E, d = a.d, k = a.k;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int t0 = blockIdx.x * RT_TM;
  const int ntok = min(RT_TM, a.T - t0);
  const Tin *__restrict__ x = (const Tin *)a.x;
  const bool force = g_force_exact != 0;

  double *xs = (double *)smem_raw;
  float *lg = (float *)(xs + RT_TM * (RT_KC + 1));
  float *keys = lg + RT_TM * E;
  int *cnt = (int *)(keys + (RT_THREADS / 32) * E);
  double *xnorm = (double *)(((uintptr_t)(cnt + E) + 15) & ~(uintptr_t)15);

  for (int e = tid; e < E; e += RT_THREADS) cnt[e] = 0;
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

  // ---- logits: warp w owns experts [e0, e0+ne) of each round, lane owns token t0+lane
  const int ew = min(RT_EWMAX, (E + 7) / 8);
  const int per_round = 8 * ew;
  for (int eb = 0; eb < E; eb += per_round) {
    double acc[RT_EWMAX];
#pragma unroll
    for (int j = 0; j < RT_EWMAX; ++j) acc[j] = 0.0;
    const int e0 = eb + warp * ew;
    const int ne = max(0, min(ew, E - e0));
    for (int kc = 0; kc < d; kc += RT_KC) {
      const int kn = min(RT_KC, d - kc);
      __syncthreads();
      for (int i = tid; i < RT_TM * kn; i += RT_THREADS) {
        const int r = i / kn, c = i - r * kn;
        double v = 0.0;
        if (r < ntok) v = (double)Elem<Tin>::to_f(x[(size_t)(t0 + r) * d + kc + c]);
        xs[r * (RT_KC + 1) + c] = v;
      }
      __syncthreads();
      if (ne > 0) {
        const double *xrow = xs + lane * (RT_KC + 1);
        const double *wbase = a.w64 + (size_t)e0 * d + kc;
        for (int c = 0; c < kn; c += 2) {
          const double x0 = xrow[c], x1 = xrow[c + 1];
#pragma unroll
          for (int j = 0; j < RT_EWMAX; ++j) {
            if (j < ne) {
              const double2 wv = *(const double2 *)(wbase + (size_t)j * d + c);
              acc[j] = fma(x0, wv.x, acc[j]);
              acc[j] = fma(x1, wv.y, acc[j]);
            }
          }
        }
      }
    }
    if (lane < ntok) {
#pragma unroll
      for (int j = 0; j < RT_EWMAX; ++j) {
        if (j < ne) {
          const int e = e0 + j;
          const double o = a.off ? (double)a.off[e] : 0.0;
          const double s = acc[j] + o;
          const double B = (double)(d + 2) * 0x1p-52 * (xnorm[lane] * a.wnorm[e] + fabs(o));
          float r, up, dn;
          double mh, ml;
          float l;
          if (rn32_certain(s, B, r, up, dn, mh, ml) && !force) l = r;
          else l = exact_logit<Tin>(x + (size_t)(t0 + lane) * d, a.w64 + (size_t)e * d, d, o, s);
          lg[lane * E + e] = l;
        }
      }
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
  __threadfence();
  __syncthreads();
  __shared__ int s_last;
  if (tid == 0) s_last = (atomicAdd(a.counter, 1u) == gridDim.x - 1);
  __syncthreads();
  if (s_last) {
    __threadfence();
    const int nb = gridDim.x;
    for (int e = tid; e < E; e += RT_THREADS) {
      int c = 0;
      float p = 0.0f;
      for (int b = 0; b < nb; ++b) {
        c += __ldcg(a.part_cnt + (size_t)b * E + e);
        p += __ldcg(a.part_prob + (size_t)b * E + e);
      }
      a.count_out[e] = c;
      a.prob_out[e] = p;
    }
    if (tid == 0) *a.counter = 0u;
  }
}

}  // namespace moe

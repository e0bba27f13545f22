// Backward of the combine and of the router: the derivative of the forward, with no gradient
// through the selection, the capacity drops or the loss's counts, none for the selection bias or
// the logit offsets, and the logits' fp32 rounding taken with derivative 1.
//
// combine_backward (Moonfrost expert card: a token's output sums its shared and top-k routed
// experts): for every kept pair (t, j) with p = slot_pos[t, j] >= 0,
//   dy_perm[p]     = topk_w[t, j] * dy[t]
//   d_topk_w[t, j] = sum_c dy[t, c] * y_perm[p, c]     (0 for a dropped pair)
// route_backward, per token:
//   l = x W_r^T + off (fp32 FMAs), p = softmax(l) or sigmoid(l);
//   dp from d_topk_w, through w_j = p_j / sum of the k selected p_j when norm_topk is set;
//   the loss term dq_i = dL alpha E f_i / T, f_i = count_i / (T k) (Quartz research page,
//   architecture table, row "Router": load-balancing weight 0.01), which for sigmoid scores
//   enters through q = sigmoid / sum over all E;
//   d_logits = p (dp + dq - <dp + dq, p>) (softmax) or dsigma sigma (1 - sigma) (sigmoid).
// then d_w_router = d_logits^T x and dx = d_logits W_r, every sum in a fixed order (the first
// split over token ranges, the partial sums kept in dx until dx itself is written).
#pragma once
#include "common.cuh"

namespace moe {

// detail code (g_err_info) of a selected expert index outside [0, E) in the backward's input
constexpr long long INFO_BAD_EXPERT_INDEX = 3;

// four consecutive elements of a row, as fp32
template <typename Ty> struct Bw4;
template <> struct Bw4<float> {
  static __device__ __forceinline__ float4 ld(const float *p) { return *(const float4 *)p; }
  static __device__ __forceinline__ void st(float *p, float4 v) { *(float4 *)p = v; }
};
template <> struct Bw4<__nv_bfloat16> {
  static __device__ __forceinline__ float4 ld(const __nv_bfloat16 *p) {
    const uint2 u = *(const uint2 *)p;
    const float2 a = __bfloat1622float2(*(const __nv_bfloat162 *)&u.x);
    const float2 b = __bfloat1622float2(*(const __nv_bfloat162 *)&u.y);
    return make_float4(a.x, a.y, b.x, b.y);
  }
  static __device__ __forceinline__ void st(__nv_bfloat16 *p, float4 v) {
    const __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y);
    const __nv_bfloat162 b = __floats2bfloat162_rn(v.z, v.w);
    uint2 u;
    u.x = *(const uint32_t *)&a;
    u.y = *(const uint32_t *)&b;
    *(uint2 *)p = u;
  }
};

// eight consecutive elements of a row: loaded raw (one 16-byte access for bf16, two for fp32),
// then widened to fp32
template <typename Ty> struct Bw8;
template <> struct Bw8<float> {
  struct Raw { float4 a, b; };
  static __device__ __forceinline__ Raw ld(const float *p) {
    return Raw{((const float4 *)p)[0], ((const float4 *)p)[1]};
  }
  static __device__ __forceinline__ void unpack(const Raw &r, float (&v)[8]) {
    v[0] = r.a.x; v[1] = r.a.y; v[2] = r.a.z; v[3] = r.a.w;
    v[4] = r.b.x; v[5] = r.b.y; v[6] = r.b.z; v[7] = r.b.w;
  }
  static __device__ __forceinline__ void st(float *p, const float (&v)[8]) {
    ((float4 *)p)[0] = make_float4(v[0], v[1], v[2], v[3]);
    ((float4 *)p)[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
};
template <> struct Bw8<__nv_bfloat16> {
  using Raw = uint4;
  static __device__ __forceinline__ Raw ld(const __nv_bfloat16 *p) { return *(const uint4 *)p; }
  static __device__ __forceinline__ void unpack(const Raw &r, float (&v)[8]) {
    const uint32_t u[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(*(const __nv_bfloat162 *)&u[i]);
      v[2 * i] = f.x;
      v[2 * i + 1] = f.y;
    }
  }
  static __device__ __forceinline__ void st(__nv_bfloat16 *p, const float (&v)[8]) {
    uint32_t u[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_bfloat162 b = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
      u[i] = *(const uint32_t *)&b;
    }
    *(uint4 *)p = make_uint4(u[0], u[1], u[2], u[3]);
  }
};

// A block of 8 warps takes tpb tokens (tpb in {1, 2, 4, 8}), 8 / tpb warps per token; a warp takes
// the token's 256-column slices w, w + 8 / tpb, ... with eight columns per lane, and issues the
// loads of all k rows of a slice before it uses them. Each dot product is summed per lane over
// its columns, over the lanes in a fixed tree, then over the token's warps in order.
template <typename Ty>
__global__ void __launch_bounds__(256, sizeof(Ty) == 2 ? 3 : 2) combine_backward_kernel(
    const float *__restrict__ dy, const Ty *__restrict__ y_perm,
    const int32_t *__restrict__ slot_pos, const float *__restrict__ w, Ty *__restrict__ dy_perm,
    float *__restrict__ d_w, int T, int k, int d, int tpb) {
  __shared__ float part[8][8];  // [warp][slot]
  griddep_wait();
  griddep_launch();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wpt = 8 / tpb;
  const int tl = warp / wpt;
  const int t = blockIdx.x * tpb + tl;
  float dot[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) dot[j] = 0.0f;
  if (t < T) {
    int pos[8];
    float wj[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      pos[j] = j < k ? slot_pos[(size_t)t * k + j] : -1;
      wj[j] = j < k ? w[(size_t)t * k + j] : 0.0f;
    }
    for (int c = ((warp - tl * wpt) * 32 + lane) * 8; c < d; c += wpt * 256) {
      typename Bw8<Ty>::Raw r[8];
      const Bw8<float>::Raw gr = Bw8<float>::ld(dy + (size_t)t * d + c);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        if (pos[j] >= 0) r[j] = Bw8<Ty>::ld(y_perm + (size_t)pos[j] * d + c);
      float g[8];
      Bw8<float>::unpack(gr, g);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (pos[j] < 0) continue;
        float v[8], o[8];
        Bw8<Ty>::unpack(r[j], v);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          dot[j] = fmaf(g[i], v[i], dot[j]);
          o[i] = wj[j] * g[i];
        }
        Bw8<Ty>::st(dy_perm + (size_t)pos[j] * d + c, o);
      }
    }
  }
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (j >= k) break;
    const float s = warp_sum_f(dot[j]);
    if (lane == 0) part[warp][j] = s;
  }
  __syncthreads();
  if ((int)threadIdx.x < tpb * k) {
    const int tt = threadIdx.x / k, j = threadIdx.x - tt * k;
    const int t2 = blockIdx.x * tpb + tt;
    if (t2 < T) {
      float s = 0.0f;
      for (int q = 0; q < wpt; ++q) s += part[tt * wpt + q][j];
      d_w[(size_t)t2 * k + j] = slot_pos[(size_t)t2 * k + j] >= 0 ? s : 0.0f;
    }
  }
}

struct RouteBwdArgs {
  const void *x, *w_router;
  const float *off;          // [E] or null
  const int32_t *idx;        // [T, k]
  const int32_t *count;      // [E] selections before capacity
  const float *d_w;          // [T, k]
  float *d_logits;           // [T, E]
  int T, d, E, k, sigmoid, norm;
  float alpha, dL;
};

// Logit tiling of route_backward: a block of 8 warps takes RB_TM tokens; lane = tg + 4 eg holds
// tokens 4 tg .. 4 tg + 3 and experts 3 eg .. 3 eg + 2 of a round of 24 experts, warp w the
// columns [w d / 8, (w + 1) d / 8) in chunks of eight. The warps' partial sums are added in warp
// order.
constexpr int RB_TM = 16;
constexpr int RB_ROUND = 24;

template <typename Tin> struct Ld8;  // eight consecutive inputs as fp32 (zeros when !ok)
template <> struct Ld8<float> {
  static __device__ __forceinline__ void ld(const float *p, bool ok, float (&v)[8]) {
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
    if (ok) { a = __ldg((const float4 *)p); b = __ldg((const float4 *)p + 1); }
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
};
template <> struct Ld8<__nv_bfloat16> {
  static __device__ __forceinline__ void ld(const __nv_bfloat16 *p, bool ok, float (&v)[8]) {
    const uint4 r = ok ? __ldg((const uint4 *)p) : make_uint4(0u, 0u, 0u, 0u);
    Bw8<__nv_bfloat16>::unpack(r, v);
  }
};

// Shared memory of route_backward_kernel (floats): the warps' partial sums of a round, the
// block's logits (then probabilities) [RB_TM][E] and one dp row [E] per warp.
__host__ __device__ constexpr size_t route_bwd_smem_floats(int E) {
  return (size_t)8 * RB_TM * RB_ROUND + (size_t)RB_TM * E + (size_t)8 * E;
}

// Everything after the logits for token t, by one warp: probabilities, dp from d_topk_w, the
// loss term and d_logits. pr holds the token's E logits (replaced by its probabilities).
__device__ __forceinline__ void route_bwd_token(const RouteBwdArgs &a, int t, float *pr,
                                                float *dp, int lane) {
  const int E = a.E, k = a.k;
  float m = -INFINITY, ssum = 0.0f;
  if (!a.sigmoid) {
    for (int e = lane; e < E; e += 32) m = fmaxf(m, pr[e]);
    m = warp_max_f(m);
    for (int e = lane; e < E; e += 32) ssum += expf(pr[e] - m);
  } else {
    for (int e = lane; e < E; e += 32) ssum += 1.0f / (1.0f + expf(-pr[e]));
  }
  ssum = warp_sum_f(ssum);
  __syncwarp();
  for (int e = lane; e < E; e += 32) {
    pr[e] = !a.sigmoid ? expf(pr[e] - m) / ssum : 1.0f / (1.0f + expf(-pr[e]));
    dp[e] = 0.0f;
  }
  __syncwarp();
  if (lane == 0) {  // the combine weights' gradient onto the selected probabilities
    const int *ir = a.idx + (size_t)t * k;
    const float *gw = a.d_w + (size_t)t * k;
    bool ok = true;
    for (int j = 0; j < k; ++j) ok = ok && ir[j] >= 0 && ir[j] < E;
    if (!ok) {
      set_device_error(MOE_ERR_DEVICE_CHECK, INFO_BAD_EXPERT_INDEX);
    } else if (a.norm) {
      float S = 0.0f;
      for (int j = 0; j < k; ++j) S += pr[ir[j]];
      float inner = 0.0f;
      for (int j = 0; j < k; ++j) inner = fmaf(gw[j], pr[ir[j]] / S, inner);
      for (int j = 0; j < k; ++j) dp[ir[j]] += (gw[j] - inner) / S;
    } else {
      for (int j = 0; j < k; ++j) dp[ir[j]] += gw[j];
    }
  }
  __syncwarp();
  // loss term: dq_e = dL alpha E count_e / (T k T)
  const float cq = a.dL * a.alpha * (float)E / ((float)a.T * (float)k * (float)a.T);
  float *dl = a.d_logits + (size_t)t * E;
  if (!a.sigmoid) {
    float dot = 0.0f;
    for (int e = lane; e < E; e += 32) dot = fmaf(dp[e] + cq * (float)a.count[e], pr[e], dot);
    dot = warp_sum_f(dot);
    for (int e = lane; e < E; e += 32) dl[e] = pr[e] * (dp[e] + cq * (float)a.count[e] - dot);
  } else {
    float qd = 0.0f;  // sum_j dq_j q_j
    for (int e = lane; e < E; e += 32) qd = fmaf(cq * (float)a.count[e], pr[e] / ssum, qd);
    qd = warp_sum_f(qd);
    for (int e = lane; e < E; e += 32) {
      const float ds = dp[e] + (cq * (float)a.count[e] - qd) / ssum;
      dl[e] = ds * pr[e] * (1.0f - pr[e]);
    }
  }
  __syncwarp();
}

template <typename Tin>
__global__ void __launch_bounds__(256) route_backward_kernel(RouteBwdArgs a) {
  extern __shared__ float rb_smem[];
  griddep_wait();
  griddep_launch();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tg = lane & 3, eg = lane >> 2;
  const int E = a.E, d = a.d;
  const int t0 = blockIdx.x * RB_TM;
  float *part = rb_smem;                          // [8][RB_TM][RB_ROUND]
  float *lg = part + 8 * RB_TM * RB_ROUND;        // [RB_TM][E]
  float *dpw = lg + (size_t)RB_TM * E;            // [8][E]
  const int cs = d / 8;                           // columns per warp (a multiple of 8)
  const int c0 = warp * cs;
  const Tin *xb = (const Tin *)a.x, *wb = (const Tin *)a.w_router;
  bool tok_ok[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) tok_ok[i] = t0 + 4 * tg + i < a.T;
  for (int e0 = 0; e0 < E; e0 += RB_ROUND) {
    float acc[4][3];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 3; ++j) acc[i][j] = 0.0f;
    bool ex_ok[3];
#pragma unroll
    for (int j = 0; j < 3; ++j) ex_ok[j] = e0 + 3 * eg + j < E;
    for (int c = c0; c < c0 + cs; c += 8) {
      float xv[4][8], wv[3][8];
#pragma unroll
      for (int i = 0; i < 4; ++i)
        Ld8<Tin>::ld(xb + (size_t)(t0 + 4 * tg + i) * d + c, tok_ok[i], xv[i]);
#pragma unroll
      for (int j = 0; j < 3; ++j)
        Ld8<Tin>::ld(wb + (size_t)(e0 + 3 * eg + j) * d + c, ex_ok[j], wv[j]);
#pragma unroll
      for (int q = 0; q < 8; ++q)
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 3; ++j) acc[i][j] = fmaf(xv[i][q], wv[j][q], acc[i][j]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 3; ++j)
        part[(warp * RB_TM + 4 * tg + i) * RB_ROUND + 3 * eg + j] = acc[i][j];
    __syncthreads();
    for (int o = threadIdx.x; o < RB_TM * RB_ROUND; o += 256) {
      const int tt = o / RB_ROUND, e = e0 + (o - tt * RB_ROUND);
      if (e < E) {
        float s = 0.0f;
#pragma unroll
        for (int w = 0; w < 8; ++w) s += part[w * RB_TM * RB_ROUND + o];
        lg[(size_t)tt * E + e] = a.off ? s + a.off[e] : s;
      }
    }
    __syncthreads();
  }
  // each warp finishes two of the block's tokens
  for (int tt = warp; tt < RB_TM; tt += 8) {
    const int t = t0 + tt;
    if (t < a.T) route_bwd_token(a, t, lg + (size_t)tt * E, dpw + (size_t)warp * E, lane);
  }
}

template <typename Tin> __device__ __forceinline__ float bw_elem(const Tin *p, size_t i);
template <> __device__ __forceinline__ float bw_elem<float>(const float *p, size_t i) { return p[i]; }
template <> __device__ __forceinline__ float bw_elem<__nv_bfloat16>(const __nv_bfloat16 *p, size_t i) {
  return __bfloat162float(p[i]);
}

// Two consecutive inputs as fp32.
template <typename Tin> __device__ __forceinline__ float2 ld2(const Tin *p);
template <> __device__ __forceinline__ float2 ld2<float>(const float *p) {
  return __ldg((const float2 *)p);
}
template <> __device__ __forceinline__ float2 ld2<__nv_bfloat16>(const __nv_bfloat16 *p) {
  const uint32_t u = __ldg((const unsigned int *)p);
  return __bfloat1622float2(*(const __nv_bfloat162 *)&u);
}

// d_w_router = d_logits^T x, split over the tokens: block (512 columns, 8 experts, split s) sums
// tokens [s T / S, (s + 1) T / S) in order into part[s][e][c], a thread two columns of eight
// experts; the split's d_logits rows pass through shared memory 64 tokens at a time, and each
// thread loads the x values of eight tokens before it uses them. router_wgrad_sum adds the S
// partial sums in split order (S = 1 writes the result directly).
template <typename Tin>
__global__ void __launch_bounds__(256) router_wgrad_kernel(const float *__restrict__ dl,
                                                           const Tin *__restrict__ x, int T, int d,
                                                           int E, int S, float *__restrict__ part) {
  __shared__ __align__(16) float g_s[64][8];
  griddep_wait();
  griddep_launch();
  const int c = 2 * (blockIdx.x * 256 + threadIdx.x), e0 = blockIdx.y * 8, s = blockIdx.z;
  const int t0 = (int)((long long)T * s / S), t1 = (int)((long long)T * (s + 1) / S);
  float acc[8][2];
#pragma unroll
  for (int i = 0; i < 8; ++i) acc[i][0] = acc[i][1] = 0.0f;
  for (int tb = t0; tb < t1; tb += 64) {
    const int n = min(64, t1 - tb);
    __syncthreads();
    for (int o = threadIdx.x; o < 64 * 8; o += 256) {
      const int tt = o >> 3, i = o & 7;
      g_s[tt][i] = (tt < n && e0 + i < E) ? dl[(size_t)(tb + tt) * E + e0 + i] : 0.0f;
    }
    __syncthreads();
    if (c < d) {
      for (int tt = 0; tt < n; tt += 8) {
        float2 xv[8];
#pragma unroll
        for (int u = 0; u < 8; ++u)
          xv[u] = tt + u < n ? ld2(x + (size_t)(tb + tt + u) * d + c) : make_float2(0.0f, 0.0f);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float4 ga = *(const float4 *)&g_s[tt + u][0];
          const float4 gb = *(const float4 *)&g_s[tt + u][4];
          const float g[8] = {ga.x, ga.y, ga.z, ga.w, gb.x, gb.y, gb.z, gb.w};
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            acc[i][0] = fmaf(g[i], xv[u].x, acc[i][0]);
            acc[i][1] = fmaf(g[i], xv[u].y, acc[i][1]);
          }
        }
      }
    }
  }
  if (c >= d) return;
#pragma unroll
  for (int i = 0; i < 8; ++i)
    if (e0 + i < E)
      *(float2 *)(part + ((size_t)s * E + e0 + i) * d + c) = make_float2(acc[i][0], acc[i][1]);
}

__global__ void __launch_bounds__(256) router_wgrad_sum_kernel(const float *__restrict__ part,
                                                               int S, int E, int d,
                                                               float *__restrict__ dwr) {
  griddep_wait();
  griddep_launch();
  const size_t i = (size_t)blockIdx.x * 256 + threadIdx.x, n = (size_t)E * d;
  if (i >= n) return;
  float acc = part[i];
  int s = 1;
  for (; s + 8 <= S; s += 8) {  // eight loads in flight, added in split order
    float v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = part[(size_t)(s + u) * n + i];
#pragma unroll
    for (int u = 0; u < 8; ++u) acc += v[u];
  }
  for (; s < S; ++s) acc += part[(size_t)s * n + i];
  dwr[i] = acc;
}

// dx[t, c..c+3] = sum over e (in order) of d_logits[t, e] W_r[e, c..c+3]: a block takes 16 tokens
// at a time (blocks stride over the token blocks) and 1024 columns, a thread four columns of the
// 16 tokens; the tokens' d_logits pass through shared memory (expert-major) 64 experts at a time.
template <typename Tin>
__global__ void __launch_bounds__(256) router_dgrad_kernel(const float *__restrict__ dl,
                                                           const Tin *__restrict__ wr, int T, int d,
                                                           int E, float *__restrict__ dx) {
  __shared__ __align__(16) float g_s[64][16];
  griddep_wait();
  griddep_launch();
  const int c = 4 * (blockIdx.x * 256 + threadIdx.x);
  for (int t0 = blockIdx.y * 16; t0 < T; t0 += gridDim.y * 16) {
  float4 acc[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) acc[i] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
  for (int eb = 0; eb < E; eb += 64) {
    const int n = min(64, E - eb);
    __syncthreads();
    for (int o = threadIdx.x; o < 64 * 16; o += 256) {
      const int e = o >> 4, tt = o & 15;
      g_s[e][tt] = (e < n && t0 + tt < T) ? dl[(size_t)(t0 + tt) * E + eb + e] : 0.0f;
    }
    __syncthreads();
    if (c < d) {
#pragma unroll 4
      for (int e = 0; e < n; ++e) {
        const float4 v = Bw4<Tin>::ld(wr + (size_t)(eb + e) * d + c);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float4 g = *(const float4 *)&g_s[e][4 * q];
          const float gg[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            float4 &r = acc[4 * q + u];
            r.x = fmaf(gg[u], v.x, r.x);
            r.y = fmaf(gg[u], v.y, r.y);
            r.z = fmaf(gg[u], v.z, r.z);
            r.w = fmaf(gg[u], v.w, r.w);
          }
        }
      }
    }
  }
  if (c < d) {
#pragma unroll
    for (int i = 0; i < 16; ++i)
      if (t0 + i < T) *(float4 *)(dx + (size_t)(t0 + i) * d + c) = acc[i];
  }
  }
}


// ------------------------------------------------------------------ expert steps of the backward
// The weight gradients are products over a group's rows (dW_d[e] = dY_e^T h_e, dW_g[e] =
// dg_e^T X_e, dW_u[e] = du_e^T X_e). For SwiGLU layers the tensor cores read both operands
// MN-major from the row-major activations, in 64-row K-blocks aligned to each expert's last row
// (kstart below); h and [dg | du] are written with zero rows in front of each expert's rows, so
// the rows a block reads before the expert's first row contribute nothing. The low-rank layers'
// activations are still transposed into K-major copies, each expert's rows padded with zeros to a
// multiple of 64; the weights are transposed for the data gradients (dh = dY W_d,
// dX = [dg | du] [W_g; W_u]) the same way.

// koff[e] = sum over e' < e of the expert's row count rounded up to 64; koff[E] is the total.
// kstart[e] = offsets[e+1] - (koff[e+1] - koff[e]): the row of the grouped activations at which
// the expert's padded row range starts when it is aligned to the expert's last row (the rows
// before offsets[e] belong to earlier experts, or lie before row 0).
// korder: the experts by padded row count, largest first (ties: lower index first), the order in
// which the weight-gradient products list their groups (each group's K is its row count, so
// longest first balances the CTA pairs' round-robin share of the tiles).
// Also the group tables of the shared experts' T rows cut into nc chunks of ch rows (ch a
// multiple of 64): off_s[i] = min(i ch, T), koff_s[i] = the same rounded up to 64. One block;
// E <= 1024, nc <= 64.
__global__ void __launch_bounds__(1024) pad_offsets_kernel(const int32_t *__restrict__ offsets,
                                                           int E, int32_t *__restrict__ koff,
                                                           int32_t *__restrict__ korder,
                                                           int32_t *__restrict__ kstart,
                                                           int T, int nc, int ch,
                                                           int32_t *__restrict__ off_s,
                                                           int32_t *__restrict__ koff_s) {
  griddep_wait();
  griddep_launch();
  __shared__ int s[1024];
  __shared__ int sz[1024];
  __shared__ int tmp[1024 / 32 + 1];
  const int e = threadIdx.x;
  s[e] = e < E ? ((offsets[e + 1] - offsets[e] + 63) & ~63) : 0;
  sz[e] = s[e];
  __syncthreads();
  const int total = block_excl_scan_inplace(s, 1024, tmp);
  if (e < E) {
    koff[e] = s[e];
    kstart[e] = offsets[e + 1] - sz[e];
    const int v = sz[e];
    int r = 0;
    for (int h = 0; h < E; ++h) r += (sz[h] > v || (sz[h] == v && h < e)) ? 1 : 0;
    korder[r] = e;
  }
  if (e == 0) koff[E] = total;
  if (e <= nc) {
    const int v = min(e * ch, T);
    off_s[e] = v;
    koff_s[e] = (v + 63) & ~63;
  }
}

// Tiled bf16 transpose through shared memory: a CTA moves 64 input rows x 128 input columns
// (16 KB) with 16-byte loads and stores.
//   grouped (in_offsets != null): group g's rows offsets[g] .. offsets[g+1] of the sources
//     [rows, C] (row stride ldi) go to nseg segments of columns of out [C, ldo]: segment s
//     spans columns nseg koff[g] + s P .. + P, P = koff[g+1] - koff[g] (the group's row count
//     rounded up to 64), and holds the rows of source s, zeros past the group's rows
//     (blockIdx.y runs over 64-column blocks of out, blockIdx.z = 0);
//   dense: batch b = blockIdx.z, in0 + b * ibs is [R, C] (row stride ldi) and goes to
//     out + b * obs + col0 as [C, R] with row stride ldo; blockIdx.y runs over 64-row blocks
//     (R a multiple of 8).
// C and ldi are multiples of 64, ldo of 8; pointers 16-byte aligned.
constexpr int TR_COLS = 128;
__global__ void __launch_bounds__(256) transpose_bf16_kernel(
    const __nv_bfloat16 *__restrict__ in0, const __nv_bfloat16 *__restrict__ in1,
    const __nv_bfloat16 *__restrict__ in2, int nseg, int C, int ldi,
    const int32_t *__restrict__ in_offsets, const int32_t *__restrict__ koff, int G, int R,
    size_t ibs, __nv_bfloat16 *__restrict__ out, int ldo, size_t obs, int col0) {
  griddep_wait();
  griddep_launch();
  // [64][128] with the 16-byte chunk index of row r XORed with (r / 8) % 8: the store phase
  // reads rows 8 apart, which then fall in different banks
  __shared__ __align__(16) __nv_bfloat16 tile[64][TR_COLS];
  const int c0 = blockIdx.x * TR_COLS;
  int r_in0, n_rows, o_col0;  // first input row, valid rows of the block, first output column
  const __nv_bfloat16 *src = in0;
  __nv_bfloat16 *dst = out;
  if (in_offsets) {
    const int p0 = blockIdx.y * 64;  // column block of out
    if (p0 >= nseg * koff[G]) return;
    int lo = 0, hi = G - 1;          // group with nseg koff[g] <= p0 < nseg koff[g+1]
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (nseg * koff[mid] <= p0) lo = mid;
      else hi = mid - 1;
    }
    const int P = koff[lo + 1] - koff[lo];
    const int local = p0 - nseg * koff[lo];
    const int seg = local / P, lr = local - seg * P;
    src = seg == 0 ? in0 : (seg == 1 ? in1 : in2);
    r_in0 = in_offsets[lo] + lr;
    n_rows = max(0, min(64, in_offsets[lo + 1] - in_offsets[lo] - lr));
    o_col0 = p0;
  } else {
    src += (size_t)blockIdx.z * ibs;
    dst += (size_t)blockIdx.z * obs + col0;
    r_in0 = blockIdx.y * 64;
    n_rows = max(0, min(64, R - r_in0));
    o_col0 = r_in0;
  }
  const int ncols = min(TR_COLS, C - c0);  // 64 or 128
  // load: 64 rows x 16 vectors of 8 columns, zeros past the valid rows
  for (int q = threadIdx.x; q < 64 * (TR_COLS / 8); q += 256) {
    const int r = q >> 4, v = q & 15;
    uint4 val = make_uint4(0u, 0u, 0u, 0u);
    if (r < n_rows && v * 8 < ncols)
      val = *(const uint4 *)(src + (size_t)(r_in0 + r) * ldi + c0 + v * 8);
    *(uint4 *)&tile[r][(v ^ ((r >> 3) & 7)) * 8] = val;
  }
  __syncthreads();
  // store: output row c (an input column) takes 8 vectors of 8 input rows
  const int n_out = in_offsets ? 64 : n_rows;  // grouped: the padding columns are written too
  for (int q = threadIdx.x; q < TR_COLS * 8; q += 256) {
    const int c = q >> 3, v = q & 7;
    if (c >= ncols || v * 8 >= n_out) continue;
    uint32_t w[4];
    const int cx = (((c >> 3) ^ v) << 3) + (c & 7);  // rows v*8 .. v*8+7 share (r / 8) % 8 = v
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const __nv_bfloat16 a = tile[v * 8 + 2 * i][cx], b = tile[v * 8 + 2 * i + 1][cx];
      w[i] = (uint32_t)__bfloat16_as_ushort(a) | ((uint32_t)__bfloat16_as_ushort(b) << 16);
    }
    *(uint4 *)(dst + (size_t)(c0 + c) * ldo + o_col0 + v * 8) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// out[i] = sum over c < nc of part[c][i], in chunk order (partial weight gradients of chunks).
__global__ void __launch_bounds__(256) sum_chunks_kernel(const float *__restrict__ part, int nc,
                                                         size_t n, float *__restrict__ out) {
  griddep_wait();
  griddep_launch();
  for (size_t i = ((size_t)blockIdx.x * 256 + threadIdx.x) * 4; i < n; i += (size_t)gridDim.x * 1024) {
    float4 a = *(const float4 *)(part + i);
    for (int c = 1; c < nc; ++c) {
      const float4 b = *(const float4 *)(part + (size_t)c * n + i);
      a.x += b.x;
      a.y += b.y;
      a.z += b.z;
      a.w += b.w;
    }
    *(float4 *)(out + i) = a;
  }
}

// Rows of in [rows, d] (fp32) as two bf16 terms: out[r] = [hi (d) | lo (d)], hi = bf16(v),
// lo = bf16(v - hi); d a multiple of 4.
__global__ void __launch_bounds__(256) split_bf16_kernel(const float *__restrict__ in, int d,
                                                         size_t rows, __nv_bfloat16 *__restrict__ out) {
  griddep_wait();
  griddep_launch();
  const size_t n = rows * (size_t)d;
  for (size_t i = ((size_t)blockIdx.x * 256 + threadIdx.x) * 4; i < n; i += (size_t)gridDim.x * 1024) {
    const float4 v = *(const float4 *)(in + i);
    const size_t r = i / d, c = i - r * d;
    const __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
    const float2 af = __bfloat1622float2(a), bf = __bfloat1622float2(b);
    const __nv_bfloat162 al = __floats2bfloat162_rn(v.x - af.x, v.y - af.y);
    const __nv_bfloat162 bl = __floats2bfloat162_rn(v.z - bf.x, v.w - bf.y);
    uint2 hi, lo;
    hi.x = *(const uint32_t *)&a;
    hi.y = *(const uint32_t *)&b;
    lo.x = *(const uint32_t *)&al;
    lo.y = *(const uint32_t *)&bl;
    *(uint2 *)(out + r * 2 * d + c) = hi;
    *(uint2 *)(out + r * 2 * d + d + c) = lo;
  }
}

// Low-rank experts: for the 64-row block b of the padded grouped rows (koff, as the transposes
// use), with z = X V^T and dzs = dY U (fp32 [rows, r]) and the expert's s:
//   dz = dzs s and zs = z s as bf16 hi + lo terms ([rows, 2r]: hi | lo);
//   ds_part[b][j] = sum over the block's rows of dzs[., j] z[., j] (4 row groups in fixed order).
__global__ void __launch_bounds__(256) lowrank_elem_kernel(
    const float *__restrict__ z, const float *__restrict__ dzs, const float *__restrict__ s,
    const int32_t *__restrict__ offsets, const int32_t *__restrict__ koff, int E, int r,
    __nv_bfloat16 *__restrict__ dz2, __nv_bfloat16 *__restrict__ zs2,
    float *__restrict__ ds_part) {
  griddep_wait();
  griddep_launch();
  __shared__ float part[4][64];
  const int p0 = blockIdx.x * 64;
  if (p0 >= koff[E]) return;
  int lo = 0, hi = E - 1;  // expert with koff[e] <= p0 < koff[e+1]
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (koff[mid] <= p0) lo = mid;
    else hi = mid - 1;
  }
  const int local = p0 - koff[lo];
  const int row0 = offsets[lo] + local, nrow = max(0, min(64, offsets[lo + 1] - offsets[lo] - local));
  const int cl = threadIdx.x & 63, rg = threadIdx.x >> 6;
  for (int j0 = 0; j0 < r; j0 += 64) {
    const int j = j0 + cl;
    const float sj = s[(size_t)lo * r + j];
    float acc = 0.0f;
    for (int i = rg; i < nrow; i += 4) {
      const size_t row = (size_t)(row0 + i);
      const float zv = z[row * r + j], dv = dzs[row * r + j];
      acc = fmaf(dv, zv, acc);
      const float a = dv * sj, b = zv * sj;
      const __nv_bfloat16 ah = __float2bfloat16_rn(a), bh = __float2bfloat16_rn(b);
      dz2[row * 2 * r + j] = ah;
      dz2[row * 2 * r + r + j] = __float2bfloat16_rn(a - __bfloat162float(ah));
      zs2[row * 2 * r + j] = bh;
      zs2[row * 2 * r + r + j] = __float2bfloat16_rn(b - __bfloat162float(bh));
    }
    part[rg][cl] = acc;
    __syncthreads();
    if (rg == 0)
      ds_part[(size_t)blockIdx.x * r + j] = ((part[0][cl] + part[1][cl]) + part[2][cl]) + part[3][cl];
    __syncthreads();
  }
}

// ds[e][j] = sum of the expert's block partials in block order (0 for an expert with no rows).
__global__ void __launch_bounds__(256) lowrank_ds_kernel(const float *__restrict__ ds_part,
                                                         const int32_t *__restrict__ koff, int r,
                                                         float *__restrict__ ds) {
  griddep_wait();
  griddep_launch();
  const int e = blockIdx.x;
  const int b0 = koff[e] / 64, b1 = koff[e + 1] / 64;
  for (int j = threadIdx.x; j < r; j += blockDim.x) {
    float acc = 0.0f;
    for (int b = b0; b < b1; ++b) acc += ds_part[(size_t)b * r + j];
    ds[(size_t)e * r + j] = acc;
  }
}

// Zero the gradient slices of experts that received no rows (their weight-gradient products
// have no tiles): up to three arrays with `per` floats per expert each.
__global__ void __launch_bounds__(256) zero_empty_experts_kernel(
    const int32_t *__restrict__ offsets, float *__restrict__ a, size_t pa, float *__restrict__ b,
    size_t pb, float *__restrict__ c, size_t pc) {
  griddep_wait();
  griddep_launch();
  const int e = blockIdx.x;
  if (offsets[e + 1] != offsets[e]) return;
  for (size_t i = (size_t)blockIdx.y * 256 + threadIdx.x; i < pa; i += (size_t)gridDim.y * 256)
    a[(size_t)e * pa + i] = 0.0f;
  if (b)
    for (size_t i = (size_t)blockIdx.y * 256 + threadIdx.x; i < pb; i += (size_t)gridDim.y * 256)
      b[(size_t)e * pb + i] = 0.0f;
  if (c)
    for (size_t i = (size_t)blockIdx.y * 256 + threadIdx.x; i < pc; i += (size_t)gridDim.y * 256)
      c[(size_t)e * pc + i] = 0.0f;
}

}  // namespace moe

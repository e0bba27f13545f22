/*
 * moe.h - C ABI of the B200 fine-grained mixture-of-experts FFN layer (forward and backward).
 *
 * The layer is the DeepSeek-style fine-grained MoE FFN that the source pages describe:
 *   - Vertex AGI research page / quartz-micro-preview-base model card, "Architecture":
 *     24 narrow routed experts (FFN 640) at hidden 1,024, top-6, 2 always-active shared experts,
 *     a load-balancing loss with weight 0.01;
 *   - Moonfrost, expert card: 32 routed experts + 1 shared, top-3, experts held as three stacked
 *     (E, hidden, ffn) tensors with routing under a per-expert capacity instead of a per-expert loop;
 *   - Sutra-1.3B, "48 + 1 experts": top-4 by sigmoid score with balancing through a per-expert bias;
 *   - dormouse, "dropless MoE" and "TSCT low-rank experts": 1,024 experts U*diag(s)*V^T of
 *     rank 64, top-2, dropless.
 *
 * Conventions for every call:
 *   - Ownership: the caller allocates every buffer. The library allocates no device or host
 *     memory; scratch comes from a caller-provided workspace of moe_workspace_size() bytes.
 *   - Pointers are device pointers unless stated otherwise, 16-byte aligned, row-major and
 *     densely packed. "dtype" below means fp32 for MOE_DTYPE_F32 and bf16 for MOE_DTYPE_BF16.
 *   - Asynchrony: calls only enqueue work on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and return. Argument errors are detected on the host and returned at once,
 *     with nothing enqueued. Faults detected on the device (a bounded wait that ran out, an
 *     internal consistency check) set a device error word that moe_get_device_error() reads.
 *     No call aborts, exits or traps.
 *   - Determinism: every output is bitwise reproducible run to run (no floating-point atomics).
 *   - Shapes: d, ffn, ffn_shared and rank must be multiples of 64; 1 <= top_k <= min(E, 8);
 *     1 <= E <= 1024; n_shared <= 8; rank <= 256; the router's per-CTA tile (16 token rows of
 *     d elements, the staging ring of the router rows and 16 x E logits) must fit in 227 KB of
 *     shared memory, so d up to about 6,000 (bf16) or 2,600 (fp32) for small E, and at
 *     d = 1536 with sigmoid keys E up to 991. T may be 0.
 *     Other values return MOE_ERR_UNSUPPORTED.
 *   - Inputs must be finite. Router logits of +-inf or NaN make the routing unspecified.
 */
#ifndef MOE_H
#define MOE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,   /* null pointer, negative size, misaligned pointer */
  MOE_ERR_UNSUPPORTED = 2,   /* a shape or option outside the supported set */
  MOE_ERR_WORKSPACE = 3,     /* ws_bytes smaller than moe_workspace_size() */
  MOE_ERR_CUDA = 4,          /* a CUDA runtime call failed (launch error, no device) */
  MOE_ERR_TIMEOUT = 5,       /* device: a bounded wait ran out; the kernel returned early */
  MOE_ERR_DEVICE_CHECK = 6   /* device: an internal check failed (see moe_get_device_error) */
} moe_status_t;

typedef enum { MOE_SCORE_SOFTMAX = 0, MOE_SCORE_SIGMOID = 1 } moe_score_t;
typedef enum { MOE_EXPERT_SWIGLU = 0, MOE_EXPERT_LOWRANK = 1 } moe_expert_t;
typedef enum { MOE_DTYPE_F32 = 0, MOE_DTYPE_BF16 = 1 } moe_dtype_t;
/* Storage of the routed experts' weights. MOE_STORAGE_FP8_E4M3 is the fp8 rung of the storage
 * ladder of the low-rank experts (dormouse, "TSCT low-rank experts": the U*diag(s)*V^T
 * factorisation carries a storage ladder fp8 -> NVFP4 -> ternary): V and U as E4M3 rows with
 * one fp32 scale per row (see moe_quantize_fp8), computed on the fp8 tensor cores. bf16 low-rank
 * layers only. */
typedef enum { MOE_STORAGE_DTYPE = 0, MOE_STORAGE_FP8_E4M3 = 1 } moe_storage_t;

/* Problem statement of one layer call (the arguments the pages' architecture tables give:
 * hidden size, routed experts, top-k, shared experts, expert FFN width, scoring, capacity). */
typedef struct {
  int32_t T;            /* tokens in the call (batch x sequence, flattened) */
  int32_t d;            /* hidden size */
  int32_t E;            /* routed experts */
  int32_t top_k;        /* experts selected per token */
  int32_t n_shared;     /* always-active shared experts (SwiGLU), 0 for none */
  int32_t ffn;          /* routed SwiGLU expert width (ignored for low-rank experts) */
  int32_t ffn_shared;   /* shared expert width */
  int32_t rank;         /* low-rank expert rank r (ignored for SwiGLU experts) */
  int32_t score;        /* moe_score_t */
  int32_t expert;       /* moe_expert_t */
  int32_t dtype;        /* moe_dtype_t: activations and weights */
  int32_t norm_topk;    /* 1: divide the k selected weights by their sum */
  float capacity_factor;/* <= 0: dropless; else C = ceil(cf*T*top_k/E), exact on this fp32 */
  float aux_alpha;      /* load-balancing loss weight (0.01 on the Quartz pages) */
  int32_t expert_storage; /* moe_storage_t of the routed experts' weights (0: dtype) */
} moe_config_t;

/* Weights, all device pointers in dtype unless noted; [a,b,c] = row-major shape. */
typedef struct {
  const void *w_router;      /* [E, d] */
  const float *logit_offset; /* [E] fp32 added to the logit before rounding, or NULL */
  const float *select_bias;  /* [E] fp32 selection-only bias (sigmoid scoring), or NULL */
  const void *w_gate;        /* SwiGLU: [E, ffn, d] */
  const void *w_up;          /* SwiGLU: [E, ffn, d] */
  const void *w_down;        /* SwiGLU: [E, d, ffn] */
  const void *lr_V;          /* low-rank: [E, rank, d]  (V^T of each expert) */
  const void *lr_U;          /* low-rank: [E, d, rank] */
  const float *lr_s;         /* low-rank: [E, rank] fp32 */
  const void *ws_gate;       /* shared: [n_shared, ffn_shared, d] */
  const void *ws_up;         /* shared: [n_shared, ffn_shared, d] */
  const void *ws_down;       /* shared: [n_shared, d, ffn_shared] */
  /* MOE_STORAGE_FP8_E4M3 only (then lr_V and lr_U are not read), as moe_quantize_fp8 writes
   * them from V and U: */
  const uint8_t *lr_V8;      /* [E, rank, d] E4M3 codes */
  const float *lr_V_scale;   /* [E, rank] fp32 row scales */
  const uint8_t *lr_U8;      /* [E, d, rank] E4M3 codes */
  const float *lr_U_scale;   /* [E, d] fp32 row scales */
} moe_weights_t;

/* Bytes of workspace that every call below needs for `cfg` (the largest, moe_layer_forward).
 * Returns 0 for an invalid or unsupported configuration. */
size_t moe_workspace_size(const moe_config_t *cfg);

/* Per-expert capacity C of this configuration, or -1 for dropless, or -2 if cfg is invalid.
 * C = ceil(capacity_factor * T * top_k / E) evaluated exactly on the fp32 capacity_factor
 * (Moonfrost expert card: routing under a per-expert capacity; the bound is taken over the call's T). */
int32_t moe_capacity(const moe_config_t *cfg);

/* Router: logits, scoring, top-k, combine weights and the per-expert statistics.
 * (Quartz architecture table, row "Router": 6 of 24 experts; Moonfrost expert card: top-3
 * routing; Sutra-1.3B, "48 + 1 experts": top-4 by sigmoid score, balanced by a per-expert bias.)
 *   l[t,e] = RN32(sum_i x[t,i]*w_router[e,i] + logit_offset[e])  - exact sum, rounded once
 *   key    = l (softmax) or RN32(sigmoid(l) + select_bias[e]) (sigmoid), exact, rounded once
 *   topk_idx[t,j]  [T, top_k] int32: experts by descending key, equal keys -> lower index
 *   topk_w[t,j]    [T, top_k] fp32: softmax over all E of l (or sigmoid(l)) of the selected
 *                  expert, divided by the sum over the selected k when norm_topk is set
 *   expert_count[e][E] int32: number of tokens that selected e (before capacity)
 *   prob_sum[e]    [E] fp32: sum over tokens of the token's probability of e (softmax; for
 *                  sigmoid scoring, sigmoids normalised over all E), fixed-order sums */
moe_status_t moe_route(const moe_config_t *cfg, const void *x /*[T,d]*/,
                       const moe_weights_t *w, int32_t *topk_idx, float *topk_w,
                       int32_t *expert_count, float *prob_sum,
                       void *ws, size_t ws_bytes, void *stream);

/* Token permutation grouped by expert (the stacked-expert layout of the Moonfrost card).
 * Per expert, routed (token, slot) pairs are ranked by ascending token; rank >= C is dropped.
 *   offsets  [E+1] int32: exclusive scan of kept counts; offsets[E] = N kept pairs
 *   slot_pos [T, top_k] int32: row of pair (t,j) in the grouped order, -1 if dropped
 *   src_token[T*top_k] int32: token of each grouped row (first N entries valid)
 *   x_perm   [T*top_k, d] dtype: x_perm[r] = x[src_token[r]] (first N rows valid); may be
 *            NULL to skip the copy. */
moe_status_t moe_permute(const moe_config_t *cfg, const void *x, const int32_t *topk_idx,
                         int32_t *offsets, int32_t *slot_pos, int32_t *src_token,
                         void *x_perm, void *ws, size_t ws_bytes, void *stream);

/* Grouped expert GEMMs on the grouped rows, and the shared experts on all tokens
 * (quartz-micro-preview-base card, "Architecture": routed SwiGLU experts of FFN width 640 and 2
 * shared experts that every token passes through; Moonfrost expert card: the experts held as
 * stacked (E, hidden, ffn) tensors; dormouse, "TSCT low-rank experts": experts U*diag(s)*V^T).
 *   SwiGLU expert e on row r (offsets[e] <= r < offsets[e+1]):
 *     y_perm[r] = W_down[e] (silu(W_gate[e] x_perm[r]) * (W_up[e] x_perm[r]))
 *   low-rank expert: y_perm[r] = U[e] (s[e] * (V[e] x_perm[r]))
 *   y_shared[t] = sum over shared experts of their SwiGLU output on x[t]
 * The SwiGLU hidden activations are rounded to dtype, since they are the next tensor-core
 * product's operand; a bf16 low-rank projection is kept as two bf16 terms (its value and its
 * rounding residual); accumulation is fp32.
 * y_perm: [T*top_k, d] (first offsets[E] rows written), each row rounded once from its fp32
 * accumulator: bf16 for bf16 SwiGLU layers, fp32 for fp32 layers and for low-rank layers. A
 * SwiGLU row enters y through a weighted sum of top_k rows plus the shared output, which
 * averages its rounding; a low-rank layer's y can be a sum of as few as two rows with no shared
 * output, where one bf16 rounding alone exceeds the error budget.
 * y_shared: [T, d] fp32 (the S shared outputs summed in fp32), may be NULL when n_shared = 0;
 * it enters y alone, so it stays fp32.
 * fp8 storage (expert_storage = MOE_STORAGE_FP8_E4M3): each x_perm row is quantised as
 * moe_quantize_fp8 does (its E4M3 codes xq, scale sx), then per expert e, on the fp8 tensor
 * cores with fp32 sums:
 *   z = (xq V8[e]^T) * sx * V_scale[e] * s[e]  (per column);  zq, sz = the quantised rows of z;
 *   y_perm[r] = (zq U8[e]^T) * sz * U_scale[e]  (fp32).
 * The shared experts keep the layer's dtype. */
moe_status_t moe_expert_forward(const moe_config_t *cfg, const void *x_perm,
                                const int32_t *offsets, const void *x,
                                const moe_weights_t *w, void *y_perm, void *y_shared,
                                void *ws, size_t ws_bytes, void *stream);

/* Weighted un-permute (Moonfrost expert card: a token's output is the shared expert plus its
 * top-k routed experts; Quartz architecture table: the 2 shared experts are always active):
 * y[t] = y_shared[t] + sum_j [slot_pos[t,j] >= 0] topk_w[t,j] *
 * y_perm[slot_pos[t,j]], summed in fp32 in slot order. y_perm as moe_expert_forward writes it
 * (bf16 for bf16 SwiGLU layers, else fp32); y_shared and y are fp32 [.., d]: a bf16 rounding of
 * y itself would cost up to 2^-8 * max|y| / rms(y), the whole 2e-2 error budget of the layer.
 * No atomics. y_shared may be NULL (no shared experts). */
moe_status_t moe_combine(const moe_config_t *cfg, const void *y_perm, const void *y_shared,
                         const int32_t *slot_pos, const float *topk_w, void *y, void *stream);

/* Backward pass. The pages train with this layer but do not write its backward out; it is the
 * derivative of the forward, of J = sum(dy * y) + dL * loss, with no gradient through the
 * selection (top-k, capacity drops, the loss's counts), none for the selection bias or the logit
 * offsets, and each logit's fp32 rounding taken with derivative 1. Three calls: this one, the
 * experts' (moe_expert_backward) and the router's (moe_route_backward).
 *
 * Backward of moe_combine (Moonfrost expert card: a token's output sums its shared and top-k
 * routed experts). For every kept pair (t, j), p = slot_pos[t, j] >= 0:
 *   dy_perm[p]     = topk_w[t, j] * dy[t]
 *   d_topk_w[t, j] = sum_c dy[t, c] * y_perm[p, c]      (0 for a dropped pair)
 * dy: [T, d] fp32, the upstream gradient of y (the shared experts' upstream gradient is dy
 * itself); y_perm, slot_pos, topk_w as the forward produced them; dy_perm: [offsets[E], d] in
 * y_perm's dtype (bf16 for bf16 SwiGLU layers, else fp32), rows of dropped pairs do not exist;
 * d_topk_w: [T, top_k] fp32. Sums over c in fp32, each reduced in a fixed order: bitwise
 * reproducible. All buffers are the caller's device memory, 16-byte aligned (NULL only when
 * T = 0). Asynchronous on `stream`; bad arguments return MOE_ERR_INVALID_ARG. */
moe_status_t moe_combine_backward(const moe_config_t *cfg, const float *dy, const void *y_perm,
                                  const int32_t *slot_pos, const float *topk_w, void *dy_perm,
                                  float *d_topk_w, void *stream);

/* Weight gradients of the experts: fp32 device buffers in the weights' own layouts. */
typedef struct {
  float *d_w_gate;   /* SwiGLU: [E, ffn, d] */
  float *d_w_up;     /* SwiGLU: [E, ffn, d] */
  float *d_w_down;   /* SwiGLU: [E, d, ffn] */
  float *d_lr_V;     /* low-rank: [E, rank, d] */
  float *d_lr_s;     /* low-rank: [E, rank] */
  float *d_lr_U;     /* low-rank: [E, d, rank] */
  float *d_ws_gate;  /* shared: [n_shared, ffn_shared, d] */
  float *d_ws_up;    /* shared: [n_shared, ffn_shared, d] */
  float *d_ws_down;  /* shared: [n_shared, d, ffn_shared] */
} moe_grads_t;

/* Bytes of workspace moe_expert_backward needs for `cfg` (0 for an invalid configuration). */
size_t moe_backward_workspace_size(const moe_config_t *cfg);

/* Backward of moe_expert_forward and of the un-permute (the derivative of the forward, the
 * conventions of moe_combine_backward; Quartz architecture table and Moonfrost expert card: the
 * routed SwiGLU experts on their grouped rows and the shared experts on every token). Per expert
 * e on its grouped rows X_e with upstream gradient dY_e, g = X_e W_g^T, u = X_e W_u^T:
 *   dh = dY_e W_d[e];  du = dh * silu(g);  dg = dh * u * silu'(g);  h = silu(g) * u
 *   d_w_down[e] = dY_e^T h;  d_w_gate[e] = dg^T X_e;  d_w_up[e] = du^T X_e
 *   dX_e = dg W_g[e] + du W_u[e]
 * Low-rank expert (dormouse, "TSCT low-rank experts"), z = X_e V[e]^T, Y = (z * s) U[e]^T:
 *   dzs = dY_e U[e];  d_lr_s[e] = sum over rows of dzs * z;  dz = dzs * s;
 *   d_lr_V[e] = dz^T X_e;  d_lr_U[e] = dY_e^T (z * s);  dX_e = dz V[e]
 * and likewise for the shared experts on all T tokens with upstream gradient dy. Then
 *   dx[t] = dX_shared[t] + sum over the token's kept pairs (t, j) of dX[slot_pos[t, j]]
 * (the experts' part of the input gradient; the router's part comes from moe_route_backward).
 * x_perm, offsets, slot_pos: as moe_permute produced them; x: the layer input; dy_perm: [T*k, d]
 * in y_perm's dtype (bf16 for SwiGLU, fp32 for low-rank layers), rows of kept pairs from
 * moe_combine_backward; dy: [T, d] fp32 (used for the shared experts, may be NULL when
 * n_shared = 0); dx: [T, d] fp32 output. g and u are recomputed in fp32; every product
 * accumulates in fp32 in a fixed order (bitwise reproducible). Experts with no rows get zero gradients.
 * Operands that are not exact bf16 values (g, u, dg, du, h, z, dz, z s, the fp32 dy and the
 * low-rank layers' fp32 dy_perm) enter the tensor-core products as two bf16 terms, value and
 * rounding residual, so each gradient carries no single bf16 rounding of its operands.
 * Supported: bf16 layers (SwiGLU or low-rank experts); fp32 layers and layers whose experts are
 * stored in fp8 (training stays bf16) return MOE_ERR_UNSUPPORTED.
 * SwiGLU weight gradients read x_perm and dy_perm in place, in 64-row blocks aligned to each
 * expert's last row: up to 63 rows before an expert's first row (earlier experts' rows) are
 * multiplied by zeros, so rows of x_perm and dy_perm past offsets[E] are never read, but a
 * non-finite value in one expert's rows can make the next expert's weight gradients non-finite.
 * ws: moe_backward_workspace_size(cfg) bytes of the caller's device memory. Asynchronous. */
moe_status_t moe_expert_backward(const moe_config_t *cfg, const void *x_perm,
                                 const int32_t *offsets, const int32_t *slot_pos, const void *x,
                                 const moe_weights_t *w, const void *dy_perm, const float *dy,
                                 float *dx, const moe_grads_t *g, void *ws, size_t ws_bytes,
                                 void *stream);

/* Backward of moe_route and of the load-balancing loss (Quartz: architecture table, row
 * "Router"; Sutra-1.3B, "48 + 1 experts" for sigmoid scores). Per token t, with the logits
 * recomputed as l = x W_r^T + off in fp32 (not the forward's exact rounding: a difference of a
 * few fp32 steps) and p = softmax(l) or sigmoid(l):
 *   dp[e_j] gets d_topk_w[t, j], through w_j = p_j / (sum of the k selected p) when norm_topk
 *   is set: dp[e_j] = (d_topk_w[t, j] - sum_i d_topk_w[t, i] w_i) / (that sum);
 *   dq[e] = d_loss * aux_alpha * E * (expert_count[e] / (T top_k)) / T, the loss's term;
 *   softmax: d_logits = p * (dp + dq - <dp + dq, p>);
 *   sigmoid: d_logits = (dp + (dq - <dq, q>) / sum(p)) * p * (1 - p), q = p / sum(p).
 * Then d_w_router = d_logits^T x ([E, d] fp32, the sum over t in token order) and
 * dx = d_logits W_r ([T, d] fp32, the router's part of the input gradient, sum over e in order).
 * x, w->w_router, w->logit_offset, topk_idx and expert_count (counts before capacity) as the
 * forward took or returned them; d_topk_w from moe_combine_backward; d_logits: [T, E] fp32
 * output; dx also holds the weight gradient's partial sums (over token ranges) until the call
 * writes it. Data-parallel replicas whose loss is formed from the statistics summed over the
 * ranks (T_global = world * T tokens) pass the summed counts and d_loss * (T / T_global)^2, then
 * sum d_w_router over the ranks. With T = 0 only d_w_router is written (zeros). All buffers
 * are the caller's device memory, 16-byte aligned; d_loss must be finite. Asynchronous on
 * `stream`; bad arguments return MOE_ERR_INVALID_ARG. */
moe_status_t moe_route_backward(const moe_config_t *cfg, const void *x, const moe_weights_t *w,
                                const int32_t *topk_idx, const int32_t *expert_count,
                                const float *d_topk_w, float d_loss, float *d_logits,
                                float *d_w_router, float *dx, void *stream);

/* Load-balancing loss (Quartz: architecture table, row "Router", weight 0.01):
 *   loss = aux_alpha * E * sum_i (expert_count[i] / (T*top_k)) * (prob_sum[i] / T)
 * written to the device scalar `loss` (fp32); 0 when T = 0. */
moe_status_t moe_aux_loss(const moe_config_t *cfg, const int32_t *expert_count,
                          const float *prob_sum, float *loss, void *stream);

/* Loss-free balancing step (dormouse, "dropless MoE": a bias on the router balances the load in
 * place of an auxiliary loss, after arXiv 2408.15664). For every expert i:
 *   select_bias[i] <- RN32(select_bias[i] + u * sign(mean - expert_count[i])),
 *   mean = sum_j expert_count[j] / E,
 * the sign decided exactly on integers (sign(0) = 0), one fp32 rounding (nearest even).
 * expert_count: [E] int32 on the device, the per-expert selection counts before capacity drops
 * (as moe_route and moe_layer_forward return them); select_bias: [E] fp32 on the device,
 * updated in place and read by the next sigmoid-scored routing call; u: the step size (the
 * pages give none). Only cfg->E of the configuration is used, but the whole configuration is
 * validated. Asynchronous on `stream`; bad arguments return MOE_ERR_INVALID_ARG. */
moe_status_t moe_bias_update(const moe_config_t *cfg, const int32_t *expert_count,
                             float *select_bias, float u, void *stream);

/* The whole layer: route -> permute -> experts -> combine -> loss, no host synchronisation
 * (the layer of the Quartz architecture table: router, 24 routed experts top-6, 2 shared experts,
 * load-balancing loss 0.01; the Moonfrost expert card's stacked experts under a capacity, whose
 * per-expert host loop this call replaces: no count returns to the host).
 *   y [T, d] fp32; aux_loss: device fp32 scalar (may be NULL); expert_count: optional [E]
 *   int32 output of the router's per-expert selection counts (may be NULL). */
moe_status_t moe_layer_forward(const moe_config_t *cfg, const void *x, const moe_weights_t *w,
                               void *y, float *aux_loss, int32_t *expert_count,
                               void *ws, size_t ws_bytes, void *stream);

/* moe_route without a workspace, for callers that cannot allocate device memory.
 * The source pages have no counterpart to this entry point; it serves integration needs only.
 * Some callers cannot call cudaMalloc or hand out a workspace: for example a plugin that runs
 * inside a host framework whose allocator owns all device memory, or a latency-critical loop
 * where cudaMalloc's implicit device-wide synchronisation is not acceptable. This variant
 * computes exactly what moe_route computes (same kernels, same outputs), but its scratch lives
 * in a fixed array of MOE_ROUTE_NOALLOC_SCRATCH_BYTES in the library's own device memory, which
 * every GPU that loads the library holds until the process exits. The caller still passes x,
 * the weights and all outputs.
 *   - Limit: the scratch needed is about 8*E*ceil(T/16) bytes; configurations that need
 *     more than MOE_ROUTE_NOALLOC_SCRATCH_BYTES return MOE_ERR_WORKSPACE with nothing enqueued.
 *   - Set-up: the first call on each device looks up the array's device address (with that
 *     device current); make that first call before any stream capture begins. The address is
 *     kept per device together with the id of the context it belongs to: if the device's
 *     context is made anew (cudaDeviceReset, or another library that resets the device), the
 *     next call looks it up again, and that call too must come before any stream capture.
 *   - Sharing: every call on a device uses the same array. Calls whose work overlaps on the GPU
 *     (other streams, other host threads) race on it and must be serialised by the caller. */
#define MOE_ROUTE_NOALLOC_SCRATCH_BYTES (4u << 20)
moe_status_t moe_route_noalloc(const moe_config_t *cfg, const void *x, const moe_weights_t *w,
                               int32_t *topk_idx, float *topk_w, int32_t *expert_count,
                               float *prob_sum, void *stream);

/* Per-row E4M3 quantisation, the fp8 storage of moe_storage_t (dormouse, "TSCT low-rank
 * experts": the storage ladder fp8 -> NVFP4 -> ternary of the U*diag(s)*V^T factorisation; the
 * pages fix no scale granularity or rounding, so this is one scale per row and round to nearest).
 * For every row v of `in` ([rows, cols], row-major; in_dtype MOE_DTYPE_BF16 or MOE_DTYPE_F32):
 *   amax = max_i |v_i|;  scale[row] = RN32(amax / 448), or 1 for an all-zero row;
 *   q[row, i] = E4M3 code of RN32(v_i / scale[row]), rounded to the nearest E4M3 value with ties
 *   to the even code and magnitudes above 448 saturated (E4M3: 1 sign, 4 exponent bits of bias 7,
 *   3 mantissa bits, largest finite 448; OCP FP8).
 * q: [rows, cols] uint8; scale: [rows] fp32; cols a multiple of 16; inputs finite. The weights of
 * an fp8 low-rank layer are lr_V8 / lr_V_scale = moe_quantize_fp8(V viewed as [E*rank, d]) and
 * lr_U8 / lr_U_scale = moe_quantize_fp8(U viewed as [E*d, rank]). Asynchronous on `stream`; bad
 * arguments return MOE_ERR_INVALID_ARG or MOE_ERR_UNSUPPORTED with nothing enqueued. */
moe_status_t moe_quantize_fp8(const void *in, int32_t in_dtype, int64_t rows, int32_t cols,
                              uint8_t *q, float *scale, void *stream);

/* Human-readable name of a status. Never NULL. */
const char *moe_status_str(moe_status_t s);

/* Synchronises `stream`, then returns and clears the device error word of the current device
 * (MOE_OK if no device-side fault was recorded). *info (may be NULL) receives a detail code:
 *   MOE_ERR_DEVICE_CHECK: 1 a sigmoid key that could not be resolved exactly; 2 an exact-sum
 *     expansion that ran out of terms; 3 a selected expert index outside [0, E) given to
 *     moe_route_backward; 100 + j an expert index outside [0, E) in slot j of moe_permute's
 *     topk_idx.
 *   MOE_ERR_TIMEOUT: the bounded wait that ran out: 10 operands (MMA waiting for TMA), 11 a
 *     free stage (TMA waiting for the MMA), 12 a full accumulator, 13 a free accumulator, 14 the
 *     drain of copies still in flight, 15 the router's token rows, 16 the scatter's token rows,
 *     20 the timeout probe. */
moe_status_t moe_get_device_error(void *stream, int64_t *info);

/* Test and measurement controls (synchronous, current device):
 *   MOE_DEBUG_FORCE_EXACT: 1 = route every logit and sigmoid key through the exact paths
 *     instead of only the ones the fp64 screen cannot decide; 2 = the same, with logits sent to
 *     the floating-point expansion rather than the exact integer sum (for parity tests);
 *   MOE_DEBUG_WAIT_LIMIT_NS: upper bound on any device-side wait (default 2e9 ns);
 *   MOE_DEBUG_PROFILE: 1 = record a CUDA event pair around every kernel the library launches,
 *     per kernel kind, read with moe_profile_read(). The events end the overlap of a kernel with
 *     its predecessor's tail, so a short kernel reads longer than it runs inside a layer call;
 *   MOE_DEBUG_STAMP: 1 = every forward kernel records, on the device's global timer, when its
 *     first CTA's inputs became final and when its last warp finished, per kernel kind, read with
 *     moe_stamp_read(); the launches stay overlapped as in normal operation. */
typedef enum { MOE_DEBUG_FORCE_EXACT = 1, MOE_DEBUG_WAIT_LIMIT_NS = 2, MOE_DEBUG_PROFILE = 3,
               MOE_DEBUG_STAMP = 4 } moe_debug_t;
moe_status_t moe_debug_set(int32_t what, int64_t value);

/* Kernel-level timing collected while MOE_DEBUG_PROFILE is on. Synchronises the device.
 * Fills up to `max` entries: names[i] (static strings), total_ms[i] and launches[i]; returns
 * the number of kernel kinds with at least one launch, and resets the accumulators. */
int32_t moe_profile_read(const char **names, double *total_ms, int64_t *launches, int32_t max);

/* In-step kernel durations recorded while MOE_DEBUG_STAMP is on: per kernel kind that ran since
 * the last read, the time from its first CTA's inputs becoming final to its last warp's end, in
 * microseconds (several launches of one kind in that interval count as one span). Synchronises
 * the device, fills up to `max` entries of names[i] (static strings) and us[i], returns the
 * number of kinds (or -1 on a CUDA error) and clears the records. */
int32_t moe_stamp_read(const char **names, double *us, int32_t max);

/* Test hook for failure detection: launches one tiny kernel that waits on a shared-memory
 * barrier nothing will complete, bounded by MOE_DEBUG_WAIT_LIMIT_NS; the kernel then records
 * MOE_ERR_TIMEOUT in the device error word and returns. Returns the launch status. */
moe_status_t moe_debug_wait_timeout_probe(void *stream);

#ifdef __cplusplus
}
#endif
#endif /* MOE_H */

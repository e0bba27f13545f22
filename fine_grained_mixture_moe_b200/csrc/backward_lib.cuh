// Host side of the backward entry points: launch sequences and the workspace layout of
// moe_expert_backward. Included by moe_lib.cu inside its internal namespace, after the forward
// launch helpers (launch_pdl, launch_tc2, the tensor maps) that it uses.
#pragma once

// ------------------------------------------------------------------ backward of route and combine
template <typename Tin>
moe_status_t route_backward_impl(const moe_config_t *c, const RouteBwdArgs &a, float *d_w_router,
                                 float *dx, cudaStream_t st) {
  const size_t smem = route_bwd_smem_floats(c->E) * sizeof(float);
  if (smem > 48 * 1024 &&
      cudaFuncSetAttribute(route_backward_kernel<Tin>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           (int)smem) != cudaSuccess)
    return MOE_ERR_CUDA;
  MOE_TRY(launch_pdl(route_backward_kernel<Tin>, dim3(ceil_div(c->T, RB_TM)), dim3(256), smem, st,
                     a));
  // d_w_router over S token ranges (about two blocks per SM); their partial sums [S, E, d] live
  // in dx (T x d floats, S E <= T) until the last kernel writes dx
  const int per_split = ceil_div(c->d, 512) * ceil_div(c->E, 8);
  const int S = std::max(1, std::min({64, c->T / c->E, ceil_div(2 * 148, per_split)}));
  float *part = S > 1 ? dx : d_w_router;
  MOE_TRY(launch_pdl(router_wgrad_kernel<Tin>, dim3(ceil_div(c->d, 512), ceil_div(c->E, 8), S),
                     dim3(256), 0, st, (const float *)a.d_logits, (const Tin *)a.x, c->T, c->d,
                     c->E, S, part));
  if (S > 1)
    MOE_TRY(launch_pdl(router_wgrad_sum_kernel, dim3(ceil_div((long long)c->E * c->d, 256)),
                       dim3(256), 0, st, (const float *)part, S, c->E, c->d, d_w_router));
  return launch_pdl(router_dgrad_kernel<Tin>, dim3(ceil_div(c->d, 1024), std::min(ceil_div(c->T, 16), 65535)),
                    dim3(256), 0, st, (const float *)a.d_logits, (const Tin *)a.w_router, c->T,
                    c->d, c->E, dx);
}

// ------------------------------------------------------------------ backward of the experts
// Workspace of moe_expert_backward (bf16 layers): g and u recomputed (fp32), [dg | du] and h as
// hi + lo bf16 terms (routed rows at the padded positions koff, zero padding rows first), the routed dX
// before the un-permute, the shared experts' counterparts, dy as hi + lo terms and the transposed
// weights. The SwiGLU weight gradients read the activations in place (MN-major operands); the
// low-rank ones still use transposed, per-expert zero-padded copies (2 or 3 K segments).
constexpr int BWD_SHARED_CHUNKS = 8;

struct BwdLayout {
  size_t koff, korder, kstart, off_s, koff_s;
  size_t gu, dgu, h, dxp, gu_s, dgu_s, h_s, dx_s, dy_b;
  size_t wdt, wgut, wsdt, wsgut;
  size_t ydt, xpt;
  size_t z, dzs, dys, dz2, zs2, ut, vt, dzt, zst, ds_part;  // low-rank experts
  size_t part_s;  // the shared experts' weight gradients per token chunk
  size_t total;
  int npad;
  int nc, ch;     // token chunks of the shared experts' weight gradients, rows per chunk
};

BwdLayout bwd_layout(const moe_config_t *c) {
  BwdLayout L;
  const bool swi = c->expert == MOE_EXPERT_SWIGLU;
  const size_t T = c->T, d = c->d, E = c->E, k = c->top_k;
  const size_t f = swi ? c->ffn : 0, r = swi ? 0 : c->rank;
  const size_t sf = (size_t)c->n_shared * c->ffn_shared, N = T * k;
  L.npad = (int)(((N + 64 * E) + 63) & ~(size_t)63);  // >= the sum of the padded group sizes
  // the shared experts' T rows in nc chunks of ch rows, so that their weight gradients (few
  // output tiles, long K) fill the GPU; the chunks' partial sums are added in chunk order
  L.nc = std::max(1, std::min(BWD_SHARED_CHUNKS, ceil_div((long long)T, 512)));
  L.ch = (int)(((size_t)ceil_div((long long)std::max<size_t>(T, 1), L.nc) + 63) & ~(size_t)63);
  const size_t np = L.npad;
  size_t o = 0;
  auto take = [&](size_t bytes) { size_t at = o; o = align256(o + std::max<size_t>(bytes, 1)); return at; };
  L.koff = take((E + 1) * 4);
  L.korder = take(E * 4);
  L.kstart = take(E * 4);
  L.off_s = take((BWD_SHARED_CHUNKS + 1) * 4);
  L.koff_s = take((BWD_SHARED_CHUNKS + 1) * 4);
  L.gu = take(np * 2 * f * 4);  // blocked g, u: each group's rows padded to 64
  L.dgu = take(np * 4 * f * 2);
  L.h = take(np * 2 * f * 2);
  L.dxp = take(N * d * 4);
  L.gu_s = take(((T + 63) & ~(size_t)63) * 2 * sf * 4);
  L.dgu_s = take(T * 4 * sf * 2);
  L.h_s = take(T * 2 * sf * 2);
  L.dx_s = take(T * d * 4);
  L.dy_b = take(sf ? T * 2 * d * 2 : 0);
  L.wdt = take(E * f * d * 2);
  L.wgut = take(E * d * 2 * f * 2);
  L.wsdt = take(sf * d * 2);
  L.wsgut = take(d * 2 * sf * 2);
  L.ydt = take(swi ? 0 : d * 3 * np * 2);
  L.xpt = take(swi ? 0 : d * 2 * np * 2);
  L.z = take(N * r * 4);
  L.dzs = take(N * r * 4);
  L.dys = take(r ? N * 2 * d * 2 : 0);
  L.dz2 = take(N * 2 * r * 2);
  L.zs2 = take(N * 2 * r * 2);
  L.ut = take(E * r * d * 2);
  L.vt = take(E * d * r * 2);
  L.dzt = take(r * 2 * np * 2);
  L.zst = take(r * 3 * np * 2);
  L.ds_part = take((np / 64) * r * 4);
  L.part_s = take(sf ? (size_t)L.nc * std::max(sf * d, d * (size_t)c->ffn_shared) * 4 : 0);
  L.total = o;
  return L;
}

using bf16_t = __nv_bfloat16;

// Transposes (transpose_bf16_kernel): grouped rows -> nseg padded column segments, or dense
// batches.
moe_status_t launch_transpose_grouped(int nseg, const bf16_t *s0, const bf16_t *s1,
                                      const bf16_t *s2, int C, int ldi, const int32_t *offsets,
                                      const int32_t *koff, int G, int ncolblocks, void *out,
                                      int ldo, cudaStream_t st) {
  return launch_pdl(transpose_bf16_kernel, dim3(ceil_div(C, TR_COLS), ncolblocks, 1), dim3(256), 0, st,
                    s0, s1, s2, nseg, C, ldi, offsets, koff, G, 0, (size_t)0, (bf16_t *)out, ldo,
                    (size_t)0, 0);
}
moe_status_t launch_transpose_dense(const bf16_t *in, int R, int C, int batches, size_t ibs,
                                    void *out, int ldo, size_t obs, int col0, cudaStream_t st) {
  return launch_pdl(transpose_bf16_kernel, dim3(ceil_div(C, TR_COLS), ceil_div(R, 64), batches),
                    dim3(256), 0, st, in, (const bf16_t *)nullptr, (const bf16_t *)nullptr, 1, C,
                    C, (const int32_t *)nullptr, (const int32_t *)nullptr, 0, R, ibs,
                    (bf16_t *)out, ldo, obs, col0);
}

// One weight-gradient product with groups along K: out[g] (M x N, fp32, row-major) =
// A[:, kseg koff[g] .. kseg koff[g+1]) B[:, same]^T, A [M, ld], B [N, ld] bf16. `order` (device,
// or null for group order) lists the groups in the order their tiles are dealt to the CTA pairs.
moe_status_t launch_wgrad(int G, const int32_t *koff, const int32_t *order, int kseg,
                          const void *A, int M, const void *Bm, int N, int ld, float *out,
                          cudaStream_t st) {
  GroupedGemm g;
  std::memset(&g, 0, sizeof(g));
  g.kgroup = 1;
  g.koff = koff;
  g.gorder = order;
  g.kseg = kseg;
  g.E = G;
  g.A_r = A;
  g.lda_r = ld;
  g.rows_r = M;
  g.B0_r = Bm;
  g.N_r = N;
  g.K_r = ld;
  g.out_r = out;
  g.ldo_r = N;
  return launch_tc2<MODE_PLAIN>(g, st, K_BWD_GEMM);
}

// One weight-gradient product with groups along K whose operands are read in place (MN-major):
// out[g] (M x N, fp32, row-major) = sum over segments s < kseg of A[ra, col_a[s] + m] B[rb,
// col_b[s] + n] over k < koff[g+1] - koff[g], ra = row_a[g] + k, rb = row_b[g] + k. A [rows_a,
// lda] and B [rows_b, ldb] bf16 row-major; past a group's last row one of the two operands holds
// zeros (a padded layout, or the end of the matrix).
struct MnOperand {
  const void *ptr;
  int ld, rows;
  const int32_t *row0;  // [G] device
  int col[3];
};
moe_status_t launch_wgrad_mn(int G, const int32_t *koff, const int32_t *order, int kseg,
                             const MnOperand &A, int M, const MnOperand &Bm, int N, float *out,
                             cudaStream_t st) {
  GroupedGemm g;
  std::memset(&g, 0, sizeof(g));
  g.kgroup = 1;
  g.mn = 1;
  g.koff = koff;
  g.gorder = order;
  g.kseg = kseg;
  g.E = G;
  g.A_r = A.ptr;
  g.B0_r = Bm.ptr;
  g.rows_r = M;
  g.N_r = N;
  g.mn_lda = A.ld;
  g.mn_ldb = Bm.ld;
  g.mn_rows_a = A.rows;
  g.mn_rows_b = Bm.rows;
  g.mn_row_a = A.row0;
  g.mn_row_b = Bm.row0;
  for (int s = 0; s < kseg; ++s) {
    g.mn_col_a[s] = A.col[s];
    g.mn_col_b[s] = Bm.col[s];
  }
  g.out_r = out;
  g.ldo_r = N;
  return launch_tc2<MODE_PLAIN>(g, st, K_BWD_GEMM);
}

moe_status_t expert_backward_impl(const moe_config_t *c, const void *x_perm,
                                  const int32_t *offsets, const int32_t *slot_pos, const void *x,
                                  const moe_weights_t *w, const void *dy_perm, const float *dy,
                                  float *dx, const moe_grads_t *gr, void *ws, cudaStream_t st) {
  const BwdLayout L = bwd_layout(c);
  const bool swi = c->expert == MOE_EXPERT_SWIGLU;
  const int T = c->T, d = c->d, E = c->E, k = c->top_k, f = swi ? c->ffn : 0;
  const int r = swi ? 0 : c->rank;
  const int S = c->n_shared, fs = c->ffn_shared, sf = S * fs;
  const bool sh = S > 0;
  using bf = bf16_t;
  int32_t *koff = at<int32_t>(ws, L.koff), *korder = at<int32_t>(ws, L.korder),
          *kstart = at<int32_t>(ws, L.kstart),
          *off_s = at<int32_t>(ws, L.off_s), *koff_s = at<int32_t>(ws, L.koff_s);
  float *GU = at<float>(ws, L.gu), *GUs = at<float>(ws, L.gu_s);
  bf *DGU = at<bf>(ws, L.dgu), *H = at<bf>(ws, L.h);
  float *dXp = at<float>(ws, L.dxp), *dXs = at<float>(ws, L.dx_s);
  bf *DGUs = at<bf>(ws, L.dgu_s), *Hs = at<bf>(ws, L.h_s), *dyb = at<bf>(ws, L.dy_b);
  bf *Wdt = at<bf>(ws, L.wdt), *Wgut = at<bf>(ws, L.wgut), *Wsdt = at<bf>(ws, L.wsdt),
     *Wsgut = at<bf>(ws, L.wsgut);
  bf *Ydt = at<bf>(ws, L.ydt), *Xpt = at<bf>(ws, L.xpt);
  const int np = L.npad;
  const bf *xp = (const bf *)x_perm;

  // padded group offsets of the weight gradients
  MOE_TRY(launch_pdl(pad_offsets_kernel, dim3(1), dim3(1024), 0, st, offsets, E, koff, korder,
                     kstart, T, L.nc, L.ch, off_s, koff_s));
  // the SwiGLU launches carry the routed SwiGLU experts (E groups) and / or the shared experts
  GroupedGemm base;
  std::memset(&base, 0, sizeof(base));
  base.offsets = offsets;
  base.T = T;
  base.rows_r = T * k;
  base.E = swi ? E : 0;
  base.has_shared = sh;
  const bool swiglu_launch = swi || sh;
  // g and u (fp32) of the routed rows, and of every token for the shared experts
  if (swiglu_launch) {
    GroupedGemm g = base;
    if (swi) {
      g.A_r = x_perm; g.lda_r = d; g.B0_r = w->w_gate; g.B1_r = w->w_up; g.N_r = f; g.K_r = d;
      g.out_r = GU; g.half_r = f; g.aux_row0 = koff;
    }
    if (sh) {
      g.A_s = x; g.lda_s = d; g.B0_s = w->ws_gate; g.B1_s = w->ws_up; g.N_s = sf; g.K_s = d;
      g.piece_k = d; g.b_rows_s = sf; g.out_s = GUs; g.half_s = sf;
    }
    MOE_TRY(launch_tc2<MODE_GATEUP_RAW>(g, st, K_BWD_GEMM));
  }
  // transposed weights: W_d [E][d][f] -> [E][f][d]; [W_g; W_u] -> [E][d][2f]; shared likewise
  if (swi) {
    const bf *wg = (const bf *)w->w_gate, *wu = (const bf *)w->w_up, *wd = (const bf *)w->w_down;
    MOE_TRY(launch_transpose_dense(wd, d, f, E, (size_t)d * f, Wdt, d, (size_t)f * d, 0, st));
    MOE_TRY(launch_transpose_dense(wg, f, d, E, (size_t)f * d, Wgut, 2 * f, (size_t)d * 2 * f, 0, st));
    MOE_TRY(launch_transpose_dense(wu, f, d, E, (size_t)f * d, Wgut, 2 * f, (size_t)d * 2 * f, f, st));
  }
  if (sh) {
    const bf *sg = (const bf *)w->ws_gate, *su = (const bf *)w->ws_up, *sdn = (const bf *)w->ws_down;
    MOE_TRY(launch_transpose_dense(sdn, d, fs, S, (size_t)d * fs, Wsdt, d, (size_t)fs * d, 0, st));
    MOE_TRY(launch_transpose_dense(sg, sf, d, 1, 0, Wsgut, 2 * sf, 0, 0, st));
    MOE_TRY(launch_transpose_dense(su, sf, d, 1, 0, Wsgut, 2 * sf, 0, sf, st));
    // the shared experts' upstream gradient (fp32) as hi + lo bf16 terms
    MOE_TRY(launch_pdl(split_bf16_kernel,
                       dim3((unsigned)std::min<long long>(ceil_div((long long)T * d, 1024), 65535)),
                       dim3(256), 0, st, dy, d, (size_t)T, dyb));
  }
  // dh = dY W_d with the SwiGLU backward in the epilogue: [dg | du] and h as hi + lo terms
  if (swiglu_launch) {
    GroupedGemm g = base;
    if (swi) {
      g.A_r = dy_perm; g.lda_r = d; g.B0_r = Wdt; g.N_r = f; g.K_r = d;
      g.out_r = DGU; g.ldo_r = 4 * f; g.half_r = f; g.out2_r = H; g.ld2_r = 2 * f;
      g.aux_r = GU; g.aux_row0 = koff; g.pad_out = 1;
    }
    if (sh) {  // A = [dy_hi | dy_lo], K = 2d, the weight's k wraps over its d columns
      g.A_s = dyb; g.lda_s = 2 * d; g.B0_s = Wsdt; g.N_s = sf; g.K_s = 2 * d; g.piece_k = d;
      g.piece_rows = 0; g.b_rows_s = sf; g.out_s = DGUs; g.ldo_s = 4 * sf; g.half_s = sf;
      g.out2_s = Hs; g.ld2_s = 2 * sf; g.aux_s = GUs;
    }
    MOE_TRY(launch_tc2<MODE_SWIGLU_BWD>(g, st, K_BWD_GEMM));
  }
  // dX = [dg | du]_hi [W_g; W_u] + [dg | du]_lo [W_g; W_u] (fp32; K = 4 ffn, the weight's k
  // wraps); the shared experts' dX likewise
  if (swiglu_launch) {
    GroupedGemm g = base;
    if (swi) {
      g.A_r = DGU; g.lda_r = 4 * f; g.B0_r = Wgut; g.N_r = d; g.K_r = 4 * f; g.kb_r = 2 * f;
      g.out_r = dXp; g.ldo_r = d; g.out_r_bf16 = 0;
      g.a_row_end = koff; g.rows_r = np;  // [dg | du] rows at the padded positions
    }
    if (sh) {
      g.A_s = DGUs; g.lda_s = 4 * sf; g.B0_s = Wsgut; g.N_s = d; g.K_s = 4 * sf;
      g.piece_k = 2 * sf; g.piece_rows = 0; g.b_rows_s = d; g.out_s = dXs; g.ldo_s = d;
    }
    MOE_TRY(launch_tc2<MODE_PLAIN>(g, st, K_BWD_GEMM));
  }
  if (!swi) {
    // low-rank experts, Y = (z s) U^T with z = X V^T: dzs = dY U, dz = dzs s, ds = sum dzs z,
    // dX = dz V, dV = dz^T X, dU = dY^T (z s). dY (fp32) and dz, z s run as hi + lo terms.
    float *Z = at<float>(ws, L.z), *dZS = at<float>(ws, L.dzs), *dsp = at<float>(ws, L.ds_part);
    bf *dYs = at<bf>(ws, L.dys), *DZ2 = at<bf>(ws, L.dz2), *ZS2 = at<bf>(ws, L.zs2);
    bf *Ut = at<bf>(ws, L.ut), *Vt = at<bf>(ws, L.vt), *DZt = at<bf>(ws, L.dzt),
       *ZSt = at<bf>(ws, L.zst);
    const bf *V = (const bf *)w->lr_V, *U = (const bf *)w->lr_U;
    GroupedGemm lr;
    std::memset(&lr, 0, sizeof(lr));
    lr.offsets = offsets;
    lr.T = T;
    lr.rows_r = T * k;
    lr.E = E;
    {  // z = X V^T (fp32)
      GroupedGemm g = lr;
      g.A_r = x_perm; g.lda_r = d; g.B0_r = V; g.N_r = r; g.K_r = d; g.out_r = Z; g.ldo_r = r;
      MOE_TRY(launch_tc2<MODE_PLAIN>(g, st, K_BWD_GEMM));
    }
    MOE_TRY(launch_transpose_dense(U, d, r, E, (size_t)d * r, Ut, d, (size_t)r * d, 0, st));
    MOE_TRY(launch_transpose_dense(V, r, d, E, (size_t)r * d, Vt, r, (size_t)d * r, 0, st));
    MOE_TRY(launch_pdl(split_bf16_kernel,
                       dim3((unsigned)std::min<long long>(ceil_div((long long)T * k * d, 1024), 65535)),
                       dim3(256), 0, st, (const float *)dy_perm, d, (size_t)T * k, dYs));
    {  // dzs = [dY_hi | dY_lo] U (K = 2d, U^T's k wraps over its d columns)
      GroupedGemm g = lr;
      g.A_r = dYs; g.lda_r = 2 * d; g.B0_r = Ut; g.N_r = r; g.K_r = 2 * d; g.kb_r = d;
      g.out_r = dZS; g.ldo_r = r;
      MOE_TRY(launch_tc2<MODE_PLAIN>(g, st, K_BWD_GEMM));
    }
    MOE_TRY(launch_pdl(lowrank_elem_kernel, dim3(np / 64), dim3(256), 0, st, (const float *)Z,
                       (const float *)dZS, w->lr_s, offsets, koff, E, r, DZ2, ZS2, dsp));
    MOE_TRY(launch_pdl(lowrank_ds_kernel, dim3(E), dim3(256), 0, st, (const float *)dsp, koff, r,
                       gr->d_lr_s));
    {  // dX = [dz_hi | dz_lo] V (K = 2r, V^T's k wraps over its r columns)
      GroupedGemm g = lr;
      g.A_r = DZ2; g.lda_r = 2 * r; g.B0_r = Vt; g.N_r = d; g.K_r = 2 * r; g.kb_r = r;
      g.out_r = dXp; g.ldo_r = d;
      MOE_TRY(launch_tc2<MODE_PLAIN>(g, st, K_BWD_GEMM));
    }
    const int nb2 = 2 * np / 64, nb3 = 3 * np / 64;
    MOE_TRY(launch_transpose_grouped(2, DZ2, DZ2 + r, nullptr, r, 2 * r, offsets, koff, E, nb2,
                                     DZt, 2 * np, st));
    MOE_TRY(launch_transpose_grouped(2, xp, xp, nullptr, d, d, offsets, koff, E, nb2, Xpt, 2 * np, st));
    MOE_TRY(launch_transpose_grouped(3, dYs, dYs, dYs + d, d, 2 * d, offsets, koff, E, nb3, Ydt,
                                     3 * np, st));
    MOE_TRY(launch_transpose_grouped(3, ZS2, ZS2 + r, ZS2, r, 2 * r, offsets, koff, E, nb3, ZSt,
                                     3 * np, st));
    MOE_TRY(launch_wgrad(E, koff, korder, 2, DZt, r, Xpt, d, 2 * np, gr->d_lr_V, st));
    MOE_TRY(launch_wgrad(E, koff, korder, 3, Ydt, d, ZSt, r, 3 * np, gr->d_lr_U, st));
    MOE_TRY(launch_pdl(zero_empty_experts_kernel, dim3(E, 8), dim3(256), 0, st, offsets,
                       gr->d_lr_V, (size_t)r * d, gr->d_lr_U, (size_t)d * r, (float *)nullptr,
                       (size_t)0));
  }
  // the un-permute: dx[t] = dX_s[t] + sum_j dX[pos(t, j)]
  MOE_TRY(launch_pdl(combine_kernel<float>, dim3(ceil_div(T, 8)), dim3(256), 0, st,
                     (const float *)dXp, sh ? (const float *)dXs : (const float *)nullptr,
                     slot_pos, (const float *)nullptr, dx, T, k, d, false));
  if (swi) {
    // weight gradients: one operand as hi + lo segments, the other repeated, so that each
    // product sums both terms: dW_d = dY^T (h_hi + h_lo), dW_g = (dg_hi + dg_lo)^T X, dW_u.
    // h and [dg | du] rows from koff (zeros first, then the group's rows); dY and X rows from
    // kstart, so that the group's rows meet its rows and the rows before them meet zeros
    // (the rows past the last kept pair, which no kernel writes, are never read).
    const int N = T * k;
    const MnOperand dyo{dy_perm, d, N, kstart, {0, 0, 0}};
    const MnOperand ho{H, 2 * f, np, koff, {0, f, 0}};
    const MnOperand xo{x_perm, d, N, kstart, {0, 0, 0}};
    const MnOperand dgo{DGU, 4 * f, np, koff, {0, 2 * f, 0}};
    const MnOperand duo{DGU, 4 * f, np, koff, {f, 3 * f, 0}};
    MOE_TRY(launch_wgrad_mn(E, koff, korder, 2, dyo, d, ho, f, gr->d_w_down, st));
    MOE_TRY(launch_wgrad_mn(E, koff, korder, 2, dgo, f, xo, d, gr->d_w_gate, st));
    MOE_TRY(launch_wgrad_mn(E, koff, korder, 2, duo, f, xo, d, gr->d_w_up, st));
    MOE_TRY(launch_pdl(zero_empty_experts_kernel, dim3(E, 8), dim3(256), 0, st, offsets,
                       gr->d_w_gate, (size_t)f * d, gr->d_w_up, (size_t)f * d, gr->d_w_down,
                       (size_t)d * f));
  }
  if (sh) {
    // dW_sg, dW_su: (dg_hi + dg_lo)^T x; dW_sd: (dy_hi + dy_lo)^T (h_hi + h_lo) less lo lo,
    // three segments [hi hi | hi lo | lo hi]; each over the nc token chunks (64-aligned; rows
    // past T read as zeros), then the chunks' partial sums added in order
    const int nc = L.nc;
    float *part = at<float>(ws, L.part_s);
    auto sum_chunks = [&](size_t n, float *out) {
      return launch_pdl(sum_chunks_kernel, dim3((unsigned)std::min<long long>(ceil_div((long long)n, 1024), 4096)),
                        dim3(256), 0, st, (const float *)part, nc, n, out);
    };
    const MnOperand xo{x, d, T, off_s, {0, 0, 0}};
    const MnOperand dgo{DGUs, 4 * sf, T, off_s, {0, 2 * sf, 0}};
    const MnOperand duo{DGUs, 4 * sf, T, off_s, {sf, 3 * sf, 0}};
    const MnOperand dyo{dyb, 2 * d, T, off_s, {0, 0, d}};
    MOE_TRY(launch_wgrad_mn(nc, koff_s, nullptr, 2, dgo, sf, xo, d, part, st));
    MOE_TRY(sum_chunks((size_t)sf * d, gr->d_ws_gate));
    MOE_TRY(launch_wgrad_mn(nc, koff_s, nullptr, 2, duo, sf, xo, d, part, st));
    MOE_TRY(sum_chunks((size_t)sf * d, gr->d_ws_up));
    for (int s = 0; s < S; ++s) {
      const MnOperand ho{Hs, 2 * sf, T, off_s, {s * fs, sf + s * fs, s * fs}};
      MOE_TRY(launch_wgrad_mn(nc, koff_s, nullptr, 3, dyo, d, ho, fs, part, st));
      MOE_TRY(sum_chunks((size_t)d * fs, gr->d_ws_down + (size_t)s * d * fs));
    }
  }
  return MOE_OK;
}

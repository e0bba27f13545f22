// C ABI entry points of the backward (moe_combine_backward, moe_route_backward,
// moe_backward_workspace_size, moe_expert_backward): argument checks and the calls into
// backward_lib.cuh. Included by moe_lib.cu inside its extern "C" block.
#pragma once

moe_status_t moe_combine_backward(const moe_config_t *cfg, const float *dy, const void *y_perm,
                                  const int32_t *slot_pos, const float *topk_w, void *dy_perm,
                                  float *d_topk_w, void *stream) {
  MOE_TRY(check_cfg(cfg));
  MOE_REQUIRE(tok16(cfg, dy) && tok16(cfg, y_perm) && tok16(cfg, slot_pos) && tok16(cfg, topk_w) &&
              tok16(cfg, dy_perm) && tok16(cfg, d_topk_w));
  if (cfg->T == 0) return MOE_OK;
  cudaStream_t st = (cudaStream_t)stream;
  // tokens per block: as many as leave each token's 256-column slices a warp each (8 warps)
  const int slices = ceil_div(cfg->d, 256);
  int tpb = 8;
  while (tpb > 1 && tpb * slices > 8) tpb >>= 1;
  const dim3 grid(ceil_div(cfg->T, tpb));
  if (yperm_bf16(cfg))
    return launch_pdl(combine_backward_kernel<__nv_bfloat16>, grid, dim3(256), 0, st, dy,
                      (const __nv_bfloat16 *)y_perm, slot_pos, topk_w, (__nv_bfloat16 *)dy_perm,
                      d_topk_w, cfg->T, cfg->top_k, cfg->d, tpb);
  return launch_pdl(combine_backward_kernel<float>, grid, dim3(256), 0, st, dy,
                    (const float *)y_perm, slot_pos, topk_w, (float *)dy_perm, d_topk_w, cfg->T,
                    cfg->top_k, cfg->d, tpb);
}

moe_status_t moe_route_backward(const moe_config_t *cfg, const void *x, const moe_weights_t *w,
                                const int32_t *topk_idx, const int32_t *expert_count,
                                const float *d_topk_w, float d_loss, float *d_logits,
                                float *d_w_router, float *dx, void *stream) {
  MOE_TRY(check_cfg(cfg));
  MOE_TRY(check_weights(cfg, w, true, false));
  MOE_REQUIRE(std::isfinite(d_loss));
  MOE_REQUIRE(tok16(cfg, x) && tok16(cfg, topk_idx) && aligned16(expert_count) &&
              tok16(cfg, d_topk_w) && tok16(cfg, d_logits) && aligned16(d_w_router) &&
              tok16(cfg, dx));
  cudaStream_t st = (cudaStream_t)stream;
  if (cfg->T == 0)
    return cudaMemsetAsync(d_w_router, 0, (size_t)cfg->E * cfg->d * sizeof(float), st) == cudaSuccess
               ? MOE_OK
               : MOE_ERR_CUDA;
  RouteBwdArgs a;
  std::memset(&a, 0, sizeof(a));
  a.x = x;
  a.w_router = w->w_router;
  a.off = w->logit_offset;
  a.idx = topk_idx;
  a.count = expert_count;
  a.d_w = d_topk_w;
  a.d_logits = d_logits;
  a.T = cfg->T;
  a.d = cfg->d;
  a.E = cfg->E;
  a.k = cfg->top_k;
  a.sigmoid = cfg->score == MOE_SCORE_SIGMOID;
  a.norm = cfg->norm_topk != 0;
  a.alpha = cfg->aux_alpha;
  a.dL = d_loss;
  if (cfg->dtype == MOE_DTYPE_BF16) return route_backward_impl<__nv_bfloat16>(cfg, a, d_w_router, dx, st);
  return route_backward_impl<float>(cfg, a, d_w_router, dx, st);
}

size_t moe_backward_workspace_size(const moe_config_t *cfg) {
  if (check_cfg(cfg) != MOE_OK) return 0;
  return bwd_layout(cfg).total + 256;  // + room to start the layout on a 256-byte boundary
}

moe_status_t moe_expert_backward(const moe_config_t *cfg, const void *x_perm,
                                 const int32_t *offsets, const int32_t *slot_pos, const void *x,
                                 const moe_weights_t *w, const void *dy_perm, const float *dy,
                                 float *dx, const moe_grads_t *g, void *ws, size_t ws_bytes,
                                 void *stream) {
  MOE_TRY(check_cfg(cfg));
  if (cfg->dtype != MOE_DTYPE_BF16 || cfg->expert_storage != MOE_STORAGE_DTYPE)
    return MOE_ERR_UNSUPPORTED;
  MOE_TRY(check_weights(cfg, w, false, true));
  MOE_REQUIRE(g != nullptr);
  MOE_REQUIRE(tok16(cfg, x_perm) && aligned16(offsets) && tok16(cfg, slot_pos) && tok16(cfg, x) &&
              tok16(cfg, dy_perm) && tok16(cfg, dx));
  if (cfg->expert == MOE_EXPERT_SWIGLU)
    MOE_REQUIRE(aligned16(g->d_w_gate) && aligned16(g->d_w_up) && aligned16(g->d_w_down));
  else
    MOE_REQUIRE(aligned16(g->d_lr_V) && aligned16(g->d_lr_s) && aligned16(g->d_lr_U));
  MOE_REQUIRE(cfg->n_shared == 0 || (tok16(cfg, dy) && aligned16(g->d_ws_gate) &&
                                     aligned16(g->d_ws_up) && aligned16(g->d_ws_down)));
  MOE_REQUIRE(aligned16(ws));
  if (ws_bytes < bwd_layout(cfg).total + 256) return MOE_ERR_WORKSPACE;
  // the layout starts on a 256-byte boundary (its 32-byte stores and bulk copies need 32)
  ws = (void *)(((uintptr_t)ws + 255) & ~(uintptr_t)255);
  cudaStream_t st = (cudaStream_t)stream;
  if (cfg->T == 0) {  // no rows: every gradient is zero
    const size_t E = cfg->E, f = cfg->ffn, d = cfg->d, sf = (size_t)cfg->n_shared * cfg->ffn_shared;
    const size_t r = cfg->rank;
    if (cfg->expert == MOE_EXPERT_SWIGLU) {
      if (cudaMemsetAsync(g->d_w_gate, 0, E * f * d * 4, st) != cudaSuccess ||
          cudaMemsetAsync(g->d_w_up, 0, E * f * d * 4, st) != cudaSuccess ||
          cudaMemsetAsync(g->d_w_down, 0, E * f * d * 4, st) != cudaSuccess)
        return MOE_ERR_CUDA;
    } else if (cudaMemsetAsync(g->d_lr_V, 0, E * r * d * 4, st) != cudaSuccess ||
               cudaMemsetAsync(g->d_lr_s, 0, E * r * 4, st) != cudaSuccess ||
               cudaMemsetAsync(g->d_lr_U, 0, E * d * r * 4, st) != cudaSuccess) {
      return MOE_ERR_CUDA;
    }
    if (sf && (cudaMemsetAsync(g->d_ws_gate, 0, sf * d * 4, st) != cudaSuccess ||
               cudaMemsetAsync(g->d_ws_up, 0, sf * d * 4, st) != cudaSuccess ||
               cudaMemsetAsync(g->d_ws_down, 0, sf * d * 4, st) != cudaSuccess))
      return MOE_ERR_CUDA;
    return MOE_OK;
  }
  return expert_backward_impl(cfg, x_perm, offsets, slot_pos, x, w, dy_perm, dy, dx, g, ws, st);
}

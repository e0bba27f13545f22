"""A layer object over the C ABI: device weights, a workspace, and one forward call.

torch supplies the device memory and the stream; every step of the forward pass runs in the
CUDA library (``moe_layer_forward``). Nothing here computes any part of the layer.
"""
from __future__ import annotations

from typing import Dict, Optional

import torch

from . import binding as B

TORCH_DTYPE = {B.DTYPE["f32"]: torch.float32, B.DTYPE["bf16"]: torch.bfloat16}

# tensors in the layer's dtype vs. always-fp32 tensors
FP32_WEIGHTS = ("logit_offset", "select_bias", "lr_s")


def torch_dtype(cfg: B.MoEConfig) -> torch.dtype:
    return TORCH_DTYPE[cfg.dtype]


def y_perm_dtype(cfg: B.MoEConfig) -> torch.dtype:
    """Element type of moe_expert_forward's routed output rows (moe.h): bf16 for bf16 SwiGLU
    layers, fp32 for fp32 layers and for low-rank layers."""
    if cfg.dtype == B.DTYPE["bf16"] and cfg.expert == B.EXPERT["swiglu"]:
        return torch.bfloat16
    return torch.float32


def upload_weights(cfg: B.MoEConfig, host: Dict[str, object], device) -> Dict[str, torch.Tensor]:
    """Copy host arrays (numpy or torch, values exact in the layer dtype) to the device."""
    dt = torch_dtype(cfg)
    out = {}
    for name, _ in B.MoEWeights._fields_:
        a = host.get(name)
        if a is None:
            continue
        t = torch.as_tensor(a)
        t = t.to(torch.float32 if name in FP32_WEIGHTS else dt)
        out[name] = t.contiguous().to(device)
    return out


def quantize_lowrank_weights(cfg: B.MoEConfig, weights: Dict[str, torch.Tensor],
                             stream=None) -> Dict[str, torch.Tensor]:
    """The E4M3 rows and fp32 row scales of the low-rank experts' V [E, r, d] and U [E, d, r]
    (moe_quantize_fp8 on the device), added to a copy of `weights` under the names of
    moe_weights_t's fp8 fields."""
    E, r, d = cfg.E, cfg.rank, cfg.d
    out = dict(weights)
    for name, rows, cols in (("lr_V", E * r, d), ("lr_U", E * d, r)):
        src = weights[name]
        q = torch.empty((rows, cols), dtype=torch.uint8, device=src.device)
        sc = torch.empty(rows, dtype=torch.float32, device=src.device)
        B.moe_quantize_fp8(src, rows, cols, q, sc, stream)
        out[name + "8"] = q
        out[name + "_scale"] = sc
    return out


class MoELayer:
    """Owns the device weights and the workspace of one MoE FFN layer configuration."""

    def __init__(self, cfg: B.MoEConfig, weights: Dict[str, torch.Tensor], device=None):
        self.cfg = cfg
        self.device = torch.device(device if device is not None else "cuda")
        if cfg.expert_storage == B.STORAGE["fp8"] and "lr_V8" not in weights:
            weights = quantize_lowrank_weights(cfg, weights)
        self.weights = weights
        self.wstruct = B.make_weights(weights)
        self.ws_bytes = B.moe_workspace_size(cfg)
        if self.ws_bytes == 0:
            raise B.MoEError("moe_workspace_size", 2)
        self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device=self.device)
        self.dtype = torch_dtype(cfg)

    def forward(self, x: torch.Tensor, y: Optional[torch.Tensor] = None,
                aux: Optional[torch.Tensor] = None, expert_count: Optional[torch.Tensor] = None,
                stream=None):
        T, d = self.cfg.T, self.cfg.d
        if y is None:
            y = torch.empty((T, d), dtype=torch.float32, device=self.device)
        if aux is None:
            aux = torch.empty((), dtype=torch.float32, device=self.device)
        B.moe_layer_forward(self.cfg, x, self.wstruct, y, aux, expert_count, self.ws,
                            self.ws_bytes, stream)
        return y, aux

    def update_bias(self, expert_count: torch.Tensor, u: float, stream=None) -> None:
        """Loss-free balancing step (moe_bias_update) on this layer's selection bias, from the
        expert counts a forward call returned; the next sigmoid-scored call routes with it."""
        bias = self.weights.get("select_bias")
        if bias is None:
            raise ValueError("the layer has no select_bias weight to update")
        B.moe_bias_update(self.cfg, expert_count, bias, u, stream)

    __call__ = forward

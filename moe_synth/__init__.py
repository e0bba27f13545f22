"""Seeded synthetic inputs for the fine-grained MoE FFN layer.

This module is shared by the tests, the benchmark and the oracle's callers. It holds the
configuration table and a deterministic input generator, and nothing of the layer's own
arithmetic: no routing, no scoring, no expert evaluation.

Shapes mirror the models the source pages describe:

* "Quartz" (Vertex AGI research page, "Architecture"; quartz-micro-preview-base model card,
  "Architecture" table): hidden 1,024, 24 routed experts of FFN 640, top-6, 2 shared experts,
  load-balancing loss with weight 0.01, 4,096 tokens per step.
* Moonfrost (property table and the "stacked (32, hidden, ffn) tensors" card): hidden 896,
  32 routed experts top-3 plus 1 shared, routing under a per-expert capacity.
* Sutra-1.3B ("48 + 1 experts"): top-4 of 48 by sigmoid score with balancing through a per-expert bias,
  1 shared expert.
* dormouse ("dropless MoE", "TSCT low-rank experts"): 1,024 experts, top-2, dropless, each
  expert U·diag(s)·Vᵀ of rank 64; batch 24 × sequence 1,024.

Every tensor is drawn from one ``torch.Generator('cpu')`` seeded once, in a fixed order:
x, router weight, router offset or selection bias, then per routed expert (gate, up, down) or
(V, s, U), then per shared expert (gate, up, down). Values are drawn in fp32 and, for bf16
configurations, rounded to bf16 with round-to-nearest-even. Arrays are returned as numpy fp32
arrays whose values are exactly representable in the configuration's dtype, so both the
device path (after an exact cast) and the oracle read the same numbers.

Distribution notation: ``N(0, s)`` with a plain number ``s`` means standard deviation ``s``
(GPT-style init notation); ``N(0, 1/fan_in)`` means variance ``1/fan_in``.
"""
from __future__ import annotations

import hashlib
import math
from dataclasses import dataclass, field, replace
from typing import Dict, Optional, Tuple

import numpy as np
import torch

__all__ = ["MoEConfig", "CONFIGS", "get_config", "make_inputs", "sha256_of", "WEIGHT_NAMES"]


@dataclass(frozen=True)
class MoEConfig:
    """Problem statement of one MoE FFN layer plus the recipe of its synthetic inputs."""

    name: str
    T: int                      # tokens in the call (batch × sequence, flattened)
    d: int                      # hidden size
    E: int                      # routed experts
    top_k: int
    n_shared: int               # always-on shared experts
    ffn: int                    # routed expert FFN width (SwiGLU)
    ffn_shared: int             # shared expert FFN width
    rank: int = 0               # low-rank expert rank r
    score: str = "softmax"      # "softmax" | "sigmoid"
    expert: str = "swiglu"      # "swiglu" | "lowrank"
    dtype: str = "bf16"         # "bf16" | "f32"
    norm_topk: bool = False     # renormalise the selected weights to sum 1
    capacity_factor: float = 0.0  # <= 0 means dropless
    aux_alpha: float = 0.01
    # ---- input recipe ----
    seed: int = 0
    x_std: float = 1.0
    router_std: float = 0.02
    offset: Tuple = ()          # () | ("normal", std) | ("zipf", s)
    bias: Tuple = ()            # () | ("uniform", a)  -> U(-a, a), selection only
    lowrank_s: Tuple[float, float] = (0.5, 1.5)
    note: str = ""

    def with_(self, **kw) -> "MoEConfig":
        return replace(self, **kw)


CONFIGS: Dict[str, MoEConfig] = {
    "tiny_f32": MoEConfig(
        name="tiny_f32", T=256, d=128, E=8, top_k=2, n_shared=1, ffn=64, ffn_shared=64,
        dtype="f32", note="tiny fp32 correctness configuration"),
    "quartz": MoEConfig(
        name="quartz", T=4096, d=1024, E=24, top_k=6, n_shared=2, ffn=640, ffn_shared=640,
        offset=("normal", 0.5), note="Quartz-shaped layer, 2x2048 tokens"),
    "capacity": MoEConfig(
        name="capacity", T=16384, d=896, E=32, top_k=3, n_shared=1, ffn=1024, ffn_shared=1024,
        capacity_factor=1.25, offset=("normal", 1.0),
        note="Moonfrost-shaped capacity-routed layer, 8x2048 tokens"),
    "sigmoid": MoEConfig(
        name="sigmoid", T=32768, d=1536, E=48, top_k=4, n_shared=1, ffn=768, ffn_shared=3072,
        score="sigmoid", norm_topk=True, bias=("uniform", 0.1),
        note="Sutra-shaped sigmoid + selection-bias layer, 8x4096 tokens"),
    "lowrank": MoEConfig(
        name="lowrank", T=24576, d=1024, E=1024, top_k=2, n_shared=0, ffn=0, ffn_shared=0,
        rank=64, expert="lowrank", offset=("zipf", 1.1),
        note="dormouse-shaped 1024 rank-64 experts, 24x1024 tokens"),
}


def get_config(name: str, **overrides) -> MoEConfig:
    cfg = CONFIGS[name]
    return cfg.with_(**overrides) if overrides else cfg


WEIGHT_NAMES = ("w_router", "logit_offset", "select_bias", "w_gate", "w_up", "w_down",
                "lr_V", "lr_U", "lr_s", "ws_gate", "ws_up", "ws_down")


def _round_dtype(t: torch.Tensor, dtype: str) -> np.ndarray:
    """Round an fp32 tensor to the configuration dtype (RNE) and return exact fp32 numpy."""
    if dtype == "bf16":
        t = t.to(torch.bfloat16).to(torch.float32)
    elif dtype != "f32":
        raise ValueError(dtype)
    return t.contiguous().numpy()


def _normal(g: torch.Generator, shape, std: float) -> torch.Tensor:
    return torch.randn(*shape, generator=g, dtype=torch.float32) * np.float32(std)


def _uniform(g: torch.Generator, shape, lo: float, hi: float) -> torch.Tensor:
    u = torch.rand(*shape, generator=g, dtype=torch.float32)
    return u * np.float32(hi - lo) + np.float32(lo)


def make_inputs(cfg: MoEConfig, T: Optional[int] = None) -> Dict[str, Optional[np.ndarray]]:
    """Draw the layer's input activations and weights for ``cfg``.

    Returns a dict with ``x`` [T, d] and the weight tensors in the library's layouts:
    ``w_router`` [E, d]; ``logit_offset`` [E] fp32 or None; ``select_bias`` [E] fp32 or None;
    SwiGLU ``w_gate``/``w_up`` [E, f, d], ``w_down`` [E, d, f]; low-rank ``lr_V`` [E, r, d],
    ``lr_U`` [E, d, r], ``lr_s`` [E, r] fp32; shared ``ws_gate``/``ws_up`` [S, fs, d],
    ``ws_down`` [S, d, fs]. Absent tensors are None. ``T`` overrides the token count (the
    weights do not depend on it, but x is drawn first, so a different T shifts the stream).
    """
    T = cfg.T if T is None else T
    g = torch.Generator(device="cpu")
    g.manual_seed(cfg.seed)
    dt = cfg.dtype
    out: Dict[str, Optional[np.ndarray]] = {k: None for k in ("x",) + WEIGHT_NAMES}

    out["x"] = _round_dtype(_normal(g, (T, cfg.d), cfg.x_std), dt)
    out["w_router"] = _round_dtype(_normal(g, (cfg.E, cfg.d), cfg.router_std), dt)

    if cfg.offset:
        kind = cfg.offset[0]
        if kind == "normal":
            off = _normal(g, (cfg.E,), cfg.offset[1])
        elif kind == "zipf":
            # Zipf(s) skew: expert with popularity rank r (a seeded permutation of 1..E)
            # gets logit offset -s*ln(r), i.e. prior weight proportional to r^-s.
            ranks = torch.randperm(cfg.E, generator=g).to(torch.float64) + 1.0
            off = (-float(cfg.offset[1]) * torch.log(ranks)).to(torch.float32)
        else:
            raise ValueError(cfg.offset)
        out["logit_offset"] = off.contiguous().numpy()
    if cfg.bias:
        kind, a = cfg.bias
        assert kind == "uniform"
        out["select_bias"] = _uniform(g, (cfg.E,), -a, a).contiguous().numpy()

    E, d = cfg.E, cfg.d
    if cfg.expert == "swiglu":
        f = cfg.ffn
        wg = np.empty((E, f, d), np.float32)
        wu = np.empty((E, f, d), np.float32)
        wd = np.empty((E, d, f), np.float32)
        for e in range(E):
            wg[e] = _round_dtype(_normal(g, (f, d), 1.0 / math.sqrt(d)), dt)
            wu[e] = _round_dtype(_normal(g, (f, d), 1.0 / math.sqrt(d)), dt)
            wd[e] = _round_dtype(_normal(g, (d, f), 1.0 / math.sqrt(f)), dt)
        out["w_gate"], out["w_up"], out["w_down"] = wg, wu, wd
    elif cfg.expert == "lowrank":
        r = cfg.rank
        V = np.empty((E, r, d), np.float32)
        U = np.empty((E, d, r), np.float32)
        s = np.empty((E, r), np.float32)
        lo, hi = cfg.lowrank_s
        for e in range(E):
            V[e] = _round_dtype(_normal(g, (r, d), 1.0 / math.sqrt(d)), dt)
            s[e] = _uniform(g, (r,), lo, hi).numpy()
            U[e] = _round_dtype(_normal(g, (d, r), 1.0 / math.sqrt(d)), dt)
        out["lr_V"], out["lr_U"], out["lr_s"] = V, U, s
    else:
        raise ValueError(cfg.expert)

    S, fs = cfg.n_shared, cfg.ffn_shared
    if S > 0:
        sg = np.empty((S, fs, d), np.float32)
        su = np.empty((S, fs, d), np.float32)
        sd = np.empty((S, d, fs), np.float32)
        for s_ in range(S):
            sg[s_] = _round_dtype(_normal(g, (fs, d), 1.0 / math.sqrt(d)), dt)
            su[s_] = _round_dtype(_normal(g, (fs, d), 1.0 / math.sqrt(d)), dt)
            sd[s_] = _round_dtype(_normal(g, (d, fs), 1.0 / math.sqrt(fs)), dt)
        out["ws_gate"], out["ws_up"], out["ws_down"] = sg, su, sd
    return out


def sha256_of(inputs: Dict[str, Optional[np.ndarray]]) -> Dict[str, str]:
    """sha256 of each present array's bytes (fp32 little-endian), for reproducibility records."""
    return {k: hashlib.sha256(np.ascontiguousarray(v).tobytes()).hexdigest()
            for k, v in inputs.items() if v is not None}

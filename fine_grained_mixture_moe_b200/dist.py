"""Data-parallel replicas of the MoE layer: one process per GPU, each holding every weight and
routing its own T_local tokens, with no exchange on the data path.

The forward pass has exactly one exchange. The load-balancing loss (Quartz: architecture table,
row "Router", weight 0.01) is alpha * E * sum_i f_i P_i with f_i = count_i / (T k) and
P_i = prob_sum_i / T over the whole batch. It is bilinear in the per-expert counts and probability
sums, so per-rank losses must not be averaged: the ranks sum count[E] and prob_sum[E] over the
group (one all-reduce of 2E values) and form the loss with T = T_local * world. Capacity stays per
replica (C = ceil(cf * T_local * k / E)), so drop masks are those of T_local-token calls.
"""
from __future__ import annotations

import ctypes
from typing import Optional, Tuple

import torch
import torch.distributed as dist

# Counts travel as fp32 in the same all-reduce as the probability sums; integers below 2^24 are
# exact in fp32, so the packed form is used only while the global selection total stays below it.
_FP32_EXACT_INT = 1 << 24


def allreduce_route_stats(count: torch.Tensor, prob_sum: torch.Tensor, global_pairs: int,
                          group=None, packed: Optional[torch.Tensor] = None
                          ) -> Tuple[torch.Tensor, torch.Tensor]:
    """Sum ``count`` [E] int32 and ``prob_sum`` [E] fp32 over the ranks of ``group``.

    ``global_pairs`` = T_global * k bounds every summed count. Below 2^24 both vectors travel in
    one fp32 all-reduce of 2E values (``packed``, reused when given); otherwise the counts take a
    separate int64 all-reduce. Returns (count_global int32 [E], prob_global fp32 [E]); every rank
    receives identical values.
    """
    E = count.numel()
    if global_pairs < _FP32_EXACT_INT:
        if packed is None:
            packed = torch.empty(2 * E, dtype=torch.float32, device=count.device)
        packed[:E].copy_(count)
        packed[E:].copy_(prob_sum)
        dist.all_reduce(packed, group=group)
        return packed[:E].to(torch.int32), packed[E:]
    c64 = count.to(torch.int64)
    p = prob_sum.clone()
    dist.all_reduce(c64, group=group)
    dist.all_reduce(p, group=group)
    return c64.to(torch.int32), p


def loss_config(cfg, world: int):
    """Copy of the ctypes layer configuration with T = T_local * world, the token count the
    global loss divides by."""
    g = type(cfg)()
    ctypes.memmove(ctypes.addressof(g), ctypes.addressof(cfg), ctypes.sizeof(cfg))
    g.T = cfg.T * world
    return g


def replica_loss_grad(d_loss: float, world: int) -> float:
    """The d_loss to hand moe_route_backward on a replica whose loss is the global one.

    The call forms the loss term dq_e = d_loss alpha E count_e / (T k T) with its own T =
    T_local. The global loss has T_global = T_local * world in both places, so a replica passes
    the all-reduced counts and d_loss / world^2; the ranks then sum d_w_router (and the expert
    weight gradients) as usual for data parallelism.
    """
    return d_loss / float(world * world)


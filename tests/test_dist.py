"""Data-parallel replicas on CPU: two gloo ranks route their halves of a batch with the oracle,
exchange the per-expert statistics through the package's all-reduce, and must reproduce the
single-process load-balancing loss on the whole batch (the loss is bilinear in the global counts
and probability sums, so per-rank losses are not averaged)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from fine_grained_mixture_moe_b200 import binding as B
from fine_grained_mixture_moe_b200 import dist as D
from moe_synth import MoEConfig, make_inputs

WORLD = 2
CFG = MoEConfig(name="dp", T=2 * 96, d=64, E=8, top_k=2, n_shared=1, ffn=64, ffn_shared=64,
                offset=("normal", 0.5))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, port: int, force_int64: bool):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        c = CFG
        inp = make_inputs(c)
        Tl = c.T // WORLD
        xs = inp["x"][rank * Tl:(rank + 1) * Tl]
        r = oracle.route(xs, inp["w_router"], inp.get("logit_offset"), inp.get("select_bias"),
                         c.score, c.top_k, c.norm_topk)
        cnt = torch.as_tensor(np.asarray(r["count"], np.int32))
        prob = torch.as_tensor(np.asarray(r["prob_sum"], np.float32))
        pairs = (1 << 24) if force_int64 else c.T * c.top_k
        gcnt, gprob = D.allreduce_route_stats(cnt, prob, pairs)
        assert gcnt.dtype == torch.int32 and gprob.dtype == torch.float32
        full = oracle.route(inp["x"], inp["w_router"], inp.get("logit_offset"),
                            inp.get("select_bias"), c.score, c.top_k, c.norm_topk)
        assert np.array_equal(gcnt.numpy(), np.asarray(full["count"], np.int32))
        np.testing.assert_allclose(gprob.numpy(), full["prob_sum"], rtol=1e-6, atol=1e-6)
        loss = oracle.aux_loss(gcnt.numpy(), gprob.numpy(), c.T, c.top_k, c.aux_alpha)
        ref = oracle.aux_loss(full["count"], full["prob_sum"], c.T, c.top_k, c.aux_alpha)
        assert loss == pytest.approx(ref, rel=1e-6)
        # the mean of per-rank losses is a different number: the exchange is needed
        own = oracle.aux_loss(r["count"], r["prob_sum"], Tl, c.top_k, c.aux_alpha)
        t = torch.tensor([own], dtype=torch.float64)
        dist.all_reduce(t)
        assert abs(t.item() / WORLD - ref) > 1e-9
    finally:
        dist.destroy_process_group()


def _rank_backward(rank: int, port: int):
    """Replica backward of the router: global counts, d_loss scaled for the call's own T, then a
    sum of d_w_router over the ranks, against the single-process backward on the whole batch."""
    from oracle import moe_backward as BW
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        c = CFG
        inp = make_inputs(c)
        Tl = c.T // WORLD
        dy = np.random.default_rng(4).standard_normal((c.T, c.d))
        dL = 1.3
        full = BW.layer_backward(c, inp, dy, dL)
        mine = dict(inp, x=inp["x"][rank * Tl:(rank + 1) * Tl])
        cl = c.with_(T=Tl)
        r = oracle.route(mine["x"], inp["w_router"], inp.get("logit_offset"),
                         inp.get("select_bias"), c.score, c.top_k, c.norm_topk)
        cnt = torch.as_tensor(np.asarray(r["count"], np.int32))
        prob = torch.as_tensor(np.asarray(r["prob_sum"], np.float32))
        gcnt, _ = D.allreduce_route_stats(cnt, prob, c.T * c.top_k)
        dys = dy[rank * Tl:(rank + 1) * Tl]
        # the form the device call computes: its own T, the global counts, d_loss scaled
        g = BW.layer_backward(cl, mine, dys, D.replica_loss_grad(dL, WORLD),
                              loss_count=gcnt.numpy())
        # the same term written with the global T
        g2 = BW.layer_backward(cl, mine, dys, dL, loss_count=gcnt.numpy(), loss_T=c.T)
        np.testing.assert_allclose(g["d_logits"], g2["d_logits"], rtol=1e-12, atol=1e-15)
        dwr = torch.as_tensor(g["d_w_router"])
        dist.all_reduce(dwr)
        np.testing.assert_allclose(dwr.numpy(), full["d_w_router"], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(g["dx_router"], full["dx_router"][rank * Tl:(rank + 1) * Tl],
                                   rtol=1e-10, atol=1e-12)
        # the replica's own statistics give a different gradient: the exchange is needed
        own = BW.layer_backward(cl, mine, dys, dL)
        assert np.abs(own["d_logits"] - g["d_logits"]).max() > 1e-9
    finally:
        dist.destroy_process_group()


def test_replicas_reproduce_global_router_gradient():
    mp.spawn(_rank_backward, args=(_free_port(),), nprocs=WORLD, join=True)


@pytest.mark.parametrize("force_int64", [False, True])
def test_replicas_reproduce_global_loss(force_int64):
    mp.spawn(_rank_main, args=(_free_port(), force_int64), nprocs=WORLD, join=True)


def test_loss_config_scales_tokens():
    cfg = B.make_config(T=96, d=64, E=8, top_k=2, n_shared=1, ffn=64, ffn_shared=64)
    g = D.loss_config(cfg, 4)
    assert g.T == 384 and cfg.T == 96
    assert (g.d, g.E, g.top_k, g.ffn, g.aux_alpha) == (cfg.d, cfg.E, cfg.top_k, cfg.ffn,
                                                        cfg.aux_alpha)

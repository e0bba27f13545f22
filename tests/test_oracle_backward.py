"""Pins of the backward oracle (CPU).

The backward oracle is checked against central differences of the forward. The forward is
composed from the forward oracle's own steps (probabilities, combine weights, experts, combine,
loss), with the router logits in fp64 and the selection frozen (readings B1 and B3 of the
backward oracle). Also pinned: exact properties (one expert: the router gets no gradient;
softmax logit gradients sum to zero per token), and a planted mistake that the check must catch.
"""
import numpy as np
import pytest

from oracle import moe_backward as BW
from oracle import moe_oracle as F
from moe_synth import MoEConfig, make_inputs

H = 1e-6


def _frozen_objective(cfg, inp, sel, dy, dL):
    """J = sum(dy * y) + dL * L with the selection of `sel` held fixed; logits in fp64."""
    x = np.asarray(inp["x"], np.float64)
    T = x.shape[0]
    logits = x @ np.asarray(inp["w_router"], np.float64).T
    if inp.get("logit_offset") is not None:
        logits = logits + np.asarray(inp["logit_offset"], np.float64)[None, :]
    p = F.probabilities(logits, cfg.score)
    w = F.combine_weights(p, sel["idx"], cfg.norm_topk)
    pm = sel["perm"]
    ef = F.expert_forward(x[pm["src"]], pm["offsets"], x, inp, cfg.expert)
    y = F.combine(ef["y_perm"], ef["y_shared"] if cfg.n_shared else None, pm["slot_pos"], w)
    prob_sum = F.aux_probabilities(p, cfg.score).sum(axis=0)
    L = F.aux_loss(sel["count"], prob_sum, T, cfg.top_k, cfg.aux_alpha)
    return float(np.sum(dy * y)) + dL * L


def _selection(cfg, inp):
    fwd = F.layer_forward(cfg, inp, with_outputs=False)
    return dict(idx=fwd["route"]["idx"], count=fwd["route"]["count"], perm=fwd["perm"])


def _fd_check(cfg, inp, dy, dL, grads, names, n_entries=10, rtol=2e-5):
    sel = _selection(cfg, inp)
    rng = np.random.default_rng(7)
    for name in names:
        base = np.asarray(inp[name], np.float64)
        g = grads["dx" if name == "x" else "d_" + name]
        assert g.shape == base.shape, name
        flat = rng.choice(base.size, size=min(n_entries, base.size), replace=False)
        fd = np.empty(len(flat))
        for i, f in enumerate(flat):
            vals = []
            for sgn in (1.0, -1.0):
                pert = base.copy().reshape(-1)
                pert[f] += sgn * H
                trial = dict(inp)
                trial[name] = pert.reshape(base.shape)
                vals.append(_frozen_objective(cfg, trial, sel, dy, dL))
            fd[i] = (vals[0] - vals[1]) / (2 * H)
        got = g.reshape(-1)[flat]
        scale = max(np.abs(g).max(), np.abs(fd).max(), 1e-12)
        assert np.abs(got - fd).max() <= rtol * scale, (name, got, fd)


def _cfg(**kw):
    base = dict(name="bw", T=13, d=8, E=5, top_k=2, n_shared=1, ffn=4, ffn_shared=6,
                router_std=0.6, aux_alpha=0.3, offset=("normal", 0.5))
    base.update(kw)
    return MoEConfig(**base)


CASES = {
    "softmax_shared": _cfg(),
    "softmax_norm_drops": _cfg(norm_topk=True, capacity_factor=0.7, n_shared=0, ffn_shared=0),
    "sigmoid_bias_norm_drops": _cfg(score="sigmoid", norm_topk=True, bias=("uniform", 0.1),
                                    capacity_factor=0.8, n_shared=2),
    "sigmoid_plain": _cfg(score="sigmoid", bias=("uniform", 0.1)),
    "lowrank_norm_drops": _cfg(expert="lowrank", ffn=0, rank=3, norm_topk=True,
                               capacity_factor=0.7, n_shared=1),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_backward_matches_central_differences(name):
    cfg = CASES[name]
    inp = {k: (None if v is None else np.asarray(v, np.float64)) for k, v in make_inputs(cfg).items()}
    rng = np.random.default_rng(3)
    dy = rng.standard_normal((cfg.T, cfg.d))
    dL = 1.7
    grads = BW.layer_backward(cfg, inp, dy, dL)
    names = ["x", "w_router"]
    names += ["w_gate", "w_up", "w_down"] if cfg.expert == "swiglu" else ["lr_V", "lr_s", "lr_U"]
    if cfg.n_shared:
        names += ["ws_gate", "ws_up", "ws_down"]
    _fd_check(cfg, inp, dy, dL, grads, names)
    if cfg.capacity_factor > 0:  # the case really drops pairs
        assert (_selection(cfg, inp)["perm"]["slot_pos"] < 0).any()


def test_one_expert_gives_the_router_no_gradient():
    """E = 1, k = 1, softmax: p = 1 for every token, so J does not depend on W_r at all."""
    cfg = _cfg(E=1, top_k=1, offset=())
    inp = make_inputs(cfg)
    dy = np.random.default_rng(0).standard_normal((cfg.T, cfg.d))
    g = BW.layer_backward(cfg, inp, dy, 1.0)
    assert np.array_equal(g["d_w_router"], np.zeros_like(g["d_w_router"]))
    assert np.array_equal(g["d_logits"], np.zeros_like(g["d_logits"]))


def test_softmax_logit_gradients_sum_to_zero():
    """Adding a constant to a token's logits leaves softmax unchanged: rows of dl sum to 0."""
    cfg = CASES["softmax_shared"]
    inp = make_inputs(cfg)
    dy = np.random.default_rng(1).standard_normal((cfg.T, cfg.d))
    dl = BW.layer_backward(cfg, inp, dy, 2.0)["d_logits"]
    assert np.abs(dl.sum(axis=1)).max() <= 1e-15 * max(1.0, np.abs(dl).max()) * cfg.E


def test_planted_mistake_is_caught():
    """The difference check fails when the backward leaves out the loss term (dL = 0 there)."""
    cfg = CASES["softmax_shared"]
    inp = {k: (None if v is None else np.asarray(v, np.float64)) for k, v in make_inputs(cfg).items()}
    dy = np.random.default_rng(3).standard_normal((cfg.T, cfg.d))
    wrong = BW.layer_backward(cfg, inp, dy, 0.0)
    with pytest.raises(AssertionError):
        _fd_check(cfg, inp, dy, 1.7, wrong, ["w_router"])

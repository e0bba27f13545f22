"""Pins of the CPU oracle against brute force, closed forms, invariants and textbook reductions.

These run without a GPU. Each test is chosen so that a plausible slip in the oracle (a dropped
term, a transposed weight, a wrong softmax domain, a double rounding, an off-by-one in the
capacity) fails at least one of them.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from moe_synth import MoEConfig, get_config, make_inputs
from tests import bruteforce as bf

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def tiny(**kw):
    base = dict(name="t", T=24, d=16, E=6, top_k=2, n_shared=1, ffn=8, ffn_shared=8,
                offset=("normal", 0.5))
    base.update(kw)
    return MoEConfig(**base)


# ------------------------------------------------------------------ exact fp32 rounding
def test_rn32_dyadic_matches_ieee_conversion():
    rng = np.random.default_rng(1)
    exps = rng.integers(-160, 130, size=4000)
    vals = rng.standard_normal(4000) * np.exp2(exps.astype(np.float64))
    with np.errstate(over="ignore"):
        ref = vals.astype(np.float32)   # single rounding of an exactly known fp64 value
    for v, r in zip(vals, ref):
        m, e = math.frexp(v)
        got = oracle.rn32_dyadic(int(m * 2 ** 53), e - 53)
        assert got == float(r) or (math.isinf(got) and np.isinf(r) and np.sign(got) == np.sign(r)), v


def test_rn32_ties_to_even_and_subnormals():
    # 1 + 2^-24 is the midpoint of 1 and 1 + 2^-23: even significand (1.0) wins
    assert oracle.rn32_dyadic((1 << 24) + 1, -24) == 1.0
    # 1 + 3*2^-24 is the midpoint of 1+2^-23 and 1+2^-22: even is 1+2^-22
    assert oracle.rn32_dyadic((1 << 24) + 3, -24) == 1.0 + 2.0 ** -22
    # half of the smallest subnormal rounds to zero (even), 3/2 of it to 2 of it
    assert oracle.rn32_dyadic(1, -150) == 0.0
    assert oracle.rn32_dyadic(3, -150) == 2.0 ** -148
    # largest finite and overflow
    assert oracle.rn32_dyadic((1 << 24) - 1, 104) == float(np.finfo(np.float32).max)
    assert math.isinf(oracle.rn32_dyadic((1 << 25) - 1, 103))


def test_rn32_fraction_vs_bruteforce():
    rng = np.random.default_rng(2)
    for _ in range(400):
        num = int(rng.integers(-10 ** 12, 10 ** 12))
        den = int(rng.integers(1, 10 ** 9)) * 3
        scale = Fraction(2) ** int(rng.integers(-140, 100))
        v = Fraction(num, den) * scale
        assert oracle.rn32_fraction(v) == bf.nearest_f32(v)


# ------------------------------------------------------------------ router logits
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_router_logits_exact_random(dtype):
    cfg = tiny(dtype=dtype, T=12, d=40, E=5)
    inp = make_inputs(cfg)
    got = oracle.router_logits(inp["x"], inp["w_router"], inp["logit_offset"])
    for t in range(cfg.T):
        for e in range(cfg.E):
            ref = bf.exact_logit(inp["x"][t], inp["w_router"][e], inp["logit_offset"][e])
            assert got[t, e] == np.float32(ref)


def test_router_logits_adversarial_midpoints():
    # exact sums placed on or next to fp32 rounding boundaries; a plain fp64 dot product
    # followed by a cast rounds rows 1 and 3 the wrong way (double rounding)
    x = np.array([
        [1.0, 2.0 ** -24, 0.0],              # 1 + 2^-24: tie -> 1.0
        [1.0, 2.0 ** -24, 2.0 ** -60],       # just above the tie -> 1 + 2^-23
        [1.0, 2.0 ** -24, -2.0 ** -60],      # just below the tie -> 1.0
        [1.0, 3 * 2.0 ** -24, -2.0 ** -70],  # just below 1+3*2^-24 -> 1 + 2^-23
    ], np.float32)
    w = np.ones((1, 3), np.float32)
    got = oracle.router_logits(x, w)[:, 0]
    expect = [1.0, 1.0 + 2.0 ** -23, 1.0, 1.0 + 2.0 ** -23]
    assert [float(v) for v in got] == expect
    naive = (x.astype(np.float64) @ w.T.astype(np.float64))[:, 0].astype(np.float32)
    assert float(naive[1]) != expect[1] and float(naive[3]) != expect[3]
    for t in range(4):
        assert float(got[t]) == bf.exact_logit(x[t], w[0])


def test_router_logit_offset_enters_before_rounding():
    x = np.array([[1.0]], np.float32)
    w = np.array([[1.0]], np.float32)
    off = np.array([2.0 ** -24 + 2.0 ** -40], np.float32)  # pushes 1 just past the midpoint
    assert float(oracle.router_logits(x, w, off)[0, 0]) == 1.0 + 2.0 ** -23


# ------------------------------------------------------------------ sigmoid keys
def test_sigmoid_keys_vs_rigorous_enclosure():
    rng = np.random.default_rng(3)
    l = (rng.standard_normal((6, 7)) * 3).astype(np.float32)
    b = rng.uniform(-0.1, 0.1, 7).astype(np.float32)
    keys = oracle.selection_keys(l, "sigmoid", b)
    for t in range(6):
        for e in range(7):
            assert float(keys[t, e]) == bf.sigmoid_key(float(l[t, e]), float(b[e]))


def test_sigmoid_keys_at_and_near_boundaries():
    # l = 0: sigma = 1/2 exactly; 1/2 + 2^-25 is a tie between 0.5 and 0.5+2^-24 -> 0.5
    l = np.array([[0.0, 2.0 ** -23, 2.0 ** -23]], np.float32)
    b = np.array([2.0 ** -25, 0.0, 2.0 ** -24], np.float32)
    keys = oracle.selection_keys(l, "sigmoid", b)
    # sigma(2^-23) = 1/2 + 2^-25 - (tiny cubic term): just below the tie -> 0.5
    assert float(keys[0, 0]) == 0.5
    assert float(keys[0, 1]) == 0.5
    for e in range(3):
        assert float(keys[0, e]) == bf.sigmoid_key(float(l[0, e]), float(b[e]))


def test_softmax_keys_are_logits():
    l = np.array([[0.5, -1.25]], np.float32)
    assert np.array_equal(oracle.selection_keys(l, "softmax"), l)


# ------------------------------------------------------------------ top-k
def test_topk_ties_lower_index_and_order():
    keys = np.array([[1.0, 3.0, 3.0, 2.0, 3.0],
                     [0.0, 0.0, 0.0, 0.0, 0.0],
                     [-1.0, -0.0, 0.0, -2.0, 5.0]], np.float32)
    got = oracle.topk(keys, 3)
    assert got.tolist() == [[1, 2, 4], [0, 1, 2], [4, 1, 2]]
    rng = np.random.default_rng(4)
    keys = rng.integers(0, 4, size=(50, 9)).astype(np.float32)  # many ties
    got = oracle.topk(keys, 4)
    for t in range(50):
        assert got[t].tolist() == bf.topk_ref(keys[t], 4)


# ------------------------------------------------------------------ capacity and permutation
def test_capacity_exact():
    assert oracle.capacity(16384, 3, 32, 1.25) == 1920
    assert oracle.capacity(10, 1, 3, 1.0) == 4
    assert oracle.capacity(30, 1, 3, 1.0) == 10
    assert oracle.capacity(10, 3, 3, 0.0) is None
    assert oracle.capacity(10, 3, 3, -1.0) is None
    # the fp32 value of 1.1 is 1.10000002384..., so 1.1 * 10 is just above 11
    assert oracle.capacity(10, 3, 3, 1.1) == 12


def _check_perm_invariants(idx, E, C, pm):
    T, k = idx.shape
    count = np.bincount(idx.reshape(-1), minlength=E)
    assert count.sum() == T * k
    assert np.array_equal(pm["count"], count)
    kept = count if C is None else np.minimum(count, C)
    assert np.array_equal(pm["kept"], kept)
    assert np.array_equal(np.diff(pm["offsets"]), kept)
    sp = pm["slot_pos"]
    N = int(pm["offsets"][-1])
    used = sp[sp >= 0]
    assert len(used) == N and len(np.unique(used)) == N  # each kept pair once, bijection
    if C is None:
        assert (sp >= 0).all()
    seen = np.zeros(E, np.int64)
    for t in range(T):
        for j in range(k):
            e = idx[t, j]
            if sp[t, j] >= 0:
                assert pm["offsets"][e] <= sp[t, j] < pm["offsets"][e + 1]
                assert pm["src"][sp[t, j]] == t
            assert (sp[t, j] < 0) == (C is not None and seen[e] >= C)
            seen[e] += 1
    for e in range(E):
        rows = pm["src"][pm["offsets"][e]:pm["offsets"][e + 1]]
        assert np.all(np.diff(rows) > 0)   # ascending token order within an expert


@pytest.mark.parametrize("C", [None, 0, 1, 3, 7])
def test_permute_invariants(C):
    rng = np.random.default_rng(5)
    T, E, k = 40, 7, 3
    logits = rng.standard_normal((T, E)) + np.array([2.0, 1, 0, 0, 0, -1, -3])
    idx = oracle.topk(logits.astype(np.float32), k)
    pm = oracle.permute(idx, E, C)
    _check_perm_invariants(idx, E, C, pm)


def test_capacity_drop_order_token_order():
    idx = np.zeros((10, 1), np.int32)
    pm = oracle.permute(idx, 2, 4)
    assert pm["slot_pos"][:, 0].tolist() == [0, 1, 2, 3, -1, -1, -1, -1, -1, -1]
    assert pm["offsets"].tolist() == [0, 4, 4]


# ------------------------------------------------------------------ whole layer vs brute force
TINY_CASES = {
    "softmax_dropless": dict(),
    "softmax_norm": dict(norm_topk=True),
    "softmax_capacity": dict(capacity_factor=0.75, offset=("normal", 1.5)),
    "sigmoid_bias": dict(score="sigmoid", norm_topk=True, bias=("uniform", 0.1), offset=()),
    "two_shared": dict(n_shared=2, ffn_shared=4),
    "no_shared": dict(n_shared=0, ffn_shared=0),
    "lowrank": dict(expert="lowrank", rank=4, ffn=0, n_shared=0, ffn_shared=0,
                    offset=("zipf", 1.1), E=9),
    "f32": dict(dtype="f32", top_k=3),
}


@pytest.mark.parametrize("case", sorted(TINY_CASES))
def test_layer_matches_per_token_bruteforce(case):
    cfg = tiny(**TINY_CASES[case])
    inp = make_inputs(cfg)
    out = oracle.layer_forward(cfg, inp)
    ref = bf.layer_bruteforce(cfg, inp)
    assert np.array_equal(out["route"]["idx"], ref["idx"])
    assert np.array_equal(out["perm"]["slot_pos"] >= 0, ref["kept"])
    assert out["capacity"] == ref["C"]
    np.testing.assert_allclose(out["route"]["w"], ref["w"], rtol=1e-13, atol=1e-15)
    scale = np.sqrt(np.mean(ref["y"] ** 2))
    assert np.max(np.abs(out["y"] - ref["y"])) <= 1e-12 * scale
    assert out["aux"] == pytest.approx(ref["aux"], rel=1e-12)


def test_token_output_matches_layer():
    cfg = tiny(capacity_factor=1.0, offset=("normal", 1.0))
    inp = make_inputs(cfg)
    out = oracle.layer_forward(cfg, inp)
    r, pm = out["route"], out["perm"]
    for t in range(cfg.T):
        yt = oracle.token_output(cfg, inp, t, r["idx"][t], r["w"][t], pm["slot_pos"][t] >= 0)
        np.testing.assert_allclose(yt, out["y"][t], rtol=1e-12, atol=1e-13)


# ------------------------------------------------------------------ textbook reductions
def _t64(a):
    return torch.from_numpy(np.asarray(a, np.float64))


def test_single_expert_reduces_to_dense_swiglu():
    cfg = tiny(E=1, top_k=1, offset=())
    inp = make_inputs(cfg)
    out = oracle.layer_forward(cfg, inp)
    x = _t64(inp["x"])
    F = torch.nn.functional
    dense = F.linear(F.silu(F.linear(x, _t64(inp["w_gate"][0]))) * F.linear(x, _t64(inp["w_up"][0])),
                     _t64(inp["w_down"][0]))
    sh = F.linear(F.silu(F.linear(x, _t64(inp["ws_gate"][0]))) * F.linear(x, _t64(inp["ws_up"][0])),
                  _t64(inp["ws_down"][0]))
    assert np.allclose(out["route"]["w"], 1.0)
    np.testing.assert_allclose(out["y"], (dense + sh).numpy(), rtol=1e-11, atol=1e-12)


def test_shared_experts_equal_one_wider_expert():
    cfg = tiny(n_shared=3, ffn_shared=4)
    inp = make_inputs(cfg)
    y3 = oracle.expert_forward(inp["x"][:0], np.zeros(cfg.E + 1, np.int64), inp["x"], inp,
                               "swiglu")["y_shared"]
    wide = dict(ws_gate=inp["ws_gate"].reshape(1, 12, cfg.d), ws_up=inp["ws_up"].reshape(1, 12, cfg.d),
                ws_down=np.concatenate(list(inp["ws_down"]), axis=1)[None])
    y1 = oracle.expert_forward(inp["x"][:0], np.zeros(cfg.E + 1, np.int64), inp["x"], wide,
                               "swiglu")["y_shared"]
    np.testing.assert_allclose(y3, y1, rtol=1e-12, atol=1e-13)


def test_lowrank_unit_scale_is_u_vt():
    cfg = tiny(expert="lowrank", rank=4, ffn=0, n_shared=0, ffn_shared=0, E=3)
    inp = make_inputs(cfg)
    inp["lr_s"] = np.ones_like(inp["lr_s"])
    x = inp["x"]
    offsets = np.array([0, 10, 10, 24])
    y = oracle.expert_forward(x, offsets, x, inp, "lowrank")["y_perm"]
    for e, (a, b) in enumerate([(0, 10), (10, 10), (10, 24)]):
        ref = (_t64(x[a:b]) @ _t64(inp["lr_V"][e]).T) @ _t64(inp["lr_U"][e]).T
        np.testing.assert_allclose(y[a:b], ref.numpy(), rtol=1e-12, atol=1e-13)


def test_lowrank_linearity():
    cfg = tiny(expert="lowrank", rank=4, ffn=0, n_shared=0, ffn_shared=0, E=2)
    inp = make_inputs(cfg)
    x = inp["x"].astype(np.float64)
    offsets = np.array([0, 7, 24])
    y1 = oracle.expert_forward(x, offsets, x, inp, "lowrank")["y_perm"]
    y3 = oracle.expert_forward(3 * x, offsets, 3 * x, inp, "lowrank")["y_perm"]
    np.testing.assert_allclose(y3, 3 * y1, rtol=1e-12, atol=1e-12)


def test_norm_topk_weights_sum_to_one():
    for score in ("softmax", "sigmoid"):
        cfg = tiny(norm_topk=True, score=score, bias=("uniform", 0.1) if score == "sigmoid" else ())
        out = oracle.layer_forward(cfg, make_inputs(cfg), with_outputs=False)
        np.testing.assert_allclose(out["route"]["w"].sum(axis=1), 1.0, rtol=1e-14)


def test_token_permutation_equivariance_dropless():
    cfg = tiny()
    inp = make_inputs(cfg)
    y = oracle.layer_forward(cfg, inp)["y"]
    perm = np.random.default_rng(6).permutation(cfg.T)
    inp2 = dict(inp)
    inp2["x"] = inp["x"][perm]
    y2 = oracle.layer_forward(cfg, inp2)["y"]
    np.testing.assert_allclose(y2, y[perm], rtol=1e-12, atol=1e-13)


# ------------------------------------------------------------------ load-balancing loss
def test_aux_uniform_router_equals_alpha():
    cfg = tiny(offset=())
    inp = make_inputs(cfg)
    inp["w_router"] = np.zeros_like(inp["w_router"])
    out = oracle.layer_forward(cfg, inp, with_outputs=False)
    # all logits 0 -> p = 1/E, top-k takes experts 0..k-1 on every token:
    # f_i = 1/k for i < k, P_i = 1/E -> L = alpha * E * k * (1/k) * (1/E) = alpha
    assert out["route"]["idx"].tolist() == [[0, 1]] * cfg.T
    assert out["aux"] == pytest.approx(cfg.aux_alpha, rel=1e-14)


def test_aux_balanced_routing_equals_alpha():
    # perfectly balanced counts (f_i = 1/E) give L = alpha * sum_i P_i = alpha for any p
    count = np.full(8, 5)
    prob_sum = np.random.default_rng(7).dirichlet(np.ones(8)) * 20
    assert oracle.aux_loss(count, prob_sum, 20, 2, 0.01) == pytest.approx(0.01, rel=1e-13)


def test_aux_empty_call_is_zero():
    assert oracle.aux_loss(np.zeros(4), np.zeros(4), 0, 2, 0.01) == 0.0


# ------------------------------------------------------------------ hand-worked example
def test_worked_example():
    with open(os.path.join(GOLDEN, "worked_example.json")) as fh:
        g = json.load(fh)
    cfg = MoEConfig(name="worked", **g["config"])
    inp = {k: (None if v is None else np.array(v, np.float32)) for k, v in g["inputs"].items()}
    out = oracle.layer_forward(cfg, inp)
    assert out["route"]["idx"].tolist() == g["expect"]["idx"]
    e = math.e
    z = e * e + e + 1.0
    p_hi, p_mid, p_lo = e * e / z, e / z, 1.0 / z
    s1 = 1.0 / (1.0 + math.exp(-1.0))        # silu(1)
    sh = 0.5 * s1                            # shared expert on either token
    y_expect = [[sh + p_hi * s1 + p_mid * s1, sh + p_mid * s1],
                [sh - p_mid * s1, sh + p_hi * s1 - p_mid * s1]]
    np.testing.assert_allclose(out["route"]["w"], [[p_hi, p_mid], [p_hi, p_mid]], rtol=1e-14)
    np.testing.assert_allclose(out["y"], y_expect, rtol=1e-13, atol=1e-15)
    P = [(p_hi + p_lo) / 2, (p_lo + p_hi) / 2, p_mid]
    f = [0.25, 0.25, 0.5]
    assert out["aux"] == pytest.approx(0.01 * 3 * sum(a * b for a, b in zip(f, P)), rel=1e-13)


def test_config_table_capacity_and_shapes():
    cfg = get_config("capacity")
    assert oracle.capacity(cfg.T, cfg.top_k, cfg.E, cfg.capacity_factor) == 1920
    q = get_config("quartz")
    assert (q.d, q.E, q.top_k, q.n_shared, q.ffn) == (1024, 24, 6, 2, 640)


# ------------------------------------------------------------------ loss-free balancing
def test_bias_update_signs_and_balance():
    """Overloaded experts lose u, underloaded gain u, experts at the mean keep their bias;
    perfectly balanced counts change nothing."""
    b = np.array([0.5, 0.5, 0.5, 0.5], np.float32)
    out = oracle.bias_update(np.array([3, 1, 2, 2]), b, 0.25)
    assert out.tolist() == [0.25, 0.75, 0.5, 0.5]
    assert np.array_equal(oracle.bias_update(np.array([7, 7, 7]), b[:3], 0.1), b[:3])
    # mean 1.5 is between the counts: no expert sits on it
    assert oracle.bias_update(np.array([1, 2]), np.zeros(2, np.float32), 1.0).tolist() == [1.0, -1.0]
    # scaling every count by the same factor keeps every sign
    c = np.array([5, 0, 9, 2, 2])
    bb = np.linspace(-1, 1, 5).astype(np.float32)
    assert np.array_equal(oracle.bias_update(c, bb, 0.01), oracle.bias_update(3 * c, bb, 0.01))


def test_bias_update_rounds_once_to_nearest_even():
    """1 + 2^-24 is a midpoint between fp32 neighbours and rounds to 1 (even); 1 - 2^-24 is an
    fp32 value; a step below half an ulp leaves the bias unchanged."""
    out = oracle.bias_update(np.array([4, 0]), np.array([1.0, 1.0], np.float32), 2.0 ** -24)
    assert out[0] == np.float32(1.0 - 2.0 ** -24) and out[1] == np.float32(1.0)
    out = oracle.bias_update(np.array([0, 4]), np.array([3.0, 3.0], np.float32), 2.0 ** -30)
    assert out.tolist() == [3.0, 3.0]


def test_bias_update_matches_ieee_fp32_addition():
    """Against numpy's fp32 addition (IEEE, correctly rounded) of b and +-u, on random cases."""
    rng = np.random.default_rng(7)
    for _ in range(200):
        E = int(rng.integers(1, 40))
        c = rng.integers(0, 50, E)
        b = (rng.standard_normal(E) * 10.0 ** rng.integers(-8, 3)).astype(np.float32)
        u = np.float32(10.0 ** rng.uniform(-9, 0))
        s = np.sign(c.sum() - E * c).astype(np.float32)
        ref = b + (u * s).astype(np.float32)  # float32 + float32 in numpy: one IEEE rounding
        assert np.array_equal(oracle.bias_update(c, b, float(u)), ref)

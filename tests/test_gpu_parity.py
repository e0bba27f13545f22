"""GPU parity: every step of the CUDA path, through the C ABI, against the CPU oracle.

Integer outputs (expert indices, counts, offsets, slot positions, source tokens, the permuted
copy of x) must match bit for bit. Floating outputs must satisfy
max|y - y_oracle| / rms(y_oracle) <= 2e-2 (bf16) or 1e-4 (fp32); combine weights and the
per-expert probability sums 1e-5 relative; the load-balancing loss 1e-5 relative.
"""
import numpy as np
import pytest
import torch

import oracle
from fine_grained_mixture_moe_b200 import binding as B
from moe_synth import CONFIGS, MoEConfig, get_config, make_inputs
from tests.gpu_helpers import LayerOnGpu, np_, rel_err, rel_err_stored, tol_of

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from fine_grained_mixture_moe_b200 import build
    build.build()
    B.load()
    yield
    B.moe_debug_set(B.DEBUG_FORCE_EXACT, 0)


# Reduced-T versions of the five configurations: several M tiles per expert, several N and K
# blocks, and a ragged tail (T not a multiple of 32 or 128).
SMALL = {
    "tiny_f32": get_config("tiny_f32"),
    "quartz_s": get_config("quartz", T=515),
    "capacity_s": get_config("capacity", T=1037),
    "sigmoid_s": get_config("sigmoid", T=611),
    "lowrank_s": get_config("lowrank", T=1500, E=256),
    # the full 1,024 experts with Zipf offsets: a 1,025-group tile list (the pair kernel's
    # smaller operand ring), hundreds of empty experts and one large group
    "lowrank_E1024": get_config("lowrank", T=3000),
}

EDGE = {
    "T1": get_config("quartz", T=1),
    "T33": get_config("quartz", T=33),
    "E1k1": MoEConfig(name="E1k1", T=77, d=128, E=1, top_k=1, n_shared=1, ffn=64, ffn_shared=64),
    "k_eq_E": MoEConfig(name="kE", T=90, d=64, E=3, top_k=3, n_shared=0, ffn=128, ffn_shared=0),
    "heavy_drops": get_config("capacity", T=700, capacity_factor=0.25),
    "norm_softmax": get_config("quartz", T=200, norm_topk=True),
    "sigmoid_nobias": get_config("sigmoid", T=150, bias=()),
    "three_shared": MoEConfig(name="s3", T=160, d=256, E=8, top_k=2, n_shared=3, ffn=128,
                              ffn_shared=64, offset=("normal", 0.5)),
    "lowrank_shared": MoEConfig(name="lrs", T=300, d=256, E=16, top_k=2, n_shared=1, ffn=0,
                                ffn_shared=128, rank=64, expert="lowrank", offset=("zipf", 1.1)),
    "f32_sigmoid_cap": MoEConfig(name="f32sc", T=130, d=128, E=8, top_k=3, n_shared=1, ffn=64,
                                 ffn_shared=64, dtype="f32", score="sigmoid", norm_topk=True,
                                 bias=("uniform", 0.1), capacity_factor=0.8),
    # the fp32 configuration's low-rank path (z kept fp32 between the two split products) with a
    # shared expert, and a ragged last column tile of gate/up (ffn 192)
    "lowrank_f32_shared": MoEConfig(name="lrf32", T=210, d=128, E=8, top_k=2, n_shared=1, ffn=0,
                                    ffn_shared=192, rank=128, expert="lowrank", dtype="f32",
                                    offset=("normal", 0.5)),
    "f32_ffn192": MoEConfig(name="f32f192", T=150, d=192, E=5, top_k=2, n_shared=2, ffn=192,
                            ffn_shared=64, dtype="f32"),
    # the largest top_k, on both sides of the switch from per-pair rank selection (E <= 64) to
    # per-token warp selection
    "k8_E64": MoEConfig(name="k8e64", T=97, d=128, E=64, top_k=8, n_shared=1, ffn=64,
                        ffn_shared=64, offset=("normal", 0.5)),
    "k8_E65_sigmoid": MoEConfig(name="k8e65", T=97, d=128, E=65, top_k=8, n_shared=0, ffn=64,
                                ffn_shared=0, score="sigmoid", norm_topk=True,
                                bias=("uniform", 0.1)),
    # the first expert count of the six-experts-per-thread router tile: its second round of 48
    # experts is full, the third holds one expert
    "k8_E97": MoEConfig(name="k8e97", T=131, d=192, E=97, top_k=8, n_shared=1, ffn=64,
                        ffn_shared=64, offset=("normal", 0.5)),
    # a wide hidden size: 16 staged token rows of 8 KB in the router, K = 4096 in gate/up
    "d4096": MoEConfig(name="d4096", T=45, d=4096, E=8, top_k=2, n_shared=1, ffn=128,
                       ffn_shared=128, offset=("normal", 0.5)),
}


def check_steps(c, inp, run=None, exact_only=False):
    run = run or LayerOnGpu(c, inp)
    ref = oracle.layer_forward(c, inp, with_outputs=not exact_only)
    o = run.steps()
    r, pm = ref["route"], ref["perm"]
    T = inp["x"].shape[0]
    N = int(pm["offsets"][-1])
    # routing: bit-exact indices, weights 1e-5
    assert np.array_equal(np_(o["idx"])[:T], r["idx"]), "expert indices differ"
    np.testing.assert_allclose(np_(o["w"])[:T], r["w"], rtol=1e-5, atol=1e-7)
    assert np.array_equal(np_(o["count"]), r["count"])
    np.testing.assert_allclose(np_(o["prob"]), r["prob_sum"], rtol=1e-5, atol=1e-6)
    # permutation: bit-exact
    assert np.array_equal(np_(o["offsets"]), pm["offsets"])
    assert np.array_equal(np_(o["slot_pos"])[:T], pm["slot_pos"])
    assert np.array_equal(np_(o["src"])[:N], pm["src"])
    xp = np_(o["x_perm"])[:N]
    assert np.array_equal(xp, inp["x"][pm["src"]]), "x_perm is not an exact copy"
    if exact_only:
        return o, ref
    tol = tol_of(c)
    ef = ref["experts"]
    ydt = "bf16" if o["y_perm"].dtype == torch.bfloat16 else "f32"
    assert rel_err_stored(np_(o["y_perm"])[:N], ef["y_perm"], ydt) <= tol
    if c.n_shared:
        assert rel_err(np_(o["y_shared"])[:T], ef["y_shared"]) <= tol
    assert rel_err(np_(o["y"])[:T], ref["y"]) <= tol
    assert float(o["aux"]) == pytest.approx(ref["aux"], rel=1e-5, abs=1e-9)
    # the fused call gives bitwise the same result as the steps
    y, aux, cnt = run.layer()
    assert torch.equal(y[:T], o["y"][:T])
    assert float(aux) == float(o["aux"])
    assert torch.equal(cnt, o["count"])
    return o, ref


@pytest.mark.parametrize("name", sorted(SMALL))
def test_small_configs(name):
    c = SMALL[name]
    check_steps(c, make_inputs(c))


@pytest.mark.parametrize("name", sorted(EDGE))
def test_edge_cases(name):
    c = EDGE[name]
    check_steps(c, make_inputs(c))


@pytest.mark.parametrize("level", [1, 2])
@pytest.mark.parametrize("name", ["tiny_f32", "quartz_s", "sigmoid_s"])
def test_forced_exact_router_paths(name, level):
    """Every logit through the exact integer sum (level 1) or the floating-point expansion
    (level 2), and every sigmoid key through double-double."""
    c = SMALL[name]
    if c.T > 300:
        c = c.with_(T=300 if level == 1 else 96)
    inp = make_inputs(c)
    B.moe_debug_set(B.DEBUG_FORCE_EXACT, level)
    try:
        check_steps(c, inp, exact_only=True)
    finally:
        B.moe_debug_set(B.DEBUG_FORCE_EXACT, 0)


def test_logits_on_rounding_midpoints():
    """Exact sums on and next to fp32 rounding boundaries: a plain fp64 dot product rounded to
    fp32 would tie experts 0, 1 and 2; the exact rounding ranks expert 2 first."""
    c = MoEConfig(name="mid", T=3, d=64, E=4, top_k=3, n_shared=0, ffn=64, ffn_shared=0)
    inp = make_inputs(c)
    x = np.zeros((3, 64), np.float32)
    x[:, 0] = 1.0
    x[:, 1] = 2.0 ** -24
    x[:, 2] = 2.0 ** -60
    x[1, 2] = -2.0 ** -60
    W = np.zeros((4, 64), np.float32)
    W[0, :2] = 1.0
    W[1, 0] = 1.0
    W[2, :3] = 1.0
    W[3, 0] = 0.5
    inp["x"], inp["w_router"] = x, W
    o, ref = check_steps(c, inp, exact_only=True)
    assert ref["route"]["idx"][0].tolist() == [2, 0, 1]
    assert ref["route"]["idx"][1].tolist() == [0, 1, 2]


def test_certified_ties_round_to_even():
    """Sums exactly on fp32 midpoints with a narrow exponent span: the fp64 sum is exact, so it
    decides the tie by round-to-nearest-even without the exact pass. Expert 0 gets 1 + 2^-24
    (rounds down to 1) for token 0 and 1 + 3 2^-24 (rounds up to 1 + 2^-22) for token 1; either
    rounding the other way changes the top-2 set."""
    c = MoEConfig(name="tie", T=2, d=64, E=3, top_k=2, n_shared=0, ffn=64, ffn_shared=0)
    inp = make_inputs(c)
    x = np.zeros((2, 64), np.float32)
    x[:, 0] = 1.0
    x[0, 1] = 2.0 ** -24
    x[1, 1] = 3 * 2.0 ** -24
    x[1, 2] = 2.0 ** -22
    W = np.zeros((3, 64), np.float32)
    W[0, :2] = 1.0
    W[1, 0], W[1, 1] = 1.0, 2.0
    W[2, 0], W[2, 2] = 1.0, 1.0
    inp["x"], inp["w_router"] = x, W
    o, ref = check_steps(c, inp, exact_only=True)
    assert ref["route"]["idx"][0].tolist() == [1, 0]
    assert ref["route"]["idx"][1].tolist() == [1, 0]


def test_cancelling_sums_rounded_exactly():
    """Logits whose fp64 sums cancel below their own error bound: 1 + 2^-53 - 1 (an fp64 chain
    gives 0; the exact sum 2^-53 is decided by the integer path) and 1 + 2^-60 - 1 (an exponent
    span of 60 bits: the expansion path), against plain logits 2^-70 and 2^-100. The exact order
    of the top three is experts 0, 2, 3; rounding near the fp64 sums would put 0 and 2 last."""
    c = MoEConfig(name="cancel", T=2, d=64, E=4, top_k=3, n_shared=0, ffn=64, ffn_shared=0)
    inp = make_inputs(c)
    x = np.zeros((2, 64), np.float32)
    x[:, :3] = 1.0
    W = np.zeros((4, 64), np.float32)
    W[0, :3] = [1.0, 2.0 ** -53, -1.0]
    W[1, 0] = 2.0 ** -100
    W[2, :3] = [1.0, 2.0 ** -60, -1.0]
    W[3, 0] = 2.0 ** -70
    inp["x"], inp["w_router"] = x, W
    o, ref = check_steps(c, inp, exact_only=True)
    assert ref["route"]["idx"][0].tolist() == [0, 2, 3]
    assert ref["route"]["idx"][1].tolist() == [0, 2, 3]


@pytest.mark.parametrize("name", ["quartz", "sigmoid"])
def test_near_ties_settled_exactly(name):
    """Router rows 0 and 1 are equal except in element 0 (2^-20 against 2^-20 (1 + 2^-7)), and a
    common offset (softmax) or bias (sigmoid) puts both at the top of every token: their logits
    differ by x[t,0] 2^-27, far inside the fp32 screen's bound, so every token's order is settled
    by the exact path without forcing it. Exact sums that land in one fp32 rounding cell tie and
    go to the lower index; the others are ordered by value. Bit-exact against the oracle."""
    c = get_config(name, T=300)
    inp = make_inputs(c)
    W = inp["w_router"].copy()
    W[1] = W[0]
    W[0, 0] = 2.0 ** -20
    W[1, 0] = 2.0 ** -20 * (1.0 + 2.0 ** -7)
    inp["w_router"] = W
    if c.score == "softmax":
        off = inp["logit_offset"].copy()
        off[0] = off[1] = 8.0
        inp["logit_offset"] = off
    else:
        b = inp["select_bias"].copy()
        b[0] = b[1] = 2.0
        inp["select_bias"] = b
    o, ref = check_steps(c, inp, exact_only=True)
    idx = ref["route"]["idx"]
    assert np.array_equal(np.sort(idx[:, :2], axis=1), np.tile([0, 1], (idx.shape[0], 1)))
    assert (idx[:, 0] == 0).any() and (idx[:, 0] == 1).any()  # both orders occur


# the backward of the combine and of the router, against the backward oracle: softmax and
# sigmoid scores, norm_topk, capacity drops (heavy ones too), low-rank y_perm in fp32, fp32 layers;
# T < 2E (one token range in the router's weight gradient: T1, k8_E97) and a single expert
BACKWARD = ["tiny_f32", "quartz_s", "capacity_s", "sigmoid_s", "lowrank_s", "norm_softmax",
            "f32_sigmoid_cap", "heavy_drops", "T1", "k8_E97", "E1k1"]


@pytest.mark.parametrize("name", BACKWARD)
def test_route_and_combine_backward(name):
    from oracle import moe_backward as BW
    c = SMALL[name] if name in SMALL else EDGE[name]
    inp = make_inputs(c)
    run = LayerOnGpu(c, inp)
    o = run.steps()
    T, d, k, E = run.cfg.T, run.cfg.d, run.cfg.top_k, run.cfg.E
    dy = np.random.default_rng(11).standard_normal((T, d)).astype(np.float32)
    dL = 1.7
    ref = BW.layer_backward(c, inp, dy.astype(np.float64), dL)
    dev = run.dev
    dy_t = torch.as_tensor(dy).to(dev)
    N = int(o["offsets"][-1])

    # each step on the same inputs as the oracle's step: the combine on the forward's y_perm
    # (whose error against the oracle is the forward's own), the router on the oracle's d_w
    d_w_ref = torch.as_tensor(ref["d_w"].astype(np.float32)).to(dev)

    def backward():
        g = dict(dy_perm=torch.empty_like(o["y_perm"]),
                 d_w=torch.empty((T, k), dtype=torch.float32, device=dev),
                 d_logits=torch.empty((T, E), dtype=torch.float32, device=dev),
                 d_w_router=torch.empty((E, d), dtype=torch.float32, device=dev),
                 dx=torch.empty((T, d), dtype=torch.float32, device=dev))
        B.moe_combine_backward(run.cfg, dy_t, o["y_perm"], o["slot_pos"], o["w"], g["dy_perm"],
                               g["d_w"])
        B.moe_route_backward(run.cfg, run.x, run.ws_struct, o["idx"], o["count"], d_w_ref, dL,
                             g["d_logits"], g["d_w_router"], g["dx"])
        torch.cuda.synchronize()
        st, info = B.moe_get_device_error()
        assert st == 0, (B.status_str(st), info)
        return g

    g = backward()
    tol = tol_of(c)
    ydt = "bf16" if g["dy_perm"].dtype == torch.bfloat16 else "f32"
    assert rel_err_stored(np_(g["dy_perm"])[:N], ref["d_y_perm"], ydt) <= tol
    assert rel_err(np_(g["d_w"]), ref["d_w"]) <= tol
    assert rel_err(np_(g["d_logits"]), ref["d_logits"]) <= tol
    assert rel_err(np_(g["d_w_router"]), ref["d_w_router"]) <= tol
    assert rel_err(np_(g["dx"]), ref["dx_router"]) <= tol
    # dropped pairs get a zero weight gradient; every sum has a fixed order
    assert np.all(np_(g["d_w"])[np_(o["slot_pos"])[:T] < 0] == 0.0)
    g2 = backward()
    for key in g:
        assert torch.equal(g[key][:N] if key == "dy_perm" else g[key],
                           g2[key][:N] if key == "dy_perm" else g2[key]), key


# the backward's expert steps (moe_expert_backward): SwiGLU layers in bf16 with 0 to 3 shared
# experts, norm_topk, capacity drops (heavy ones too), one token, one expert, k = E, wide and
# narrow hidden sizes, widths that are not multiples of 256, and 97 experts (T < E: empty ones)
EXPERT_BACKWARD = ["quartz_s", "capacity_s", "sigmoid_s", "norm_softmax", "heavy_drops",
                   "three_shared", "T1", "T33", "k_eq_E", "E1k1", "k8_E97", "d4096",
                   "lowrank_s", "lowrank_shared", "lowrank_E1024"]


def _expert_grads(c, run):
    E, d, S = run.cfg.E, run.cfg.d, c.n_shared
    f, fs, r, dev = c.ffn, c.ffn_shared, c.rank, run.dev
    if c.expert == "swiglu":
        g = dict(d_w_gate=torch.empty((E, f, d), dtype=torch.float32, device=dev),
                 d_w_up=torch.empty((E, f, d), dtype=torch.float32, device=dev),
                 d_w_down=torch.empty((E, d, f), dtype=torch.float32, device=dev))
    else:
        g = dict(d_lr_V=torch.empty((E, r, d), dtype=torch.float32, device=dev),
                 d_lr_s=torch.empty((E, r), dtype=torch.float32, device=dev),
                 d_lr_U=torch.empty((E, d, r), dtype=torch.float32, device=dev))
    if S:
        g.update(d_ws_gate=torch.empty((S, fs, d), dtype=torch.float32, device=dev),
                 d_ws_up=torch.empty((S, fs, d), dtype=torch.float32, device=dev),
                 d_ws_down=torch.empty((S, d, fs), dtype=torch.float32, device=dev))
    return g


def _expert_step_reference(c, inp, dy_perm, dy):
    """The oracle's expert step on this step's own inputs: the backward oracle's per-expert
    SwiGLU backward (pinned by central differences) on the grouped rows with the device's
    dy_perm (the combine backward's output, checked against the oracle's combine step in
    test_route_and_combine_backward), the shared experts on dy, then the un-permute."""
    from oracle import moe_backward as BW
    pm = oracle.layer_forward(c, inp, with_outputs=False)["perm"]
    offs, src = pm["offsets"], pm["src"]
    N = int(offs[-1])
    x = np.asarray(inp["x"], np.float64)
    Xp = x[src]
    dYp = np.asarray(dy_perm, np.float64)[:N]
    names = (("d_w_gate", "d_w_up", "d_w_down") if c.expert == "swiglu" else
             ("d_lr_V", "d_lr_s", "d_lr_U"))
    out = {n: np.zeros(np.asarray(inp[n[2:]]).shape) for n in names}
    dXp = np.zeros((N, x.shape[1]))
    for e in range(c.E):
        a, b = int(offs[e]), int(offs[e + 1])
        if a == b:
            continue
        if c.expert == "swiglu":
            g = BW.swiglu_backward(Xp[a:b], inp["w_gate"][e], inp["w_up"][e], inp["w_down"][e],
                                   dYp[a:b])
            out["d_w_gate"][e], out["d_w_up"][e], out["d_w_down"][e] = g["dWg"], g["dWu"], g["dWd"]
        else:
            g = BW.lowrank_backward(Xp[a:b], inp["lr_V"][e], inp["lr_s"][e], inp["lr_U"][e],
                                    dYp[a:b])
            out["d_lr_V"][e], out["d_lr_s"][e], out["d_lr_U"][e] = g["dV"], g["ds"], g["dU"]
        dXp[a:b] = g["dX"]
    dx = np.zeros_like(x)
    np.add.at(dx, src, dXp)
    if c.n_shared:
        for n in ("d_ws_gate", "d_ws_up", "d_ws_down"):
            out[n] = np.zeros(np.asarray(inp[n[2:]]).shape)
        for s_ in range(c.n_shared):
            g = BW.swiglu_backward(x, inp["ws_gate"][s_], inp["ws_up"][s_], inp["ws_down"][s_],
                                   np.asarray(dy, np.float64))
            out["d_ws_gate"][s_], out["d_ws_up"][s_], out["d_ws_down"][s_] = (
                g["dWg"], g["dWu"], g["dWd"])
            dx += g["dX"]
    out["dx"] = dx
    return out


@pytest.mark.parametrize("name", EXPERT_BACKWARD)
def test_expert_backward(name):
    """moe_expert_backward against the oracle's expert step on the same inputs: dx (the
    experts' part) and every expert weight gradient within the bf16 tolerance of its rms;
    bitwise equal on a second call. Its dy_perm comes from moe_combine_backward on the forward's
    y_perm, as in a training step. (Against the whole-layer backward oracle instead, the weight
    gradients also carry dy_perm's bf16 rounding: up to 0.08 of their rms on the Quartz shape,
    a figure this step's own arithmetic does not set.)"""
    c = SMALL[name] if name in SMALL else EDGE[name]
    inp = make_inputs(c)
    run = LayerOnGpu(c, inp)
    o = run.steps()
    T, d, k = run.cfg.T, run.cfg.d, run.cfg.top_k
    dev = run.dev
    dy = np.random.default_rng(11).standard_normal((T, d)).astype(np.float32)
    dy_t = torch.as_tensor(dy).to(dev)
    dyp = torch.empty_like(o["y_perm"])
    d_w = torch.empty((T, k), dtype=torch.float32, device=dev)
    B.moe_combine_backward(run.cfg, dy_t, o["y_perm"], o["slot_pos"], o["w"], dyp, d_w)
    grads = _expert_grads(c, run)
    ws_bytes = B.moe_backward_workspace_size(run.cfg)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    dx = torch.empty((T, d), dtype=torch.float32, device=dev)

    def call():
        B.moe_expert_backward(run.cfg, o["x_perm"], o["offsets"], o["slot_pos"], run.x,
                              run.ws_struct, dyp, dy_t if c.n_shared else None, dx,
                              B.make_grads(grads), ws, ws_bytes)
        torch.cuda.synchronize()
        st, info = B.moe_get_device_error()
        assert st == 0, (B.status_str(st), info)

    call()
    ref = _expert_step_reference(c, inp, np_(dyp), dy)
    tol = tol_of(c)
    errs = {"dx": rel_err(np_(dx), ref["dx"])}
    for n, t in grads.items():
        errs[n] = rel_err(np_(t), ref[n])
    msg = f"{name}: worst max|d|/rms " + ", ".join(f"{n}={v:.2e}" for n, v in errs.items())
    print(msg)
    assert all(v <= tol for v in errs.values()), msg
    first = {n: t.clone() for n, t in grads.items()}
    dx1 = dx.clone()
    call()
    assert torch.equal(dx, dx1) and all(torch.equal(grads[n], first[n]) for n in grads)


@pytest.mark.parametrize("name", ["capacity_s", "heavy_drops"])
def test_expert_backward_never_reads_rows_past_the_kept_pairs(name):
    """Under a capacity limit x_perm and dy_perm hold rows past offsets[E] that no kernel
    writes. The weight gradients read both in place in 64-row blocks aligned to each expert's
    last row, so those rows must never be read: with NaN planted there, every output stays
    finite and within the tolerance of the oracle's expert step."""
    c = SMALL[name] if name in SMALL else EDGE[name]
    inp = make_inputs(c)
    run = LayerOnGpu(c, inp)
    o = run.steps()
    T, d, k = run.cfg.T, run.cfg.d, run.cfg.top_k
    dev = run.dev
    N = int(o["offsets"][-1])
    assert N < T * k, "the configuration drops no pair"
    dy = np.random.default_rng(13).standard_normal((T, d)).astype(np.float32)
    dy_t = torch.as_tensor(dy).to(dev)
    dyp = torch.empty_like(o["y_perm"])
    d_w = torch.empty((T, k), dtype=torch.float32, device=dev)
    B.moe_combine_backward(run.cfg, dy_t, o["y_perm"], o["slot_pos"], o["w"], dyp, d_w)
    xp = o["x_perm"].clone()
    xp[N:] = float("nan")
    dyp[N:] = float("nan")
    grads = _expert_grads(c, run)
    ws_bytes = B.moe_backward_workspace_size(run.cfg)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    dx = torch.empty((T, d), dtype=torch.float32, device=dev)
    B.moe_expert_backward(run.cfg, xp, o["offsets"], o["slot_pos"], run.x, run.ws_struct, dyp,
                          dy_t if c.n_shared else None, dx, B.make_grads(grads), ws, ws_bytes)
    torch.cuda.synchronize()
    st, info = B.moe_get_device_error()
    assert st == 0, (B.status_str(st), info)
    ref = _expert_step_reference(c, inp, np_(dyp), dy)
    tol = tol_of(c)
    outs = dict(grads, dx=dx)
    for n, t in outs.items():
        a = np_(t)
        assert np.isfinite(a).all(), n
        assert rel_err(a, ref[n]) <= tol, n


def test_expert_backward_unsupported_configurations():
    """fp32 layers are refused on the host (MOE_ERR_UNSUPPORTED)."""
    for c in (get_config("tiny_f32"), EDGE["f32_sigmoid_cap"]):
        cfg = B.make_config(T=c.T, d=c.d, E=c.E, top_k=c.top_k, n_shared=c.n_shared, ffn=c.ffn,
                            ffn_shared=c.ffn_shared, rank=c.rank, expert=c.expert, dtype=c.dtype)
        with pytest.raises(B.MoEError) as ei:
            B.moe_expert_backward(cfg, 256, 256, 256, 256, B.MoEWeights(), 256, 256, 256,
                                  B.MoEGrads(), 256, 1 << 20)
        assert ei.value.status == 2


def test_bias_update_bitwise():
    """Loss-free balancing step on the routed counts of the sigmoid configuration, then the next
    routing call with the updated bias: the bias bit-exact against the oracle, the new routing
    bit-exact as well. Balanced counts and a single expert leave the bias unchanged."""
    c = SMALL["sigmoid_s"]
    inp = make_inputs(c)
    run = LayerOnGpu(c, inp)
    o = run.steps()
    bias0 = np.asarray(inp["select_bias"], np.float32)
    for u in (1e-3, 2.0 ** -24, 0.05):
        bd = torch.tensor(bias0, device="cuda")
        B.moe_bias_update(run.cfg, o["count"], bd, u)
        assert np.array_equal(np_(bd), oracle.bias_update(np_(o["count"]), bias0, u))
    # route again with the updated bias: selections follow it exactly
    inp2 = dict(inp)
    inp2["select_bias"] = np_(bd)
    check_steps(c, inp2, exact_only=True)
    # balanced counts and E = 1: no change
    cfg = run.cfg
    flat = torch.full((c.E,), 7, dtype=torch.int32, device="cuda")
    bd = torch.tensor(bias0, device="cuda")
    B.moe_bias_update(cfg, flat, bd, 0.5)
    assert np.array_equal(np_(bd), bias0)
    one = B.make_config(T=16, d=64, E=1, top_k=1, ffn=64)
    b1 = torch.tensor([0.25], device="cuda")
    B.moe_bias_update(one, torch.tensor([16], dtype=torch.int32, device="cuda"), b1, 0.5)
    assert float(b1) == 0.25


def test_permute_without_the_copy():
    """moe_permute with x_perm = NULL computes the same offsets, slot positions and source tokens
    and copies nothing (the header allows skipping the copy)."""
    c = SMALL["capacity_s"]
    run = LayerOnGpu(c, make_inputs(c))
    o = run.steps()
    offs = torch.empty_like(o["offsets"])
    sl = torch.empty_like(o["slot_pos"])
    sr = torch.full_like(o["src"], -7)
    B.moe_permute(run.cfg, run.x, o["idx"], offs, sl, sr, None, run.ws, run.ws_bytes)
    torch.cuda.synchronize()
    N = int(o["offsets"][-1])
    assert torch.equal(offs, o["offsets"])
    assert torch.equal(sl, o["slot_pos"])
    assert torch.equal(sr[:N], o["src"][:N])


def test_empty_call():
    c = get_config("quartz", T=0)
    run = LayerOnGpu(c, make_inputs(c, T=0))
    y, aux, cnt = run.layer()
    assert float(aux) == 0.0
    assert int(cnt.abs().sum()) == 0


def test_back_to_back_calls_on_one_workspace():
    """Four layer calls queued without synchronisation on one workspace and stream, each on
    different tokens, must give exactly what each gives alone: every kernel orders its memory
    accesses after the previous one (programmatic dependent launch), including reuse of the
    workspace by the next call."""
    c = SMALL["quartz_s"]
    inp = make_inputs(c)
    run = LayerOnGpu(c, inp)
    rng = np.random.default_rng(11)
    xs = [torch.as_tensor(rng.standard_normal(inp["x"].shape).astype(np.float32)).to(run.dt)
          .contiguous().to(run.dev) for _ in range(4)]
    alone = []
    for xb in xs:
        run.x = xb
        y, aux, cnt = run.layer()
        torch.cuda.synchronize()
        alone.append((y.clone(), float(aux), cnt.clone()))
    outs = []
    for xb in xs:  # queued back to back, no host synchronisation in between
        y = torch.empty_like(alone[0][0])
        aux = torch.empty((), dtype=torch.float32, device=run.dev)
        cnt = torch.empty_like(alone[0][2])
        B.moe_layer_forward(run.cfg, xb, run.ws_struct, y, aux, cnt, run.ws, run.ws_bytes)
        outs.append((y, aux, cnt))
    torch.cuda.synchronize()
    st, info = B.moe_get_device_error()
    assert st == 0, (B.status_str(st), info)
    for (ya, aa, ca), (yb, ab, cb) in zip(alone, outs):
        assert torch.equal(ya, yb) and aa == float(ab) and torch.equal(ca, cb)


@pytest.mark.parametrize("name", ["quartz_s", "tiny_f32", "lowrank_f32_shared", "sigmoid_s"])
def test_bitwise_determinism(name):
    """Two calls on the same inputs give the same bits (bf16 and fp32 layers; the fp32 one runs
    its products on split bf16 terms)."""
    c = SMALL[name] if name in SMALL else EDGE[name]
    run = LayerOnGpu(c, make_inputs(c))
    y1, a1, _ = run.layer()
    y1 = y1.clone()
    y2, a2, _ = run.layer()
    assert torch.equal(y1, y2) and float(a1) == float(a2)


def test_in_step_stamps():
    """With MOE_DEBUG_STAMP on, one layer call leaves a positive duration for each forward kernel
    kind it launched, each within the call's own event span; with it off nothing is recorded."""
    c = SMALL["quartz_s"]
    run = LayerOnGpu(c, make_inputs(c))
    y_ref, _, _ = run.layer()
    y_ref = y_ref.clone()
    B.moe_debug_set(B.DEBUG_STAMP, 1)
    try:
        B.moe_stamp_read()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record()
        y, _, _ = run.layer()
        ev1.record()
        torch.cuda.synchronize()
        span_us = ev0.elapsed_time(ev1) * 1e3
        st = B.moe_stamp_read()
    finally:
        B.moe_debug_set(B.DEBUG_STAMP, 0)
    assert torch.equal(y, y_ref)  # stamping changes no result
    for n in ("router", "stats", "perm_scatter", "gemm_gateup", "gemm_down", "combine"):
        assert n in st and 0.0 < st[n] <= span_us, (n, st, span_us)
    run.layer()
    assert B.moe_stamp_read() == {}


def test_bounded_wait_times_out_cleanly():
    """A wait on a barrier that nothing completes ends with MOE_ERR_TIMEOUT; the context stays
    usable for the next call."""
    B.moe_get_device_error()
    B.moe_debug_set(B.DEBUG_WAIT_LIMIT_NS, 2_000_000)
    try:
        B.moe_debug_wait_timeout_probe()
        st, info = B.moe_get_device_error()
        assert st == 5 and info == 20
    finally:
        B.moe_debug_set(B.DEBUG_WAIT_LIMIT_NS, 2_000_000_000)
    c = EDGE["E1k1"]
    check_steps(c, make_inputs(c))


# ------------------------------------------------------------------ full-size configurations
@pytest.mark.parametrize("name", sorted(CONFIGS))
def test_full_size(name):
    """Every token of the full-size configuration against the oracle, element by element, in
    the launch configuration the benchmark times (moe_layer_forward, whose y must equal the
    separate steps' y bit for bit): expert indices, counts, offsets, slot positions and source
    tokens bit-exact; the combine weights and probability sums 1e-5; the grouped expert rows
    y_perm (every kept row), the shared output and y (every token) within the stated tolerance;
    the loss 1e-5. The 1,024-expert configuration reaches the 1,025-group tile list with its
    997 empty experts and one group of about 22k rows. A small sample of tokens is also checked
    against the per-token definition (oracle.token_output), which does not group the rows."""
    c = get_config(name)
    inp = make_inputs(c)
    run = LayerOnGpu(c, inp)
    o = run.steps()
    y, aux, cnt = run.layer()
    assert torch.equal(y, o["y"])
    ref = oracle.layer_forward(c, inp, with_outputs=True)
    r, pm, ef = ref["route"], ref["perm"], ref["experts"]
    assert np.array_equal(np_(o["idx"]), r["idx"])
    np.testing.assert_allclose(np_(o["w"]), r["w"], rtol=1e-5, atol=1e-7)
    assert np.array_equal(np_(o["count"]), r["count"])
    assert np.array_equal(np_(cnt), r["count"])
    np.testing.assert_allclose(np_(o["prob"]), r["prob_sum"], rtol=1e-5, atol=1e-5)
    assert np.array_equal(np_(o["offsets"]), pm["offsets"])
    assert np.array_equal(np_(o["slot_pos"]), pm["slot_pos"])
    N = int(pm["offsets"][-1])
    assert np.array_equal(np_(o["src"])[:N], pm["src"])
    assert float(o["aux"]) == pytest.approx(ref["aux"], rel=1e-5)
    assert float(aux) == float(o["aux"])
    tol = tol_of(c)
    ydt = "bf16" if o["y_perm"].dtype == torch.bfloat16 else "f32"
    errs = {"y_perm": rel_err_stored(np_(o["y_perm"])[:N], ef["y_perm"], ydt)}
    if c.n_shared:
        errs["y_shared"] = rel_err(np_(o["y_shared"]), ef["y_shared"])
    yall = np_(y)
    errs["y"] = rel_err(yall, ref["y"])
    # the per-token definition on a sample: random tokens and the 16 with the largest outputs
    rng = np.random.default_rng(123)
    sample = np.unique(np.concatenate([[0, c.T - 1], rng.choice(c.T, 30, replace=False),
                                       np.argsort(-np.abs(yall).max(axis=1))[:16]]))
    rms = float(np.sqrt(np.mean(ref["y"] ** 2)))
    errs["y_per_token"] = max(
        float(np.max(np.abs(yall[t] - oracle.token_output(c, inp, int(t), r["idx"][t], r["w"][t],
                                                            pm["slot_pos"][t] >= 0)))) / rms
        for t in sample)
    msg = f"{name}: worst max|d|/rms " + ", ".join(f"{k}={v:.3e}" for k, v in errs.items())
    print(msg)
    assert all(v <= tol for v in errs.values()), msg

"""GPU parity of the fp8 (E4M3) storage of the low-rank experts against the fp8 oracle.

The quantisation is integer output decided in fp32 on both sides: codes and scales must match
bit for bit (weights, token rows). The layer output is compared with the oracle's fp64
evaluation of the same quantised model within the bf16 bound (max |dy| / rms(y) <= 2e-2); the
only freedom is the order of the fp32 sums and, through it, an E4M3 code of z that sits on a
rounding boundary."""
import numpy as np
import pytest
import torch

from fine_grained_mixture_moe_b200 import binding as B
from moe_synth import MoEConfig, get_config, make_inputs
from oracle import moe_fp8 as F8
from oracle import moe_oracle as O
from tests.gpu_helpers import LayerOnGpu, np_, rel_err

pytestmark = pytest.mark.gpu

CASES = {
    "lr_fp8_s": get_config("lowrank", T=1500, E=256),
    "lr_fp8_E1024": get_config("lowrank", T=3000, E=1024),
    # d = 192: the V product's K ends in half a 128-element stage; rank 128: one whole stage
    "lr_fp8_r128_d192": MoEConfig(name="lf8a", T=500, d=192, E=16, top_k=2, n_shared=0, ffn=0,
                                  ffn_shared=0, rank=128, expert="lowrank", offset=("zipf", 1.1)),
    # rank 192: the U product's K is one and a half stages; shared SwiGLU experts beside
    "lr_fp8_r192_shared": MoEConfig(name="lf8b", T=300, d=256, E=16, top_k=2, n_shared=1,
                                    ffn=0, ffn_shared=128, rank=192, expert="lowrank",
                                    offset=("normal", 0.5)),
    # capacity drops (dropped pairs get no row), rank 256 (the largest tile), top-3
    "lr_fp8_cap_r256": MoEConfig(name="lf8c", T=700, d=512, E=8, top_k=3, n_shared=0, ffn=0,
                                 ffn_shared=0, rank=256, expert="lowrank", capacity_factor=0.6,
                                 offset=("normal", 1.0)),
    # one token
    "lr_fp8_T1": MoEConfig(name="lf8d", T=1, d=128, E=4, top_k=2, n_shared=0, ffn=0,
                           ffn_shared=0, rank=64, expert="lowrank"),
}


def _quantize_gpu(t: torch.Tensor, rows: int, cols: int):
    q = torch.empty((rows, cols), dtype=torch.uint8, device=t.device)
    s = torch.empty(rows, dtype=torch.float32, device=t.device)
    B.moe_quantize_fp8(t, rows, cols, q, s)
    return q, s


class Fp8Layer(LayerOnGpu):
    def __init__(self, c, inp):
        super().__init__(c, inp)
        self.cfg.expert_storage = B.STORAGE["fp8"]
        E, r, d = c.E, c.rank, c.d
        self.V8, self.sV = _quantize_gpu(self.w["lr_V"], E * r, d)
        self.U8, self.sU = _quantize_gpu(self.w["lr_U"], E * d, r)
        self.w = dict(self.w, lr_V8=self.V8, lr_V_scale=self.sV, lr_U8=self.U8,
                      lr_U_scale=self.sU)
        self.ws_struct = B.make_weights(self.w)
        self.ws_bytes = B.moe_workspace_size(self.cfg)
        self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device=self.dev)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_quantize_rows_bitexact(dtype):
    rng = np.random.default_rng(7)
    M = (rng.standard_normal((300, 272)) * np.exp(rng.uniform(-30, 30, (300, 1)))).astype(np.float32)
    M[5] = 0.0
    M[6, :] = 0.0
    M[6, 3] = -1e-38
    M[7] = np.float32(448.0) * np.sign(rng.standard_normal(272)).astype(np.float32)
    t = torch.from_numpy(M).to(torch.bfloat16 if dtype == "bf16" else torch.float32)
    ref_in = t.float().numpy()
    q, s = _quantize_gpu(t.cuda(), 300, 272)
    rq, rs = F8.quantize_rows(ref_in)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), rs.view(np.uint32))
    assert np.array_equal(q.cpu().numpy(), rq)


def test_quantize_rejects_bad_arguments():
    x = torch.zeros((4, 24), dtype=torch.bfloat16, device="cuda")
    q = torch.empty((4, 24), dtype=torch.uint8, device="cuda")
    s = torch.empty(4, dtype=torch.float32, device="cuda")
    with pytest.raises(B.MoEError):
        B.moe_quantize_fp8(x, 4, 24, q, s)  # cols not a multiple of 16


@pytest.mark.parametrize("name", sorted(CASES))
def test_fp8_lowrank_layer(name):
    c = CASES[name]
    inp = make_inputs(c)
    run = Fp8Layer(c, inp)
    ref = F8.layer_forward_fp8(c, inp)
    W8 = ref["W8"]
    # weights: codes and scales bit for bit
    assert np.array_equal(run.V8.cpu().numpy().reshape(W8["V8"].shape), W8["V8"])
    assert np.array_equal(run.U8.cpu().numpy().reshape(W8["U8"].shape), W8["U8"])
    assert np.array_equal(run.sV.cpu().numpy().reshape(W8["sV"].shape), W8["sV"])
    assert np.array_equal(run.sU.cpu().numpy().reshape(W8["sU"].shape), W8["sU"])
    # the fused layer
    y, aux, count = run.layer()
    assert np.array_equal(count.cpu().numpy(), ref["route"]["count"])
    e_layer = rel_err(np_(y), ref["y"])
    # step by step: route, permute, the expert step on the bf16 rows, combine
    o = run.steps()
    assert np.array_equal(o["idx"].cpu().numpy(), ref["route"]["idx"])
    assert np.array_equal(o["slot_pos"].cpu().numpy(), ref["perm"]["slot_pos"])
    N = int(ref["perm"]["offsets"][-1])
    e_perm = rel_err(np_(o["y_perm"])[:N], ref["y_perm"])
    e_steps = rel_err(np_(o["y"]), ref["y"])
    # both paths quantise the same rows: the fused layer and the steps agree bit for bit
    assert torch.equal(y, o["y"])
    print(f"{name}: max|dy|/rms layer {e_layer:.2e} y_perm {e_perm:.2e} steps {e_steps:.2e}")
    assert e_layer <= 2e-2 and e_perm <= 2e-2 and e_steps <= 2e-2


def test_fp8_layer_no_tokens():
    c = CASES["lr_fp8_s"]
    cfg = B.make_config(T=0, d=c.d, E=c.E, top_k=c.top_k, rank=c.rank, expert="lowrank",
                        dtype="bf16", expert_storage="fp8")
    ws_bytes = B.moe_workspace_size(cfg)
    assert ws_bytes > 0
    dev = torch.device("cuda:0")
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    w = {n: torch.zeros(16, dtype=torch.uint8, device=dev) for n in
         ("w_router", "lr_V8", "lr_U8", "lr_V_scale", "lr_U_scale", "lr_s")}
    y = torch.empty((1, c.d), dtype=torch.float32, device=dev)
    aux = torch.full((), 5.0, dtype=torch.float32, device=dev)
    cnt = torch.full((c.E,), 7, dtype=torch.int32, device=dev)
    B.moe_layer_forward(cfg, torch.empty((1, c.d), dtype=torch.bfloat16, device=dev),
                        B.make_weights(w), y, aux, cnt, ws, ws_bytes)
    torch.cuda.synchronize()
    assert float(aux) == 0.0 and int(cnt.abs().sum()) == 0


def test_fp8_layer_bitwise_determinism():
    c = CASES["lr_fp8_s"]
    run = Fp8Layer(c, make_inputs(c))
    y1, a1, _ = run.layer()
    y1 = y1.clone()
    y2, a2, _ = run.layer()
    assert torch.equal(y1, y2) and float(a1) == float(a2)

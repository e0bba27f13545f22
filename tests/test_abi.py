"""Host-side tests of the C ABI: the library loads, exports what include/moe.h declares, sizes
its workspace, computes the capacity exactly, and rejects bad arguments before touching a GPU."""
import ctypes
import os
import re

import numpy as np
import pytest

import fine_grained_mixture_moe_b200 as moe
from fine_grained_mixture_moe_b200 import binding as B
from moe_synth import CONFIGS
import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from fine_grained_mixture_moe_b200 import build
    build.build()
    return B.load()


def header_functions():
    src = open(os.path.join(ROOT, "include", "moe.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_0-9]+)\s*\(", src)))


def test_header_declares_the_six_steps():
    fns = header_functions()
    for f in ("moe_route", "moe_permute", "moe_expert_forward", "moe_combine", "moe_aux_loss",
              "moe_layer_forward"):
        assert f in fns


def test_library_exports_every_declared_symbol(lib):
    for f in header_functions():
        assert hasattr(lib, f), f
    assert sorted(B.EXPORTED) == header_functions()


def cfg_of(c, **kw):
    d = dict(T=c.T, d=c.d, E=c.E, top_k=c.top_k, n_shared=c.n_shared, ffn=c.ffn,
             ffn_shared=c.ffn_shared, rank=c.rank, score=c.score, expert=c.expert,
             dtype=c.dtype, norm_topk=c.norm_topk, capacity_factor=c.capacity_factor,
             aux_alpha=c.aux_alpha)
    d.update(kw)
    return B.make_config(**d)


def test_fp8_storage_only_for_bf16_lowrank(lib):
    """E4M3 expert storage is a rung of the low-rank experts' ladder, for bf16 layers only."""
    assert B.moe_workspace_size(cfg_of(CONFIGS["lowrank"], expert_storage="fp8")) > 0
    for name in ("quartz", "tiny_f32"):
        assert B.moe_workspace_size(cfg_of(CONFIGS[name], expert_storage="fp8")) == 0
    assert B.moe_workspace_size(cfg_of(CONFIGS["lowrank"], dtype="f32", expert_storage="fp8")) == 0
    bad = cfg_of(CONFIGS["lowrank"])
    bad.expert_storage = 7
    assert B.moe_workspace_size(bad) == 0


def test_expert_backward_refuses_fp8_storage(lib):
    cfg = cfg_of(CONFIGS["lowrank"], T=64, expert_storage="fp8")
    w = B.MoEWeights()
    g = B.MoEGrads()
    st = lib.moe_expert_backward(ctypes.byref(cfg), None, None, None, None, ctypes.byref(w), None,
                                 None, None, ctypes.byref(g), None, 0, None)
    assert st == 2  # MOE_ERR_UNSUPPORTED, before any pointer is looked at


def test_quantize_fp8_host_refusals(lib):
    # cols not a multiple of 16, a bad dtype, negative rows: refused before any device work
    assert lib.moe_quantize_fp8(None, 1, 4, 24, None, None, None) == 2
    assert lib.moe_quantize_fp8(None, 9, 4, 32, None, None, None) == 2
    assert lib.moe_quantize_fp8(None, 1, -1, 32, None, None, None) == 1
    assert lib.moe_quantize_fp8(None, 1, 0, 32, None, None, None) == B.MOE_OK
    assert lib.moe_quantize_fp8(None, 1, 4, 32, None, None, None) == 1


@pytest.mark.parametrize("name", sorted(CONFIGS))
def test_workspace_size_and_capacity(lib, name):
    c = CONFIGS[name]
    cfg = cfg_of(c)
    ws = B.moe_workspace_size(cfg)
    es = 2 if c.dtype == "bf16" else 4
    assert ws >= c.T * c.top_k * c.d * es * 2      # permuted activations and expert outputs
    cap = B.moe_capacity(cfg)
    ref = oracle.capacity(c.T, c.top_k, c.E, c.capacity_factor)
    assert cap == (-1 if ref is None else ref)


@pytest.mark.parametrize("T,k,E,cf", [(16384, 3, 32, 1.25), (10, 3, 3, 1.1), (7, 2, 5, 0.3),
                                      (1000, 8, 1024, 2.0), (3, 1, 7, 1e-6), (0, 2, 4, 1.0),
                                      (12345, 6, 24, 0.9999999), (5, 1, 1, 100.0)])
def test_capacity_matches_oracle(lib, T, k, E, cf):
    cfg = B.make_config(T=max(T, 0), d=64, E=E, top_k=min(k, E), ffn=64, capacity_factor=cf)
    assert B.moe_capacity(cfg) == oracle.capacity(T, min(k, E), E, cf)


@pytest.mark.parametrize("bad", [dict(d=100), dict(E=0), dict(E=2000), dict(top_k=9),
                                 dict(top_k=30, E=24), dict(ffn=100), dict(T=-1),
                                 dict(score=7), dict(dtype=5), dict(expert=3),
                                 dict(n_shared=1, ffn_shared=0), dict(expert="lowrank", rank=32)])
def test_unsupported_configs_are_rejected(lib, bad):
    base = dict(T=16, d=128, E=8, top_k=2, ffn=64)
    for key in ("score", "dtype", "expert"):
        if isinstance(bad.get(key), int):
            base[key] = "softmax" if key == "score" else ("bf16" if key == "dtype" else "swiglu")
    base.update({k: v for k, v in bad.items() if not isinstance(v, int) or k not in
                 ("score", "dtype", "expert")})
    cfg = B.make_config(**base)
    for key in ("score", "dtype", "expert"):
        if isinstance(bad.get(key), int):
            setattr(cfg, key, bad[key])
    assert B.moe_workspace_size(cfg) == 0
    w = B.MoEWeights()
    st = lib.moe_route(ctypes.byref(cfg), 16, ctypes.byref(w), 16, 16, 16, 16, 16, 1 << 30, None)
    assert st == 2  # MOE_ERR_UNSUPPORTED


@pytest.mark.parametrize("dtype,d_max", [("bf16", 6016), ("f32", 2624)])
def test_hidden_size_limit_of_the_router_tile(lib, dtype, d_max):
    """The router stages 16 token rows of d elements, a ring of router-row chunks and the logits
    in one CTA's shared memory (227 KB): the largest d (multiple of 64) with E = 8 is d_max, as
    the header states (about 6,000 bf16, 2,600 fp32)."""
    ok = B.make_config(T=16, d=d_max, E=8, top_k=2, ffn=64, dtype=dtype)
    too_big = B.make_config(T=16, d=d_max + 64, E=8, top_k=2, ffn=64, dtype=dtype)
    assert B.moe_workspace_size(ok) > 0
    assert B.moe_workspace_size(too_big) == 0


def test_expert_limit_falls_back_to_the_narrow_router_tile(lib):
    """From 97 experts the router keeps six experts per thread when that tile's shared memory
    fits, else three. At d = 1536 with sigmoid keys the wide tile holds up to 733 experts and the
    narrow one up to 991: every E up to 991 must be accepted, 992 refused."""
    def cfg(E):
        return B.make_config(T=16, d=1536, E=E, top_k=4, ffn=64, score="sigmoid")
    for E in (97, 733, 734, 991):
        assert B.moe_workspace_size(cfg(E)) > 0, E
    assert B.moe_workspace_size(cfg(992)) == 0


def test_bad_pointers_and_workspace_are_rejected_on_the_host(lib):
    cfg = B.make_config(T=16, d=128, E=8, top_k=2, ffn=64)
    w = B.MoEWeights()
    w.w_router = 4096
    need = B.moe_workspace_size(cfg)
    P = ctypes.byref
    # null x
    assert lib.moe_route(P(cfg), None, P(w), 16, 16, 16, 16, 16, need, None) == 1
    # misaligned output
    assert lib.moe_route(P(cfg), 16, P(w), 24, 16, 16, 16, 16, need, None) == 1
    # workspace too small
    assert lib.moe_route(P(cfg), 16, P(w), 16, 16, 16, 16, 16, need - 1, None) == 3
    # null weights struct / config
    assert lib.moe_route(P(cfg), 16, None, 16, 16, 16, 16, 16, need, None) == 1
    assert lib.moe_route(None, 16, P(w), 16, 16, 16, 16, 16, need, None) == 1
    # expert weights missing
    assert lib.moe_expert_forward(P(cfg), 16, 16, 16, P(w), 16, 16, 16, need, None) == 1
    assert lib.moe_layer_forward(P(cfg), 16, P(w), 16, None, None, 16, need, None) == 1
    assert lib.moe_combine(P(cfg), 16, 16, 16, 16, 8, None) == 1
    assert lib.moe_aux_loss(P(cfg), 16, 16, None, None) == 1
    # bias update: null counts, misaligned bias, non-finite step
    assert lib.moe_bias_update(P(cfg), None, 16, ctypes.c_float(0.1), None) == 1
    assert lib.moe_bias_update(P(cfg), 16, 20, ctypes.c_float(0.1), None) == 1
    assert lib.moe_bias_update(P(cfg), 16, 16, ctypes.c_float(float("nan")), None) == 1
    # backward: misaligned or null buffers, non-finite loss gradient
    assert lib.moe_combine_backward(P(cfg), 16, 16, 16, 16, 16, 8, None) == 1
    assert lib.moe_combine_backward(P(cfg), None, 16, 16, 16, 16, 16, None) == 1
    assert lib.moe_route_backward(P(cfg), 16, P(w), 16, 16, 16, ctypes.c_float(1.0), 16, 16,
                                  24, None) == 1
    assert lib.moe_route_backward(P(cfg), 16, P(w), 16, None, 16, ctypes.c_float(1.0), 16, 16,
                                  16, None) == 1
    assert lib.moe_route_backward(P(cfg), 16, P(w), 16, 16, 16, ctypes.c_float(float("inf")),
                                  16, 16, 16, None) == 1
    assert lib.moe_route_backward(P(cfg), 16, None, 16, 16, 16, ctypes.c_float(1.0), 16, 16, 16,
                                  None) == 1
    assert lib.moe_route_backward(None, 16, P(w), 16, 16, 16, ctypes.c_float(1.0), 16, 16, 16,
                                  None) == 1
    assert lib.moe_combine_backward(None, 16, 16, 16, 16, 16, 16, None) == 1
    # an unsupported shape is refused before any argument is touched
    bad = B.make_config(T=16, d=100, E=8, top_k=2, ffn=64)
    assert lib.moe_combine_backward(P(bad), 16, 16, 16, 16, 16, 16, None) == 2
    assert lib.moe_route_backward(P(bad), 16, P(w), 16, 16, 16, ctypes.c_float(1.0), 16, 16,
                                  16, None) == 2


def test_noalloc_route_refuses_one_token_past_its_scratch(lib):
    """moe_route_noalloc keeps its scratch (two tables of E * ceil(T/16) int32 / fp32 partials,
    each rounded up to 256 bytes) in a fixed 4 MiB array. With E = 1,024, T = 8,192 fills it
    exactly (the GPU test runs that case); T = 8,193 needs 513 rows per table and must be
    refused on the host with MOE_ERR_WORKSPACE before any device work, whatever the pointers."""
    cfg = B.make_config(T=8193, d=1024, E=1024, top_k=2, rank=64, expert="lowrank")
    w = B.MoEWeights()
    w.w_router = 256
    P = ctypes.byref
    assert lib.moe_route_noalloc(P(cfg), 256, P(w), 256, 256, 256, 256, None) == 3


def test_status_strings(lib):
    for s in range(7):
        assert B.status_str(s).startswith(B.STATUS_NAMES[s])
    assert lib.moe_status_str(99) == b"unknown moe_status_t"


def test_package_fails_loudly_without_library(tmp_path):
    with pytest.raises(RuntimeError, match="not built"):
        B._lib_saved = B._lib
        try:
            B._lib = None
            B.load(str(tmp_path / "missing.so"))
        finally:
            B._lib = B._lib_saved

"""moe_route_noalloc: the router for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc or provide a workspace, for instance a plugin inside a host
framework whose allocator owns all device memory, or a latency-critical loop that cannot take
cudaMalloc's device-wide synchronisation. For them the library routes with its scratch held in
a fixed device array of its own. These tests call that entry point through the C ABI and check
that it returns what moe_route (with a caller workspace) returns, on two calls in a row with
different inputs, so that nothing the first call leaves in the shared array leaks into the
second. The file is collected last so that a first-failure run has already run the others.
"""
import numpy as np
import pytest
import torch

from fine_grained_mixture_moe_b200 import binding as B
from moe_synth import get_config, make_inputs
from tests.gpu_helpers import LayerOnGpu, np_

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from fine_grained_mixture_moe_b200 import build
    build.build()
    B.load()


def _route_both(c):
    run = LayerOnGpu(c, make_inputs(c))
    T, k, E, dev = run.cfg.T, run.cfg.top_k, run.cfg.E, run.dev
    outs = []
    for noalloc in (False, True):
        o = dict(idx=torch.full((T, k), -7, dtype=torch.int32, device=dev),
                 w=torch.full((T, k), -7.0, dtype=torch.float32, device=dev),
                 count=torch.full((E,), -7, dtype=torch.int32, device=dev),
                 prob=torch.full((E,), -7.0, dtype=torch.float32, device=dev))
        if noalloc:
            B.moe_route_noalloc(run.cfg, run.x, run.ws_struct, o["idx"], o["w"], o["count"],
                                o["prob"])
        else:
            B.moe_route(run.cfg, run.x, run.ws_struct, o["idx"], o["w"], o["count"], o["prob"],
                        run.ws, run.ws_bytes)
        torch.cuda.synchronize()
        st, info = B.moe_get_device_error()
        assert st == 0, (B.status_str(st), info)
        outs.append({n: np_(v) for n, v in o.items()})
    return outs


def _same(ref, got):
    assert np.array_equal(got["idx"], ref["idx"])
    assert np.array_equal(got["count"], ref["count"])
    np.testing.assert_allclose(got["w"], ref["w"], rtol=1e-5, atol=1e-7)
    np.testing.assert_allclose(got["prob"], ref["prob"], rtol=1e-5, atol=1e-6)


def test_noalloc_route_matches_workspace_route_twice_in_a_row():
    # first call: Quartz-shaped softmax routing; second call: a different shape and scoring
    # (sigmoid with selection bias), reusing the same library-held scratch array
    for c in (get_config("quartz", T=1000), get_config("sigmoid", T=777)):
        ref, got = _route_both(c)
        _same(ref, got)


def test_noalloc_route_at_the_scratch_limit():
    # 1,024 experts over 8,192 tokens: two 2 MiB tables of per-CTA partials (512 CTAs x 1,024
    # experts x 4 bytes each), exactly the 4 MiB the library holds; one token more is refused
    # (host-side test in test_abi.py)
    ref, got = _route_both(get_config("lowrank", T=8192))
    _same(ref, got)


def test_noalloc_route_rejects_configurations_beyond_its_scratch():
    # the full 1,024-expert configuration (T = 24,576) needs 8 E ceil(T/16) bytes = 12 MiB
    c = get_config("lowrank")
    cfg = B.make_config(T=c.T, d=c.d, E=c.E, top_k=c.top_k, rank=c.rank, expert="lowrank")
    w = B.MoEWeights()
    w.w_router = 256
    with pytest.raises(B.MoEError) as ei:
        B.moe_route_noalloc(cfg, 256, w, 256, 256, 256, 256, stream=0)
    assert ei.value.status == 3  # MOE_ERR_WORKSPACE, nothing enqueued

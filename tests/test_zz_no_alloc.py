"""The allocation-free router entry point, afd_ffn_route_static, against afd_ffn_route.

afd_ffn_route_static serves callers that cannot allocate device memory -- an engine that owns
every device byte through its own capped pool, or the FFN service's per-layer loop, where an
allocation can synchronise the device mid-pipeline.  It keeps its scratch (the partial router
logits) in a static device array instead of a handle's workspace.  Here it is called through
the C ABI twice in a row on the same inputs (the second call reuses the array the first one
left behind) and its outputs must match the handle-based router: expert indices bit for bit,
gate weights within the tolerance of the other router tests.

This file is collected last so that a run stopping at the first failure has already run every
other test; it also passes on its own in a fresh process.
"""
import numpy as np
import pytest
import torch

import ffn_side_expert_b200 as afd
import synth
from layer_support import W_TOL, Layer

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name", ["tiny", "mid"])
def test_route_static_matches_route_twice(name):
    L = Layer(synth.CONFIGS[name])
    try:
        cfg = L.cfg
        idx_ref, w_ref = L.route()
        torch.cuda.synchronize()
        for _ in range(2):
            idx = torch.full((cfg.T, cfg.k), -7, dtype=torch.int32, device="cuda")
            w = torch.full((cfg.T, cfg.k), -7.0, dtype=torch.float32, device="cuda")
            st = afd.afd_ffn_route_static(L.h, L.dev["router_w"], L.dev.get("router_bias"), cfg.T, cfg.H,
                                          cfg.E, cfg.k, idx, w)
            assert st == afd.AFD_OK, afd.afd_ffn_strerror(st)
            torch.cuda.synchronize()
            assert torch.equal(idx, idx_ref)
            assert float((w - w_ref).abs().max()) <= W_TOL
    finally:
        L.close()


def test_route_static_with_bias_and_ragged_T():
    cfg = synth.CONFIGS["tiny"]
    bias = torch.linspace(-0.5, 0.5, cfg.E, dtype=torch.float32)
    L = Layer(cfg, bias=bias)
    try:
        T = 37
        idx_ref, w_ref = L.route(T)
        for _ in range(2):
            idx = torch.empty((T, cfg.k), dtype=torch.int32, device="cuda")
            w = torch.empty((T, cfg.k), dtype=torch.float32, device="cuda")
            st = afd.afd_ffn_route_static(L.h, L.dev["router_w"], L.dev["router_bias"], T, cfg.H, cfg.E,
                                          cfg.k, idx, w)
            assert st == afd.AFD_OK
            torch.cuda.synchronize()
            assert torch.equal(idx, idx_ref)
            assert float((w - w_ref).abs().max()) <= W_TOL
    finally:
        L.close()


def test_route_static_rejects_sizes_beyond_its_scratch():
    E = 256
    T = afd.AFD_FFN_ROUTE_STATIC_SCRATCH_FLOATS // E + 1
    st = afd.afd_ffn_route_static(0, 0, None, T, 7168, E, 8, 0, 0)
    assert st == afd.AFD_ERR_UNSUPPORTED
    assert afd.afd_ffn_route_static(0, 0, None, 4, 7168, E, 0, 0, 0) == afd.AFD_ERR_INVALID_ARG

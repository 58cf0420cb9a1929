"""The allocation-free router entry point, afd_ffn_route_static, against afd_ffn_route and the
fp64 oracle.

afd_ffn_route_static serves callers that cannot allocate device memory -- an engine that owns
every device byte through its own capped pool, or the FFN service's per-layer loop, where an
allocation can synchronise the device mid-pipeline.  It keeps its scratch (the partial router
logits) in a static device array instead of a handle's workspace.  Each case calls it through
the C ABI twice in a row on the same inputs (the second call reuses the array the first one
left behind).  Its outputs must match the handle-based router (expert indices bit for bit,
gate weights within the tolerance of the other router tests) and the oracle's routing of the
same inputs (indices bit for bit -- every input keeps the 1e-3 top-(k+1) logit margin, found
with the same router bias the call uses -- and gate weights within that tolerance).

This file is collected last so that a run stopping at the first failure has already run every
other test; it also passes on its own in a fresh process.
"""
import os
import sys

import numpy as np
import pytest
import torch

import ffn_side_expert_b200 as afd
import synth
from layer_support import W_TOL, Layer
from oracle import moe

pytestmark = pytest.mark.gpu

sys.path.insert(0, os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden"))


def _route_static_twice(h, Wr, bias, T, cfg):
    """Two calls in a row; both results (host numpy)."""
    outs = []
    for _ in range(2):
        idx = torch.full((max(T, 1), cfg.k), -7, dtype=torch.int32, device="cuda")
        w = torch.full((max(T, 1), cfg.k), -7.0, dtype=torch.float32, device="cuda")
        st = afd.afd_ffn_route_static(h, Wr, bias, T, cfg.H, cfg.E, cfg.k, idx, w)
        assert st == afd.AFD_OK, afd.afd_ffn_strerror(st)
        torch.cuda.synchronize()
        outs.append((idx[:T].cpu().numpy(), w[:T].cpu().numpy().astype(np.float64)))
    return outs


def _check_against_oracle(outs, hidden, Wr, bias, k):
    _, ridx, rw = moe.route(hidden, Wr, bias, k)
    for idx, w in outs:
        assert np.array_equal(idx, ridx)
        assert np.max(np.abs(w - rw)) <= W_TOL
        assert np.max(np.abs(w.sum(axis=1) - 1.0)) <= 1e-6


@pytest.mark.parametrize("name", ["tiny", "mid"])
def test_route_static_matches_route_and_oracle_twice(name):
    L = Layer(synth.CONFIGS[name])
    try:
        cfg = L.cfg
        idx_ref, w_ref = L.route()
        torch.cuda.synchronize()
        outs = _route_static_twice(L.h, L.dev["router_w"], L.dev.get("router_bias"), cfg.T, cfg)
        for idx, w in outs:
            assert np.array_equal(idx, idx_ref.cpu().numpy())
            assert np.max(np.abs(w - w_ref.cpu().numpy())) <= W_TOL
        _check_against_oracle(outs, L.hidden, L.Wr, L.bias, cfg.k)
    finally:
        L.close()


def test_route_static_with_bias_and_ragged_T():
    # the tiny shape with the Zipf router bias; margin redraws found with that bias
    from make_margin_redraws import find_redraws
    cfg = synth.CONFIGS["tiny"].with_(name="tiny_zipf", zipf_s=1.1, zipf_alpha=0.30)
    L = Layer(cfg, redraws=find_redraws(cfg))
    try:
        T = 37
        idx_ref, w_ref = L.route(T)
        torch.cuda.synchronize()
        outs = _route_static_twice(L.h, L.dev["router_w"], L.dev["router_bias"], T, cfg)
        for idx, w in outs:
            assert np.array_equal(idx, idx_ref.cpu().numpy())
            assert np.max(np.abs(w - w_ref.cpu().numpy())) <= W_TOL
        _check_against_oracle(outs, L.hidden[:T], L.Wr, L.bias, cfg.k)
    finally:
        L.close()


def test_route_static_narrows_its_split_to_fit_the_scratch():
    # DeepSeek-V3 router shape (T=256, H=7168, E=256, top-8): the split of H that fills the
    # SMs (19 slices of 12 x 32 columns) holds 19 x 256 x 256 partial logits, more than the
    # 2^20-float scratch, so the call narrows it to 16 slices of 14 x 32 columns.  Only the
    # router is drawn (no expert weights); the stored margin redraws of the workload apply.
    cfg = synth.CONFIGS["dsv3_256"]
    assert 19 * cfg.T * cfg.E > afd.AFD_FFN_ROUTE_STATIC_SCRATCH_FLOATS >= 16 * cfg.T * cfg.E
    hidden = synth.gen_hidden(cfg)
    Wr, bias = synth.gen_router(cfg)
    h, wr = hidden.cuda(), Wr.cuda()
    outs = _route_static_twice(h, wr, None, cfg.T, cfg)
    _check_against_oracle(outs, hidden, Wr, bias, cfg.k)
    assert np.array_equal(outs[0][0], outs[1][0]) and np.array_equal(outs[0][1], outs[1][1])


def test_route_static_rejects_sizes_beyond_its_scratch():
    E = 256
    T = afd.AFD_FFN_ROUTE_STATIC_SCRATCH_FLOATS // E + 1
    st = afd.afd_ffn_route_static(0, 0, None, T, 7168, E, 8, 0, 0)
    assert st == afd.AFD_ERR_UNSUPPORTED
    assert afd.afd_ffn_route_static(0, 0, None, 4, 7168, E, 0, 0, 0) == afd.AFD_ERR_INVALID_ARG

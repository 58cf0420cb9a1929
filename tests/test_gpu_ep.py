"""Expert parallelism through the library's kernels on one GPU (a one-rank NCCL group).

With one rank the all-to-all exchanges are local copies, so this exercises every library call
of the expert-parallel forward -- handle-free routing and dispatch, the expert block on rows
grouped by expert, the row-block moves and the external-row combine -- against the fp64 oracle.
The exchange itself over several ranks is covered on CPU ranks (test_ep_gloo.py).
"""
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist

import ffn_side_expert_b200 as afd
import synth
from ffn_side_expert_b200.ep import ExpertParallelFfn
from layer_support import BF16_TOL, FP8_TOL, Layer, rel_max_err, to64

pytestmark = pytest.mark.gpu


def _redraws(cfg):
    import sys
    sys.path.insert(0, os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden"))
    from make_margin_redraws import find_redraws
    return find_redraws(cfg)


@pytest.mark.parametrize("T", [64, 37])
def test_expert_parallel_layer_on_one_rank(T):
    cfg = synth.MoEConfig("ep", T=64, H=256, E=8, k=2, I=512, S=1, seed=30)
    L = Layer(cfg, redraws=_redraws(cfg))
    port = 29700 + (os.getpid() + T) % 1000
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1)
    ep = None
    try:
        d = L.dev
        ep = ExpertParallelFfn(H=cfg.H, E=cfg.E, k=cfg.k, I=cfg.I, T_max=cfg.T, router_w=d["router_w"],
                               local_w13=d["w13"][:cfg.E], local_w2=d["w2"][:cfg.E],
                               shared_w13=d["w13"][cfg.E], shared_w2=d["w2"][cfg.E])
        out = ep.forward(L.h[:T])
        torch.cuda.synchronize()
        assert afd.afd_ffn_rows_error() == afd.AFD_OK
        ref = L.oracle(tokens=np.arange(T))
        err = rel_max_err(to64(out), ref["out"])
        print(f"expert-parallel T={T}: max|err|/RMS = {err:.4e} (bar {BF16_TOL})")
        assert err <= BF16_TOL, err
        w = ep.last_wire
        assert w.dispatch_sent == T * cfg.k * cfg.H * 2 and w.dispatch_remote == 0   # bf16 rows, all local
        assert w.combine_sent == T * cfg.k * cfg.H * 4 and w.combine_remote == 0     # fp32 outputs back
    finally:
        if ep is not None:
            ep.close()
        dist.destroy_process_group()
        L.close()


def _ep_fp8(L, cfg):
    d = L.dev
    return ExpertParallelFfn(H=cfg.H, E=cfg.E, k=cfg.k, I=cfg.I, T_max=cfg.T, router_w=d["router_w"],
                             local_w13=d["w13"][:cfg.E], local_w2=d["w2"][:cfg.E],
                             local_w13_scale=d["w13_scale"][:cfg.E], local_w2_scale=d["w2_scale"][:cfg.E],
                             shared_w13=d["w13"][cfg.E], shared_w2=d["w2"][cfg.E],
                             shared_w13_scale=d["w13_scale"][cfg.E], shared_w2_scale=d["w2_scale"][cfg.E])


@pytest.mark.parametrize("name,T", [("ep8", 64), ("ep8", 29), ("ep8_chunked", 4500)])
def test_w8a8_expert_parallel_layer_on_one_rank(name, T):
    # W8A8 experts: rows travel as e4m3 codes + an fp32 scale per row (A/F 分离, 通信账 counts
    # the dispatch at FP8), outputs come back as bf16.  ep8_chunked: T x E = 4500 x 256 exceeds
    # the allocation-free router's scratch, so the layer routes in two chunks.
    from oracle import comm
    cfg = (synth.MoEConfig("ep8", T=64, H=256, E=8, k=2, I=512, S=1, dtype="fp8", seed=31) if name == "ep8" else
           synth.MoEConfig("ep8_chunked", T=4500, H=256, E=256, k=8, I=256, S=1, dtype="fp8", seed=32))
    assert name != "ep8_chunked" or T * cfg.E > afd.AFD_FFN_ROUTE_STATIC_SCRATCH_FLOATS
    L = Layer(cfg, redraws=_redraws(cfg))
    port = 27700 + (os.getpid() + T) % 1000
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1)
    ep = None
    try:
        ep = _ep_fp8(L, cfg)
        out = ep.forward(L.h[:T])
        torch.cuda.synchronize()
        assert afd.afd_ffn_rows_error() == afd.AFD_OK
        ref = L.oracle(tokens=np.arange(T))
        err = rel_max_err(to64(out), ref["out"])
        print(f"W8A8 expert-parallel {name} T={T}: max|err|/RMS = {err:.4e} (bar {FP8_TOL})")
        assert err <= FP8_TOL, err
        w = ep.last_wire
        account = comm.element_bytes(ref["idx"], cfg.H, 1) + comm.dispatched_rows(ref["idx"]) * 4
        assert w.dispatch_sent == T * cfg.k * (cfg.H + 4) == account and w.dispatch_remote == 0
        assert w.combine_sent == T * cfg.k * cfg.H * 2 and w.combine_remote == 0     # bf16 outputs back
    finally:
        if ep is not None:
            ep.close()
        dist.destroy_process_group()
        L.close()


def test_expert_parallel_layer_on_the_wide_tiles():
    # T*k rows per local expert block well above 32 per expert: the rank's expert handle runs the
    # large-micro-batch GEMMs (f16 activations with their row scales, computed by
    # afd_ffn_expert_rows for rows that arrive already grouped), and the shared expert too
    cfg = synth.MoEConfig("epw", T=600, H=256, E=4, k=2, I=256, S=1, seed=33)
    L = Layer(cfg, redraws=_redraws(cfg))
    port = 26700 + os.getpid() % 1000
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1)
    ep = None
    try:
        d = L.dev
        ep = ExpertParallelFfn(H=cfg.H, E=cfg.E, k=cfg.k, I=cfg.I, T_max=cfg.T, router_w=d["router_w"],
                               local_w13=d["w13"][:cfg.E], local_w2=d["w2"][:cfg.E],
                               shared_w13=d["w13"][cfg.E], shared_w2=d["w2"][cfg.E])
        out = ep.forward(L.h)
        torch.cuda.synchronize()
        assert afd.afd_ffn_rows_error() == afd.AFD_OK
        ref = L.oracle()
        err = rel_max_err(to64(out), ref["out"])
        print(f"expert-parallel wide T={cfg.T}: max|err|/RMS = {err:.4e} (bar {BF16_TOL})")
        assert err <= BF16_TOL, err
    finally:
        if ep is not None:
            ep.close()
        dist.destroy_process_group()
        L.close()

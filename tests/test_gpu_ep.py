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
from layer_support import BF16_TOL, Layer, rel_max_err, to64

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

"""GPU parity of every stage and of the fused layer against the fp64 oracle, whole tensors,
on the tiny workload (narrow GEMM tiles) and the h=4096/k=8 workload (wide GEMM tiles).

Bars: expert indices, counts, offsets, positions and sources bit-exact; gate weights within
1e-5 and summing to 1 within 1e-6; expert outputs and the layer output within
2e-2 x RMS(oracle) (bf16).  All calls go through the C ABI.
"""
import numpy as np
import pytest
import torch

import ffn_side_expert_b200 as afd
import synth
from layer_support import BF16_TOL, W_TOL, Layer, rel_max_err, to64
from oracle import moe

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", params=["tiny", "mid"])
def layer(request):
    L = Layer(synth.CONFIGS[request.param])
    yield L
    L.close()


def test_route_bit_exact(layer):
    idx, w = layer.route()
    _, ridx, rw = layer.oracle_routing()
    assert np.array_equal(idx.cpu().numpy(), ridx)
    wg = w.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(wg - rw)) <= W_TOL
    assert np.max(np.abs(wg.sum(axis=1) - 1.0)) <= 1e-6
    assert layer.mod.get_error() == 0


def test_permute_bit_exact(layer):
    _, ridx, _ = layer.oracle_routing()
    idx = torch.from_numpy(ridx).cuda()
    counts, offsets, pos, src = layer.permute(idx)
    rc, ro, rp, rs = moe.permute(ridx, layer.cfg.E)
    assert np.array_equal(counts.cpu().numpy(), rc)
    assert np.array_equal(offsets.cpu().numpy(), ro)
    assert np.array_equal(pos.cpu().numpy(), rp)
    assert np.array_equal(src.cpu().numpy(), rs)


def test_expert_outputs(layer):
    ref = layer.oracle()
    idx = torch.from_numpy(ref["idx"]).cuda()
    T, k = idx.shape
    counts, offsets, pos, src = layer.permute(idx)
    Y, Ys = layer.expert_gemm(offsets, T)
    torch.cuda.synchronize()
    p = pos.cpu().numpy()
    Yg = to64(Y)
    assert np.isfinite(Yg).all()
    want = np.zeros_like(Yg)
    want[p.ravel()] = ref["y_routed"].reshape(T * k, -1)
    assert rel_max_err(Yg, want) <= BF16_TOL
    if layer.cfg.S:
        assert rel_max_err(to64(Ys), ref["y_shared"]) <= BF16_TOL


def test_forward_and_staged_agree_with_oracle(layer):
    ref = layer.oracle()
    out = layer.forward()
    idx, w = layer.route()
    counts, offsets, pos, src = layer.permute(idx)
    layer.expert_gemm(offsets, idx.shape[0])
    staged = layer.combine(w, pos, idx.shape[0])
    torch.cuda.synchronize()
    assert layer.mod.get_error() == 0
    err = rel_max_err(to64(out), ref["out"])
    print(f"{layer.cfg.name}: max|err|/RMS = {err:.4e} (bar {BF16_TOL})")
    assert err <= BF16_TOL, err
    assert torch.equal(out, staged)                    # same kernels, same order


def test_forward_is_deterministic(layer):
    a = layer.forward().clone()
    b = layer.forward()
    assert torch.equal(a, b)


def test_forward_host_buffers(layer):
    out = layer.forward()
    hin = layer.hidden.clone().pin_memory()
    hout = torch.empty_like(hin).pin_memory()
    layer.mod.forward_host(hin, hout)
    assert torch.equal(hout, out.cpu())


def test_forward_host_batches_pipeline(layer):
    # four different micro-batches through the FFN-service loop (copies overlapped with the
    # layer on separate streams) give the same bits as one forward per batch
    T = layer.hidden.shape[0]
    g = torch.Generator().manual_seed(7)
    batches = [layer.hidden[torch.randperm(T, generator=g)].contiguous().pin_memory() for _ in range(4)]
    outs = [torch.empty_like(b).pin_memory() for b in batches]
    layer.mod.forward_host_batches(batches, outs)
    for b, o in zip(batches, outs):
        want = torch.empty((T, layer.cfg.H), dtype=torch.bfloat16, device="cuda")
        layer.mod.forward(b.cuda(), want)
        torch.cuda.synchronize()
        assert torch.equal(o, want.cpu())
    assert layer.mod.get_error() == 0


def test_cuda_graph_replay(layer):
    eager = layer.forward().clone()
    out = torch.empty_like(eager)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        layer.mod.forward(layer.h, out, stream=s)      # warm-up on the capture stream
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        layer.mod.forward(layer.h, out, stream=s)
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, eager)
    del g


def test_sparse_stage_events(layer):
    # only the boundaries around stage 5 (the expert GEMMs) are recorded; the others are NULL
    eager = layer.forward().clone()
    n = afd.AFD_FFN_NUM_STAGES + 1
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    events = [e0 if s == 5 else e1 if s == 6 else None for s in range(n)]
    layer.mod.set_stage_events(events)
    out = layer.forward()
    layer.mod.set_stage_events(None)
    torch.cuda.synchronize()
    assert e0.elapsed_time(e1) > 0.0
    assert torch.equal(out, eager)
    assert layer.mod.get_error() == 0

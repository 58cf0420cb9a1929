"""Edge cases of the GPU path: empty and ragged micro-batches, T_max, T beyond T_max,
invalid expert indices, degenerate routings (one expert, all experts, every token on the same
experts), several N tiles of one expert, the shared expert and the W8A8 path at small sizes.
Each case is compared with the fp64 oracle on the same seeded inputs."""
import numpy as np
import pytest
import torch

import ffn_side_expert_b200 as afd
import synth
from layer_support import BF16_TOL, FP8_TOL, W_TOL, Layer, rel_max_err, to64
from oracle import moe

pytestmark = pytest.mark.gpu


def _redraws(cfg, T=None):
    """Margin redraws for an ad-hoc workload, found with the oracle."""
    import os
    import sys
    sys.path.insert(0, os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden"))
    from make_margin_redraws import find_redraws
    return find_redraws(cfg, T=T)


def _check_layer(L, T, tol=BF16_TOL):
    out = L.forward(T)
    torch.cuda.synchronize()
    assert L.mod.get_error() == 0
    ref = moe.forward(L.hidden[:T], L.Wr, L.bias, L.expert_fn, L.cfg.E, L.cfg.k, L.cfg.S, fp8=L.fp8)
    idx, _ = L.route(T)
    assert np.array_equal(idx.cpu().numpy(), ref["idx"])
    err = rel_max_err(to64(out), ref["out"])
    print(f"{L.cfg.name} T={T}: max|err|/RMS = {err:.4e} (bar {tol})")
    assert err <= tol, err
    return out


@pytest.fixture(scope="module")
def tiny():
    L = Layer(synth.CONFIGS["tiny"])
    yield L
    L.close()


def test_empty_batch_is_a_no_op(tiny):
    out = torch.full((1, tiny.cfg.H), 3.0, dtype=torch.bfloat16, device="cuda")
    assert afd.afd_ffn_forward(tiny.mod.h, tiny.h, 0, out) == afd.AFD_OK
    torch.cuda.synchronize()
    assert torch.all(out == 3.0)
    assert tiny.mod.get_error() == 0


@pytest.mark.parametrize("T", [1, 2, 37, 63, 64])
def test_ragged_and_full_batches(tiny, T):
    _check_layer(tiny, T)


def test_T_beyond_T_max_fails_fast(tiny):
    out = torch.empty((65, tiny.cfg.H), dtype=torch.bfloat16, device="cuda")
    assert afd.afd_ffn_forward(tiny.mod.h, tiny.h, 65, out) == afd.AFD_ERR_T_TOO_LARGE
    assert afd.afd_ffn_forward(tiny.mod.h, tiny.h, -1, out) == afd.AFD_ERR_INVALID_ARG


def test_invalid_expert_indices_are_skipped_and_flagged(tiny):
    _, ridx, _ = tiny.oracle_routing()
    bad = ridx.copy()
    bad[3, 1] = tiny.cfg.E          # out of range
    bad[10, 0] = -5
    counts, offsets, pos, src = tiny.permute(torch.from_numpy(bad).cuda())
    torch.cuda.synchronize()
    assert tiny.mod.get_error() == afd.AFD_ERR_DEVICE_FLAG
    assert tiny.mod.get_error() == afd.AFD_OK               # cleared by the read
    rc, ro, rp, rs = moe.permute(bad, tiny.cfg.E)
    assert np.array_equal(counts.cpu().numpy(), rc)
    assert np.array_equal(offsets.cpu().numpy(), ro)
    assert np.array_equal(pos.cpu().numpy(), rp)
    assert np.array_equal(src.cpu().numpy()[:len(rs)], rs)


def test_combine_flags_positions_out_of_range(tiny):
    idx, w = tiny.route()
    counts, offsets, pos, src = tiny.permute(idx)
    tiny.expert_gemm(offsets, idx.shape[0])
    pos2 = pos.clone()
    pos2[0, 0] = 10 ** 6
    tiny.combine(w, pos2, idx.shape[0])
    torch.cuda.synchronize()
    assert tiny.mod.get_error() == afd.AFD_ERR_DEVICE_FLAG


def test_every_token_on_the_same_experts():
    # a large bias on experts 2 and 5 sends every token there: two groups of T rows, the
    # other experts empty
    cfg = synth.MoEConfig("skewed", T=64, H=256, E=8, k=2, I=512, seed=21)
    bias = np.zeros(cfg.E, dtype=np.float32)
    bias[2], bias[5] = 60.0, 40.0
    L = Layer(cfg, bias=torch.from_numpy(bias), redraws={})
    try:
        out = _check_layer(L, cfg.T)
        idx, _ = L.route()
        assert set(np.unique(idx.cpu().numpy())) == {2, 5}
    finally:
        L.close()


def test_single_expert_top1_is_dense_ffn():
    cfg = synth.MoEConfig("e1k1", T=40, H=256, E=1, k=1, I=256, seed=22)
    L = Layer(cfg, redraws={})
    try:
        out = L.forward()
        w13, w2 = moe.expert_weights_f64(L.expert_fn(0))
        dense, _ = moe.swiglu_ffn(moe._f64(L.hidden), w13, w2)
        assert rel_max_err(to64(out), dense) <= BF16_TOL
    finally:
        L.close()


def test_all_experts_selected_with_shared_expert():
    cfg = synth.MoEConfig("kE", T=48, H=256, E=4, k=4, I=128, S=1, seed=23)
    L = Layer(cfg, redraws=_redraws(cfg))
    try:
        _check_layer(L, cfg.T)
    finally:
        L.close()


@pytest.mark.parametrize("T", [600, 520])
def test_wide_tiles_with_several_n_tiles_per_expert(T):
    # T*k > 32 E selects the wide tiles: N tiles of up to 128 rows.  ~T/2 rows per expert gives
    # several N tiles with a ragged last one; the shared expert's T rows end in an 88-row tile
    # (T=600) or an 8-row one (T=520)
    cfg = synth.MoEConfig("wide", T=600, H=256, E=2, k=1, I=256, S=1, seed=24)
    L = Layer(cfg, redraws=_redraws(cfg))
    try:
        _check_layer(L, T)
    finally:
        L.close()


@pytest.mark.parametrize("dtype", ["bf16", "fp8"])
def test_wide_tiles_when_i_is_not_a_multiple_of_256(dtype):
    # I = 384 = 3 x 128: an odd number of 128-row gate/up units per N tile (wide tiles, N <= 128)
    cfg = synth.MoEConfig("wide384", T=300, H=256, E=2, k=1, I=384, S=1, dtype=dtype, seed=27)
    L = Layer(cfg, redraws=_redraws(cfg))
    try:
        _check_layer(L, cfg.T, tol=FP8_TOL if dtype == "fp8" else BF16_TOL)
    finally:
        L.close()


@pytest.mark.parametrize("T", [1500, 2100])
def test_router_tiles_around_the_size_thresholds(T):
    # T >= 1024: 128-token router GEMM tiles (T = 1500, 2100), against 64-token tiles below;
    # with H = 256 every micro-batch size keeps the reduction in one stretch of H
    cfg = synth.MoEConfig("thresholds", T=2100, H=256, E=16, k=4, I=256, S=1, seed=29)
    L = Layer(cfg, redraws=_redraws(cfg))
    try:
        _check_layer(L, T)
        idx, w = L.route(T)
        _, ridx, rw = moe.route(L.hidden[:T], L.Wr, L.bias, cfg.k)
        assert np.array_equal(idx.cpu().numpy(), ridx)
        wg = w.cpu().numpy().astype(np.float64)
        assert np.max(np.abs(wg - rw)) <= W_TOL
        assert np.max(np.abs(wg.sum(axis=1) - 1.0)) <= 1e-6
    finally:
        L.close()


@pytest.mark.parametrize("T", [40, 200])
def test_largest_top_k(T):
    # k = 32, the largest top-k the library takes: a full warp of selections per token, 1024
    # threads per CTA in the gate-weight refinement, 33 destinations per dispatched token.
    # T=40 runs the decode tiles (fused kernel), T=200 the wide ones.
    cfg = synth.MoEConfig("k32", T=200, H=256, E=64, k=32, I=256, S=1, seed=28)
    L = Layer(cfg, redraws=_redraws(cfg))
    try:
        _check_layer(L, T)
    finally:
        L.close()


@pytest.mark.parametrize("T", [64, 23])
def test_w8a8_small(T):
    cfg = synth.MoEConfig("fp8s", T=64, H=512, E=8, k=2, I=256, S=1, dtype="fp8", seed=25)
    L = Layer(cfg, redraws=_redraws(cfg))
    try:
        _check_layer(L, T, tol=FP8_TOL)
    finally:
        L.close()


def test_w8a8_wide_tiles():
    cfg = synth.MoEConfig("fp8w", T=512, H=256, E=4, k=2, I=256, S=1, dtype="fp8", seed=26)
    L = Layer(cfg, redraws=_redraws(cfg))
    try:
        _check_layer(L, cfg.T, tol=FP8_TOL)
    finally:
        L.close()


@pytest.mark.parametrize("shape", ["decode", "wide"])
def test_large_gate_preactivations(shape):
    # hidden rows scaled by 64 or 128 (exact in bf16; the logits scale exactly, so the margin redraws
    # still hold): gate pre-activations z reach |z| > 90, where e^-z overflows fp32 and silu
    # must still give z (z > 0) or -0 (z < 0), and the SwiGLU output reaches ~10^4-10^5 -- past
    # the f16 range on the wide path, which stores each row with its power-of-two scale.
    # decode: tiny (T*k <= 32 E, fused kernel, two-term bf16 act); wide: T*k > 32 E (f16 act)
    base = (synth.CONFIGS["tiny"] if shape == "decode"
            else synth.MoEConfig("wide", T=600, H=256, E=2, k=1, I=256, S=1, seed=24))
    red = synth.load_redraws("tiny") if shape == "decode" else _redraws(base)
    hidden = synth.gen_hidden(base, redraws=red) * (64 if shape == "decode" else 128)
    L = Layer(base, hidden=hidden)
    try:
        x = moe._f64(hidden)
        zmin, zmax, amax = 0.0, 0.0, 0.0
        for e in range(base.E + base.S):
            w13, _ = moe.expert_weights_f64(L.expert_fn(e))
            z = x @ w13[:base.I].T
            act = moe.silu(z) * (x @ w13[base.I:].T)
            zmin, zmax, amax = min(zmin, z.min()), max(zmax, z.max()), max(amax, np.abs(act).max())
        assert zmin < -90 and zmax > 90
        if shape == "wide":
            assert amax > 65504                              # past the f16 range
        _check_layer(L, base.T)
    finally:
        L.close()


def test_w8a8_zero_rows():
    # W8A8 rows whose amax is 0 take the scale 1 on the GPU too: token 5 is an all-zero hidden
    # row (its logits all tie at 0: experts 0 and 1, lower index first, weights 1/2), and expert 3
    # has all-zero up rows, so every SwiGLU row it produces is zero
    cfg = synth.MoEConfig("fp8s", T=64, H=512, E=8, k=2, I=256, S=1, dtype="fp8", seed=25)
    hidden = synth.gen_hidden(cfg, redraws=_redraws(cfg))
    hidden[5] = 0

    def zero_up(ex):
        ex["w13"][3, cfg.I:] = torch.zeros((cfg.I, cfg.H), dtype=torch.float32).to(torch.float8_e4m3fn)

    L = Layer(cfg, hidden=hidden, edit_experts=zero_up)
    try:
        out = _check_layer(L, cfg.T, tol=FP8_TOL)
        idx, w = L.route()
        assert idx[5].tolist() == [0, 1] and w[5].tolist() == [0.5, 0.5]
        assert (idx == 3).any()
        ref = L.oracle()
        assert np.all(ref["y_routed"][np.nonzero(ref["idx"] == 3)] == 0.0)
        assert torch.isfinite(out.float()).all()
    finally:
        L.close()


def test_wide_bf16_without_the_f16_copy_of_w2():
    # a W2 weight beyond the f16 range (1e5) leaves the handle without its f16 copy of W2, so the
    # large-micro-batch path runs the two-term bf16 down GEMM (hi and lo act planes) instead.
    # The weight sits in an act column that is exactly zero (its gate row is zero, silu(0) = 0),
    # so the outputs keep their usual range and the 2e-2 x RMS bar stays meaningful.
    cfg = synth.MoEConfig("wide", T=600, H=256, E=2, k=1, I=256, S=1, seed=24)

    def big_weight(ex):
        ex["w13"][1, 3] = 0
        ex["w2"][1, 7, 3] = 1.0e5

    L = Layer(cfg, redraws=_redraws(cfg), edit_experts=big_weight)
    try:
        assert float(L.experts["w2"][1, 7, 3]) > 65504
        _check_layer(L, cfg.T)
    finally:
        L.close()


def test_no_w2_copy_option():
    # AFD_CREATE_NO_W2_COPY: a bf16 handle for large micro-batches keeps no f16 copy of W2 (device
    # memory drops by (E+S) H I 2 bytes) and its wide path runs the two-term bf16 down GEMM
    cfg = synth.MoEConfig("wide_big", T=300, H=2048, E=2, k=1, I=8192, S=1, seed=34)   # a 100 MB copy
    L = Layer(cfg, redraws=_redraws(cfg))
    try:
        copy_bytes = (cfg.E + cfg.S) * cfg.H * cfg.I * 2
        torch.cuda.synchronize()
        free0 = torch.cuda.mem_get_info()[0]
        lean = afd.AfdFfn(T_max=cfg.T, H=cfg.H, E=cfg.E, k=cfg.k, I=cfg.I, n_shared=cfg.S, fp8=False,
                          weights=L.dev, flags=afd.AFD_CREATE_NO_W2_COPY)
        free1 = torch.cuda.mem_get_info()[0]
        full = afd.AfdFfn(T_max=cfg.T, H=cfg.H, E=cfg.E, k=cfg.k, I=cfg.I, n_shared=cfg.S, fp8=False,
                          weights=L.dev)
        free2 = torch.cuda.mem_get_info()[0]
        assert (free1 - free2) - (free0 - free1) >= copy_bytes - (4 << 20)   # the copy, within pages
        outs = []
        for mod in (lean, full):
            out = torch.empty_like(L.h)
            mod.forward(L.h, out)
            torch.cuda.synchronize()
            assert mod.get_error() == 0
            outs.append(out)
        ref = L.oracle()
        for out in outs:
            assert rel_max_err(to64(out), ref["out"]) <= BF16_TOL
        lean.close()
        full.close()
    finally:
        L.close()


def test_w8a8_row_codes_bit_exact():
    # R9 on the device: every dispatched row's e4m3 codes and fp32 scale equal the oracle's bit for
    # bit (the codes are integer decisions taken in fp32 on both sides).  Rows 0..63 put an exact
    # e4m3 tie in every element: the row maximum is 448 * 2^j, so the scale is 2^j and x / s is
    # exact, and the other values are midpoints between neighbouring e4m3 values (ties to even)
    # at every binade; the rest are N(0, 1) rows, with one all-zero row (scale 1).
    from oracle import fp8 as ofp8
    T, H, E, k = 512, 1024, 16, 4
    rng = np.random.default_rng(41)
    x = rng.standard_normal((T, H)).astype(np.float32)
    grid = np.array(sorted({float(ofp8.e4m3_round(np.float64(v))) for v in np.linspace(0.001, 448, 4000)}))
    mids = (grid[:-1] + grid[1:]) / 2
    for t in range(64):
        j = t % 16 - 8
        row = rng.choice(mids, size=H) * np.where(rng.random(H) < 0.5, -1.0, 1.0)
        row[0] = 448.0
        x[t] = (row * 2.0 ** j).astype(np.float32)
    x[100] = 0.0
    hidden32 = torch.from_numpy(x).to(torch.bfloat16)
    assert torch.equal(hidden32.float()[:64], torch.from_numpy(x[:64]))  # the ties survive bf16
    idx = torch.from_numpy(np.argsort(rng.random((T, E)), axis=1)[:, :k].astype(np.int32))
    dev = "cuda"
    hidden, idx_d = hidden32.to(dev), idx.to(dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    pos = torch.empty((T, k), dtype=torch.int32, device=dev)
    src = torch.empty(T * k, dtype=torch.int32, device=dev)
    rows = torch.empty((T * k + T, H), dtype=torch.uint8, device=dev)
    scales = torch.empty(T * k + T, dtype=torch.float32, device=dev)
    scratch = torch.empty(2 * ((T + 127) // 128) * E, dtype=torch.int32, device=dev)
    st = afd.afd_ffn_dispatch_rows_fp8(hidden, idx_d, T, k, E, H, 1, counts, offsets, pos, src, rows, scales, scratch)
    assert st == afd.AFD_OK
    assert afd.afd_ffn_rows_error() == afd.AFD_OK
    q, s = ofp8.quantize_rows(hidden32.float().numpy())
    codes = ofp8.e4m3_encode(q)
    src_h = src.cpu().numpy().astype(np.int64)
    tok = np.concatenate([src_h, np.arange(T)])            # routed rows, then every token once
    got_codes, got_scales = rows.cpu().numpy(), scales.cpu().numpy()
    assert np.array_equal(got_scales.view(np.uint32), s[tok].view(np.uint32))
    bad = np.argwhere(got_codes != codes[tok])
    assert bad.size == 0, f"{len(bad)} codes differ, first at row {bad[0][0]} column {bad[0][1]}"

"""Pins of the oracle's expert FFN, shared expert and combine (CPU only).

Each expert is a large matrix multiplication (A/F 分离, 为什么要拆); outputs are combined
back per token (same page, 机制).  The SwiGLU form, the shared expert and the weighted
combine are this library's reading of the layer; the pins below tie each to numbers derived
by hand from closed forms, to textbook special cases and to brute force.
"""
import math

import numpy as np
import pytest

import synth
from oracle import moe

# textbook values of the logistic function sigma(z) = 1 / (1 + e^-z)
SIG_1 = 0.7310585786300049
SIG_M1 = 0.2689414213699951
SIG_M2 = 0.11920292202211755


def test_silu_closed_forms():
    assert moe.silu(0.0) == 0.0
    assert moe.silu(1.0) == pytest.approx(SIG_1, rel=1e-15)
    assert moe.silu(-1.0) == pytest.approx(-SIG_M1, rel=1e-15)
    assert moe.silu(50.0) == pytest.approx(50.0, rel=1e-15)        # z -> +inf: z
    assert abs(moe.silu(-50.0)) < 1e-19                             # z -> -inf: 0
    assert moe.silu(-1000.0) == 0.0                                 # no overflow error
    z = np.linspace(-6, 6, 101)
    assert np.allclose(moe.silu(z) - moe.silu(-z), z, atol=1e-14)  # silu(z) - silu(-z) = z


def test_swiglu_worked_example():
    # H = 2, I = 3.  x = (1, -2)
    # gate rows (1,0), (0,1), (1,1)  -> g = (1, -2, -1)
    # up rows   (2,0), (1,1), (0,-1) -> u = (2, -1, 2)
    # act = silu(g) * u = (1*s(1)*2, -2*s(-2)*(-1), -1*s(-1)*2)
    #     = (1.4621171572600098, 0.2384058440442351, -0.5378828427399902)
    # down rows (1,0,2), (0,-1,1): y = (act0 + 2 act2, -act1 + act2)
    x = np.array([[1.0, -2.0]])
    w13 = np.array([[1, 0], [0, 1], [1, 1], [2, 0], [1, 1], [0, -1]], dtype=np.float64)
    w2 = np.array([[1, 0, 2], [0, -1, 1]], dtype=np.float64)
    y, act = moe.swiglu_ffn(x, w13, w2)
    act_hand = [2 * SIG_1, 2 * SIG_M2, -2 * SIG_M1]
    y_hand = [act_hand[0] + 2 * act_hand[2], -act_hand[1] + act_hand[2]]
    assert np.allclose(act[0], act_hand, rtol=0, atol=1e-15)
    assert np.allclose(y[0], y_hand, rtol=0, atol=1e-15)
    assert y[0, 0] == pytest.approx(0.3863514717800294, abs=1e-15)
    assert y[0, 1] == pytest.approx(-0.7762886867842253, abs=1e-15)


def _tiny_layer(cfg):
    h = synth.gen_hidden(cfg)
    Wr, bias = synth.gen_router(cfg)
    experts = {e: synth.gen_expert(cfg, e) for e in range(cfg.E + cfg.S)}
    return h, Wr, bias, experts


def test_single_expert_top1_is_dense_ffn():
    # E = 1, k = 1: routing selects expert 0 with weight 1 for every token, so the layer is
    # the dense SwiGLU FFN of that expert
    cfg = synth.MoEConfig("e1k1", T=20, H=64, E=1, k=1, I=128, seed=5)
    h, Wr, bias, ex = _tiny_layer(cfg)
    res = moe.forward(h, Wr, bias, ex.__getitem__, cfg.E, cfg.k, 0)
    assert np.all(res["idx"] == 0) and np.all(res["w"] == 1.0)
    w13, w2 = moe.expert_weights_f64(ex[0])
    dense, _ = moe.swiglu_ffn(moe._f64(h), w13, w2)
    assert np.max(np.abs(res["out"] - dense)) < 1e-12


def test_forward_against_scalar_loops():
    # the whole tiny layer recomputed token by token with scalar Python arithmetic (math.exp,
    # no numpy products) -- a different evaluation of the same definition
    cfg = synth.MoEConfig("loop", T=6, H=16, E=4, k=2, I=8, S=1, seed=9)
    h, Wr, bias, ex = _tiny_layer(cfg)
    res = moe.forward(h, Wr, bias, ex.__getitem__, cfg.E, cfg.k, cfg.S)
    X = h.float().numpy().astype(float).tolist()
    W = Wr.numpy().astype(float).tolist()
    mats = {e: [m.float().numpy().astype(float).tolist() for m in (ex[e]["w13"], ex[e]["w2"])]
            for e in ex}

    def expert(e, x):
        w13, w2 = mats[e]
        I = cfg.I
        act = []
        for i in range(I):
            g = sum(w13[i][c] * x[c] for c in range(cfg.H))
            u = sum(w13[I + i][c] * x[c] for c in range(cfg.H))
            act.append(g / (1.0 + math.exp(-g)) * u)
        return [sum(w2[r][i] * act[i] for i in range(I)) for r in range(cfg.H)]

    for t in range(cfg.T):
        logit = [sum(X[t][c] * W[e][c] for c in range(cfg.H)) for e in range(cfg.E)]
        chosen = sorted(range(cfg.E), key=lambda e: (-logit[e], e))[:cfg.k]
        z = [math.exp(logit[e] - logit[chosen[0]]) for e in chosen]
        out = expert(cfg.E, X[t])
        for j, e in enumerate(chosen):
            y = expert(e, X[t])
            out = [o + z[j] / sum(z) * yy for o, yy in zip(out, y)]
        assert res["idx"][t].tolist() == chosen
        assert np.max(np.abs(np.array(out) - res["out"][t])) < 1e-12


def test_combine_one_hot_is_gather_plus_shared():
    rng = np.random.default_rng(0)
    y = rng.standard_normal((5, 3, 7))
    ys = rng.standard_normal((5, 7))
    w = np.zeros((5, 3))
    w[np.arange(5), [0, 2, 1, 1, 0]] = 1.0
    out = moe.combine(w, y, ys)
    assert np.allclose(out, y[np.arange(5), [0, 2, 1, 1, 0]] + ys, atol=0)


def test_combine_linearity():
    rng = np.random.default_rng(1)
    y = rng.standard_normal((4, 2, 6))
    ys = rng.standard_normal((4, 6))
    w = rng.random((4, 2))
    base = moe.combine(w, y, np.zeros_like(ys))
    assert np.allclose(moe.combine(2.5 * w, y, ys) - ys, 2.5 * base, atol=1e-13)


def test_sampled_tokens_equal_full_forward():
    cfg = synth.CONFIGS["tiny"]
    h, Wr, bias, ex = _tiny_layer(cfg)
    full = moe.forward(h, Wr, bias, ex.__getitem__, cfg.E, cfg.k, cfg.S)
    tok = [0, 5, 63, 17]
    part = moe.forward(h, Wr, bias, ex.__getitem__, cfg.E, cfg.k, cfg.S, tokens=tok)
    assert np.array_equal(part["idx"], full["idx"][tok])
    assert np.max(np.abs(part["out"] - full["out"][tok])) < 1e-13
    reused = moe.forward(h, Wr, bias, ex.__getitem__, cfg.E, cfg.k, cfg.S, tokens=tok,
                         routing=(full["idx"], full["w"]))
    assert np.max(np.abs(reused["out"] - full["out"][tok])) < 1e-13


def test_shared_expert_adds_linearly():
    cfg = synth.MoEConfig("sh", T=8, H=32, E=4, k=2, I=64, S=1, seed=2)
    h, Wr, bias, ex = _tiny_layer(cfg)
    with_s = moe.forward(h, Wr, bias, ex.__getitem__, cfg.E, cfg.k, 1)
    without = moe.forward(h, Wr, bias, ex.__getitem__, cfg.E, cfg.k, 0)
    w13, w2 = moe.expert_weights_f64(ex[cfg.E])
    ys, _ = moe.swiglu_ffn(moe._f64(h), w13, w2)
    assert np.max(np.abs(with_s["out"] - without["out"] - ys)) < 1e-12


# ----------------------------------------------------------------------------- W8A8
# The FFN service is benchmarked on DeepSeek-V3.2 W8A8 (vLLM AFD Plugin, 效能基準測試 / 同步
# Decode 吞吐量).  The reading of that path: the hidden row and the SwiGLU output row are each
# quantised to e4m3 with one fp32 scale (row amax / 448, 1 for a zero row) right before the
# product that consumes them; weights arrive as e4m3 codes times one fp32 scale per output row.

SIG_35 = 0.9706877692486436     # textbook logistic values: 1 / (1 + e^-3.5)
SIG_275 = 0.9399133498259924    # 1 / (1 + e^-2.75)


def _w8a8_example_expert():
    """H = 4, I = 2.  e4m3 codes times per-row scales (all products exact):
    gate rows  (2,0,0,0) x 0.25 = (0.5,0,0,0)   and (0,0,0,1) x 1   = (0,0,0,1)
    up rows    (0,0,0,4) x 0.125 = (0,0,0,0.5)  and (0,1,0,0) x 2   = (0,2,0,0)
    down rows  (1,0), (0,1), (1,1) x 1  and (1,-2) x 0.5 = (0.5,-1)"""
    import torch
    w13 = torch.tensor([[2, 0, 0, 0], [0, 0, 0, 1], [0, 0, 0, 4], [0, 1, 0, 0]], dtype=torch.float32)
    w2 = torch.tensor([[1, 0], [0, 1], [1, 1], [1, -2]], dtype=torch.float32)
    return {"w13": w13.to(torch.float8_e4m3fn), "w2": w2.to(torch.float8_e4m3fn),
            "w13_scale": torch.tensor([0.25, 1.0, 0.125, 2.0]),
            "w2_scale": torch.tensor([1.0, 1.0, 1.0, 0.5])}


def test_w8a8_worked_example():
    import torch
    # hidden row (bf16 values): amax 7, so the scale is fp32(7 / 448) = 2^-6 exactly and the
    # quotients are x * 64 = (448, -90, 27, 170).  e4m3 steps: 8 in [64, 128), 2 in [16, 32), 16
    # in [128, 256).  -90 -> -88 (nearer), 27 -> 28 (tie between 26 = 1.625*16, odd mantissa, and
    # 28 = 1.75*16, even), 170 -> 176 (nearer).  Dequantised: (7, -1.375, 0.4375, 2.75).
    x = torch.tensor([[7.0, -1.40625, 0.421875, 2.65625]], dtype=torch.bfloat16)
    xq = moe.layer_input(x, fp8=True)
    assert xq.tolist() == [[7.0, -1.375, 0.4375, 2.75]]
    # g = (0.5 * 7, 2.75) = (3.5, 2.75); u = (0.5 * 2.75, 2 * -1.375) = (1.375, -2.75)
    # act = silu(g) * u = (3.5 * s(3.5) * 1.375, 2.75 * s(2.75) * -2.75)
    act_exact = [3.5 * SIG_35 * 1.375, -2.75 * 2.75 * SIG_275]
    assert act_exact[0] == pytest.approx(4.671434889509098, abs=1e-14)
    assert act_exact[1] == pytest.approx(-7.108094708059067, abs=1e-14)
    # fp32 act: 0x1.2af8cap+2 and -0x1.c6eb06p+2; amax = 0x1.c6eb06p+2 (7.108094692230225);
    # scale = fp32(amax / 448) = 0x1.03f404p-6 (the exact quotient is 0.0158662827951...)
    # quotients: act0 / scale = 294.4253 -> 288 (step 32 in [256, 448]); act1 / scale = -448
    s = float.fromhex("0x1.03f404p-6")
    w13, w2 = moe.expert_weights_f64(_w8a8_example_expert())
    assert w13.tolist() == [[0.5, 0, 0, 0], [0, 0, 0, 1], [0, 0, 0, 0.5], [0, 2, 0, 0]]
    y, act = moe.swiglu_ffn(xq, w13, w2, quant_act=True)
    assert act.tolist() == [[288 * s, -448 * s]]
    # y = act W2^T = (288s, -448s, 288s - 448s, 0.5 * 288s + 448s): every product and sum exact
    y_hand = [288 * s, -448 * s, -160 * s, 592 * s]
    assert y.tolist() == [y_hand]
    # the same through the whole layer: one expert, top-1 (weight 1), no shared expert
    res = moe.forward(x, torch.zeros((1, 4)), None, lambda e: _w8a8_example_expert(), 1, 1, 0, fp8=True)
    assert res["out"].tolist() == [y_hand]
    # without quantisation the layer is the fp64 SwiGLU of the bf16 row (a different number)
    plain, _ = moe.swiglu_ffn(moe._f64(x), w13, w2)
    assert abs(plain[0, 0] - y_hand[0]) > 1e-3


def test_w8a8_forward_against_scalar_loops():
    # the W8A8 layer token by token in scalar Python: fp32 roundings via numpy float32 scalars,
    # e4m3 rounding via ml_dtypes (an independent implementation), math.exp for silu, no numpy
    # products.  Token 3 is an all-zero row: scale 1 for the hidden row and for its act rows.
    import ml_dtypes
    cfg = synth.MoEConfig("loop8", T=6, H=16, E=4, k=2, I=8, S=1, dtype="fp8", seed=9)
    h, Wr, bias, ex = _tiny_layer(cfg)
    h[3] = 0
    res = moe.forward(h, Wr, bias, ex.__getitem__, cfg.E, cfg.k, cfg.S, fp8=True)
    X = h.float().numpy().astype(float).tolist()
    W = Wr.numpy().astype(float).tolist()

    def deq(e, name):
        q = ex[e][name].float().numpy().astype(float)
        s = ex[e][name + "_scale"].numpy().astype(float)
        return (q * s[:, None]).tolist()

    mats = {e: (deq(e, "w13"), deq(e, "w2")) for e in ex}

    def quant_row(v):
        v32 = [np.float32(a) for a in v]
        amax = max(abs(a) for a in v32)
        s = amax / np.float32(448.0) if amax > 0 else np.float32(1.0)
        assert isinstance(s, np.float32)
        q = [float(np.float32(a / s).astype(ml_dtypes.float8_e4m3fn)) for a in v32]
        return [c * float(s) for c in q]

    def expert(e, xq):
        w13, w2 = mats[e]
        I = cfg.I
        act = []
        for i in range(I):
            g = sum(w13[i][c] * xq[c] for c in range(cfg.H))
            u = sum(w13[I + i][c] * xq[c] for c in range(cfg.H))
            act.append(g / (1.0 + math.exp(-g)) * u)
        a = quant_row(act)
        return [sum(w2[r][i] * a[i] for i in range(I)) for r in range(cfg.H)]

    for t in range(cfg.T):
        logit = [sum(X[t][c] * W[e][c] for c in range(cfg.H)) for e in range(cfg.E)]
        chosen = sorted(range(cfg.E), key=lambda e: (-logit[e], e))[:cfg.k]
        z = [math.exp(logit[e] - logit[chosen[0]]) for e in chosen]
        xq = quant_row(X[t])
        out = expert(cfg.E, xq)
        for j, e in enumerate(chosen):
            y = expert(e, xq)
            out = [o + z[j] / sum(z) * yy for o, yy in zip(out, y)]
        assert res["idx"][t].tolist() == chosen
        assert np.max(np.abs(np.array(out) - res["out"][t])) < 1e-12
    assert np.all(res["out"][3] == 0.0)

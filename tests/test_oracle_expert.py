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

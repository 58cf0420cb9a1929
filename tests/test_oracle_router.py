"""Pins of the oracle's router, selection and gate weights (CPU only).

The pages name the routing computation (vLLM AFD Plugin, Attention-FFN 解耦的原理) and the
sparse activation of a few experts per token (LLM 推理提速: Attention与FFN分离AFD方, 一个在
啃带宽，一个在吃算力) without defining either; the checks below pin the oracle's reading
(softmax top-k, renormalised) to brute force, a hand-worked example and invariants.
"""
import itertools
import math

import numpy as np
import pytest

import synth
from oracle import moe


def test_router_worked_example():
    # hidden (1, 2); Wr rows (1,0), (0,1), (1,1); bias (0, 0.5, -3)
    # logits = (1, 2 + 0.5, 3 - 3) = (1, 2.5, 0); top-2 = experts 1 then 0;
    # weights = softmax(2.5, 1) = (1/(1+e^-1.5), 1/(1+e^1.5)) = (0.8175744761936437, ...)
    hidden = np.array([[1.0, 2.0]])
    Wr = np.array([[1.0, 0.0], [0.0, 1.0], [1.0, 1.0]])
    bias = np.array([0.0, 0.5, -3.0])
    logits, idx, w = moe.route(hidden, Wr, bias, k=2)
    assert np.allclose(logits, [[1.0, 2.5, 0.0]], atol=0, rtol=0)
    assert idx.tolist() == [[1, 0]]
    assert w[0, 0] == pytest.approx(0.8175744761936437, abs=1e-15)
    assert w[0, 1] == pytest.approx(1.0 - 0.8175744761936437, abs=1e-15)


def _brute_topk(row, k):
    best = max(itertools.combinations(range(len(row)), k), key=lambda s: sum(row[i] for i in s))
    return sorted(best, key=lambda e: (-row[e], e))


@pytest.mark.parametrize("E,k", [(8, 2), (6, 3), (5, 1), (4, 4)])
def test_topk_matches_brute_force(E, k):
    rng = np.random.default_rng(7)
    logits = rng.standard_normal((40, E))
    idx = moe.topk_select(logits, k)
    for t in range(logits.shape[0]):
        assert idx[t].tolist() == _brute_topk(logits[t], k)


def test_topk_ties_go_to_lower_index():
    logits = np.array([[0.5, 2.0, 2.0, -1.0, 2.0]])
    assert moe.topk_select(logits, 3).tolist() == [[1, 2, 4]]
    assert moe.topk_select(logits, 2).tolist() == [[1, 2]]


def test_gate_weights_two_readings_agree_and_sum_to_one():
    rng = np.random.default_rng(3)
    for E, k in [(8, 2), (64, 8), (256, 8)]:
        logits = 3.0 * rng.standard_normal((100, E))
        idx = moe.topk_select(logits, k)
        w1 = moe.gate_weights(logits, idx)
        w2 = moe.gate_weights_renorm(logits, idx)
        assert np.max(np.abs(w1 - w2)) < 1e-12
        assert np.max(np.abs(w1.sum(axis=1) - 1.0)) < 1e-12
        assert np.all(np.diff(w1, axis=1) <= 0)          # descending logits -> descending w


def test_gate_weights_shift_invariant():
    rng = np.random.default_rng(4)
    logits = rng.standard_normal((10, 16))
    idx = moe.topk_select(logits, 4)
    assert np.allclose(moe.gate_weights(logits, idx), moe.gate_weights(logits + 123.0, idx),
                       atol=1e-12)


def test_bias_shifts_selection():
    # a large positive bias on one expert forces it first for every token; a sign error or
    # a dropped bias fails this
    cfg = synth.CONFIGS["tiny"]
    h = synth.gen_hidden(cfg)
    Wr, _ = synth.gen_router(cfg)
    bias = np.zeros(cfg.E)
    bias[5] = 100.0
    _, idx, w = moe.route(h, Wr, bias, cfg.k)
    assert np.all(idx[:, 0] == 5)
    assert np.all(w[:, 0] > 0.99)


@pytest.mark.parametrize("name", list(synth.CONFIGS))
def test_stored_redraws_give_margin(name):
    cfg = synth.CONFIGS[name]
    h = synth.gen_hidden(cfg)
    Wr, bias = synth.gen_router(cfg)
    ok = moe.margin_ok(moe.router_logits(h, Wr, bias), cfg.k, 1e-3)
    assert ok.all(), f"{(~ok).sum()} tokens lack the 1e-3 top-(k+1) margin"


def test_zipf_skew_calibration():
    # the skewed workload: a few experts receive about ten times the mean load
    cfg = synth.CONFIGS["dsv3_4096"]
    h = synth.gen_hidden(cfg)
    Wr, bias = synth.gen_router(cfg)
    _, idx, _ = moe.route(h, Wr, bias, cfg.k)
    counts = np.bincount(idx.ravel(), minlength=cfg.E)
    ratio = counts.max() / counts.mean()
    assert 8.0 <= ratio <= 13.0, ratio
    assert counts.min() > 0


def test_margin_ok_definition():
    logits = np.array([[3.0, 2.0, 1.0, 0.0],
                       [3.0, 2.9995, 1.0, 0.0],      # gap inside top-2
                       [3.0, 2.0, 1.0005, 1.0]])     # gap between 3rd and 4th (k+1 = 4)
    assert moe.margin_ok(logits, 2).tolist() == [True, False, True]
    assert moe.margin_ok(logits, 3).tolist() == [True, False, False]


def test_softmax_value_against_closed_form():
    # two selected logits a, b: w_0 = 1 / (1 + exp(b - a))
    logits = np.array([[0.3, -1.2, 5.0]])
    idx = moe.topk_select(logits, 2)
    w = moe.gate_weights(logits, idx)
    assert idx.tolist() == [[2, 0]]
    assert w[0, 0] == pytest.approx(1.0 / (1.0 + math.exp(0.3 - 5.0)), rel=1e-14)

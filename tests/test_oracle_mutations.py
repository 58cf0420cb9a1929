"""Planted mistakes in the oracle are caught by its pins (CPU only).

Each case patches one oracle function with a plausible error -- a dropped term, a swapped
operand, a wrong sign or order -- and checks that at least one of the pin tests fails on the
patched oracle.  The mistakes are planted in the oracle on the CPU; nothing here runs on a GPU.
"""
import numpy as np
import pytest

import test_oracle_dispatch as tdisp
import test_oracle_expert as texp
import test_oracle_fp8 as tfp8
import test_oracle_router as trouter
from oracle import fp8, moe


def _swapped_gate_up(x, w13, w2, quant_act=False):
    I = w13.shape[0] // 2
    g = x @ w13[:I].T
    u = x @ w13[I:].T
    act = g * moe.silu(u)                                 # silu on the wrong half
    return act @ w2.T, act


def _no_shared(w, y_routed, y_shared):
    out = np.zeros_like(np.asarray(y_shared, dtype=np.float64))
    for j in range(w.shape[1]):
        out += w[:, j:j + 1] * y_routed[:, j]
    return out


def _ascending_topk(logits, k):
    return np.argsort(logits, axis=1, kind="stable")[:, :k].astype(np.int32)


def _bias_subtracted(hidden, Wr, bias=None):
    logits = moe._f64(hidden) @ moe._f64(Wr).T
    return logits if bias is None else logits - moe._f64(bias)[None, :]


def _unnormalised_weights(logits, idx):
    p = np.exp(logits - logits.max(axis=1, keepdims=True))
    p = p / p.sum(axis=1, keepdims=True)
    return np.take_along_axis(p, idx.astype(np.int64), axis=1)


def _unstable_permute(idx, E):
    counts, offsets, pos, src = _ORIG_PERMUTE(idx, E)
    T, k = idx.shape
    pos = pos.copy()
    if T >= 2:                                            # reverse the order inside experts
        for e in range(E):
            sel = np.nonzero(idx == e)
            p = np.sort(pos[sel])
            pos[sel] = p[::-1]
    return counts, offsets, pos, src


_ORIG_PERMUTE = moe.permute


# ---- the W8A8 quantisation mirror (activation rows quantised to e4m3 before each product)
def _dequant(v):
    q, s = fp8.quantize_rows(np.asarray(v).astype(np.float32))
    return q * s.astype(np.float64)[:, None]


def _quant_after_down(x, w13, w2, quant_act=False):
    I = w13.shape[0] // 2
    act = moe.silu(x @ w13[:I].T) * (x @ w13[I:].T)
    y = act @ w2.T
    return (_dequant(y) if quant_act else y), act            # quantises the output instead


def _no_dequant_scale(x, w13, w2, quant_act=False):
    I = w13.shape[0] // 2
    act = moe.silu(x @ w13[:I].T) * (x @ w13[I:].T)
    if quant_act:
        act, _ = fp8.quantize_rows(act.astype(np.float32))  # codes used without "* scale"
    return act @ w2.T, act


def _quant_before_silu(x, w13, w2, quant_act=False):
    I = w13.shape[0] // 2
    g, u = x @ w13[:I].T, x @ w13[I:].T
    if quant_act:                                          # quantises the projections instead
        g, u = _dequant(g), _dequant(u)
    act = moe.silu(g) * u
    return act @ w2.T, act


def _fp64_scale(x32):
    x = np.asarray(x32, dtype=np.float32).astype(np.float64)
    amax = np.abs(x).max(axis=1)
    scale = np.where(amax > 0, amax / 448.0, 1.0)            # fp64 scale and quotient
    return fp8.e4m3_round(x / scale[:, None]), scale


def _hidden_not_quantised(hidden, fp8):  # noqa: F811 (keeps the keyword of layer_input)
    return moe._f64(hidden)


W8A8_PINS = [texp.test_w8a8_worked_example, texp.test_w8a8_forward_against_scalar_loops]

MUTATIONS = [
    (moe, "swiglu_ffn", _swapped_gate_up, [texp.test_swiglu_worked_example]),
    (moe, "combine", _no_shared, [texp.test_combine_one_hot_is_gather_plus_shared]),
    (moe, "topk_select", _ascending_topk, [trouter.test_router_worked_example]),
    (moe, "router_logits", _bias_subtracted, [trouter.test_bias_shifts_selection]),
    (moe, "gate_weights", _unnormalised_weights,
     [trouter.test_gate_weights_two_readings_agree_and_sum_to_one]),
    (moe, "permute", _unstable_permute, [tdisp.test_permute_against_quadratic_recount]),
    (moe, "swiglu_ffn", _quant_after_down, W8A8_PINS),
    (moe, "swiglu_ffn", _no_dequant_scale, W8A8_PINS),
    (moe, "swiglu_ffn", _quant_before_silu, W8A8_PINS),
    (fp8, "quantize_rows", _fp64_scale,
     [tfp8.test_quantize_rows_scale_and_quotient_are_fp32, tfp8.test_quantize_rows_matches_torch_fp32_path,
      texp.test_w8a8_worked_example]),
    (moe, "layer_input", _hidden_not_quantised, W8A8_PINS),
]
IDS = ["swapped_gate_up", "no_shared", "ascending_topk", "bias_sign", "unnormalised_weights",
       "unstable_permute", "w8a8_quant_after_down", "w8a8_no_dequant_scale", "w8a8_quant_before_silu",
       "w8a8_fp64_scale", "w8a8_hidden_not_quantised"]


@pytest.mark.parametrize("mod,name,bad,pins", MUTATIONS, ids=IDS)
def test_planted_mistake_is_caught(monkeypatch, mod, name, bad, pins):
    monkeypatch.setattr(mod, name, bad)
    caught = 0
    for pin in pins:
        try:
            pin()
        except AssertionError:
            caught += 1
    assert caught == len(pins), f"pins did not catch the planted mistake in {name}"

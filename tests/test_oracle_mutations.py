"""Planted mistakes in the oracle are caught by its pins (CPU only).

Each case patches one oracle function with a plausible error -- a dropped term, a swapped
operand, a wrong sign or order -- and checks that at least one of the pin tests fails on the
patched oracle.  The mistakes are planted in the oracle on the CPU; nothing here runs on a GPU.
"""
import numpy as np
import pytest

import test_oracle_dispatch as tdisp
import test_oracle_expert as texp
import test_oracle_router as trouter
from oracle import moe


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

MUTATIONS = [
    ("swiglu_ffn", _swapped_gate_up, [texp.test_swiglu_worked_example]),
    ("combine", _no_shared, [texp.test_combine_one_hot_is_gather_plus_shared]),
    ("topk_select", _ascending_topk, [trouter.test_router_worked_example]),
    ("router_logits", _bias_subtracted, [trouter.test_bias_shifts_selection]),
    ("gate_weights", _unnormalised_weights,
     [trouter.test_gate_weights_two_readings_agree_and_sum_to_one]),
    ("permute", _unstable_permute, [tdisp.test_permute_against_quadratic_recount]),
]


@pytest.mark.parametrize("name,bad,pins", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(monkeypatch, name, bad, pins):
    monkeypatch.setattr(moe, name, bad)
    caught = 0
    for pin in pins:
        try:
            pin()
        except AssertionError:
            caught += 1
    assert caught == len(pins), f"pins did not catch the planted mistake in {name}"

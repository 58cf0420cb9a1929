"""Pins of the oracle's dispatch order and of the pages' communication account (CPU only).

Dispatch moves each token's hidden state to its selected experts and combine brings the
outputs back (A/F 分离, 机制); the per-token byte account is the 通信账 paragraph of the
same page's 深入推导 section.
"""
import json
import os

import numpy as np
import pytest

import synth
from oracle import comm, moe

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _random_idx(T, E, k, seed):
    rng = np.random.default_rng(seed)
    return np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)


@pytest.mark.parametrize("T,E,k", [(1, 4, 1), (17, 8, 2), (64, 8, 8), (33, 16, 3), (0, 4, 2)])
def test_permute_bijection_counts_and_stability(T, E, k):
    idx = _random_idx(T, E, k, seed=T + E) if T else np.zeros((0, k), np.int32)
    counts, offsets, pos, src = moe.permute(idx, E)
    assert counts.sum() == T * k
    assert offsets[0] == 0 and offsets[-1] == T * k
    assert np.all(np.diff(offsets) == counts)
    assert sorted(pos.ravel().tolist()) == list(range(T * k))        # bijection
    for t in range(T):
        for j in range(k):
            e = idx[t, j]
            p = pos[t, j]
            assert src[p] == t
            assert offsets[e] <= p < offsets[e + 1]
    for e in range(E):                                                # ascending t per expert
        seg = src[offsets[e]:offsets[e + 1]]
        assert np.all(np.diff(seg) > 0)


def test_permute_against_quadratic_recount():
    T, E, k = 40, 8, 3
    idx = _random_idx(T, E, k, seed=11)
    counts, offsets, pos, src = moe.permute(idx, E)
    for e in range(E):                                                # O(T k E) recount
        assert counts[e] == sum(1 for t in range(T) for j in range(k) if idx[t, j] == e)
    for t in range(T):                                                # O(T^2 k) definition
        for j in range(k):
            e = idx[t, j]
            before = sum(1 for t2 in range(t) if e in idx[t2])
            assert pos[t, j] == offsets[e] + before


def test_permute_skips_out_of_range_experts():
    idx = np.array([[0, 9], [1, -1], [1, 0]], dtype=np.int32)
    counts, offsets, pos, src = moe.permute(idx, 4)
    assert counts.tolist() == [2, 2, 0, 0]
    assert pos.tolist() == [[0, -1], [2, -1], [3, 1]]
    assert src.tolist() == [0, 2, 1, 2]


def test_dispatch_counts_on_workloads():
    for name in ["tiny", "mid", "dsv3_256"]:
        cfg = synth.CONFIGS[name]
        _, idx, _ = moe.route(synth.gen_hidden(cfg), *synth.gen_router(cfg), cfg.k)
        counts, offsets, pos, src = moe.permute(idx, cfg.E)
        assert counts.sum() == cfg.T * cfg.k == comm.dispatched_rows(idx)
        assert all(len(set(row.tolist())) == cfg.k for row in idx)     # k distinct experts


def test_comm_account_matches_page():
    with open(os.path.join(GOLDEN, "comm_account.json")) as f:
        g = json.load(f)
    acc = comm.page_account(g["h"], g["k"], g["bytes_per_elem"])
    assert acc["total"] == g["per_token_per_layer_bytes"]
    # "about 131 KB": the printed figure, in decimal kilobytes, rounded
    assert round(acc["total"] / 1000) == g["printed_kb"]
    # "about 10 MB over 80 layers"
    assert round(acc["total"] * g["layers"] / 1e6) == g["printed_mb_all_layers"]


def test_comm_element_bytes():
    # element level: one h-wide row per selected pair; at 1 byte/elem, h*k per token each way
    idx = _random_idx(5, 16, 8, seed=1)
    assert comm.element_bytes(idx, 4096, 1) == 5 * 8 * 4096
    assert comm.page_account(4096, 8)["dispatch"] == 2 * 8 * 4096

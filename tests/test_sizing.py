"""A/F sizing helpers (CPU only): rate-matched split and the rank-layout rule."""
import json
import os

import pytest

from ffn_side_expert_b200 import sizing

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "rank_layouts.json")


def test_page_examples_of_the_rank_rule():
    with open(GOLDEN) as f:
        g = json.load(f)
    for a, f_ in g["valid"]:
        assert sizing.layout_error(a, f_) is None
        sizing.RankLayout(a, f_)
    for a, f_ in g["invalid"]:
        assert sizing.layout_error(a, f_) is not None
        with pytest.raises(ValueError):
            sizing.RankLayout(a, f_)


def test_rank_roles_ffn_first():
    lay = sizing.RankLayout(64, 16)
    assert lay.world_size == 80
    assert [lay.role(r) for r in (0, 15, 16, 79)] == ["ffn", "ffn", "attention", "attention"]
    assert lay.attention_per_ffn() == 4
    assert [lay.ffn_rank_of(r) for r in (16, 19, 20, 79)] == [0, 0, 1, 15]
    assert sizing.RankLayout(1, 1).role(0) == "ffn"


@pytest.mark.parametrize("a,f,n,want", [
    (1.0, 1.0, 8, (4, 4)),
    (1.0, 3.0, 8, (2, 6)),
    (3.0, 1.0, 8, (6, 2)),
    (1.0, 1.0, 3, (2, 1)),      # 1.5 -> 2 (half to even)
    (1.0, 1.0, 5, (2, 3)),      # 2.5 -> 2 (half to even)
    (0.0, 1.0, 8, (1, 7)),      # attention keeps at least one GPU
    (1.0, 126.0, 128, (1, 127)),
])
def test_rate_matched_split(a, f, n, want):
    got = sizing.rate_matched_split(a, f, n)
    assert got == want
    assert sum(got) == n and got[0] >= 1


def test_rate_matched_split_tracks_cost_share():
    for n in (16, 64, 128):
        for share in (0.1, 0.25, 0.5, 0.8):
            attn, ffn = sizing.rate_matched_split(share, 1.0 - share, n)
            assert abs(attn - share * n) <= 0.5 + 1e-9
    with pytest.raises(ValueError):
        sizing.rate_matched_split(1.0, 1.0, 1)

"""Sizing of an Attention-FFN split: rate matching and the rank-layout rule (host-side helpers).

Two facts from the pages, restated:

- Rate matching (AFD Disagg MoE study note, 案例 2：用"产能对齐"理解 attention/FFN GPU 比例): give
  attention a share of the GPUs proportional to its cost, attn_cost / (attn_cost + ffn_cost),
  rounded to a whole number of GPUs and at least one; the FFN side takes the rest.  The note
  presents this as a beginner's reading of rate matching, not the paper's search.  Reading
  taken here: "rounded" is round-half-to-even, as in the note's own arithmetic.
- Rank layout (Separar Attention de FFN page, section "Con qué te vas a tropezar"): FFN ranks
  come first, then attention ranks; the number of attention ranks must be at least the number
  of FFN ranks and a multiple of it (64 attention + 16 FFN is valid; 16 + 64 and 64 + 24 are
  not).
"""
from __future__ import annotations

import math
from dataclasses import dataclass


def _round_half_even(x: float) -> int:
    f = math.floor(x)
    d = x - f
    if d > 0.5:
        return f + 1
    if d < 0.5:
        return f
    return f if f % 2 == 0 else f + 1


def rate_matched_split(attn_cost: float, ffn_cost: float, total_gpus: int) -> tuple[int, int]:
    """(attention GPUs, FFN GPUs) with attention's share proportional to its cost."""
    if total_gpus < 2:
        raise ValueError("an A/F split needs at least two GPUs")
    if attn_cost < 0 or ffn_cost < 0 or attn_cost + ffn_cost <= 0:
        raise ValueError("costs must be non-negative and not both zero")
    share = attn_cost / (attn_cost + ffn_cost)
    attn = max(1, _round_half_even(total_gpus * share))
    return attn, total_gpus - attn


def layout_error(num_attention_ranks: int, num_ffn_ranks: int) -> str | None:
    """None when the rank counts are valid, else the reason they are not."""
    if num_attention_ranks < 1 or num_ffn_ranks < 1:
        return "both roles need at least one rank"
    if num_attention_ranks < num_ffn_ranks:
        return "attention ranks must be at least as many as FFN ranks"
    if num_attention_ranks % num_ffn_ranks != 0:
        return "attention ranks must be a multiple of the FFN ranks"
    return None


@dataclass(frozen=True)
class RankLayout:
    """Global rank numbering of an A/F deployment: FFN ranks first, then attention ranks."""
    num_attention_ranks: int
    num_ffn_ranks: int

    def __post_init__(self):
        err = layout_error(self.num_attention_ranks, self.num_ffn_ranks)
        if err:
            raise ValueError(f"{self.num_attention_ranks}A{self.num_ffn_ranks}F: {err}")

    @property
    def world_size(self) -> int:
        return self.num_attention_ranks + self.num_ffn_ranks

    def role(self, rank: int) -> str:
        if not 0 <= rank < self.world_size:
            raise ValueError("rank out of range")
        return "ffn" if rank < self.num_ffn_ranks else "attention"

    def attention_per_ffn(self) -> int:
        """Attention ranks served by each FFN rank."""
        return self.num_attention_ranks // self.num_ffn_ranks

    def ffn_rank_of(self, attention_rank: int) -> int:
        """The FFN rank an attention rank sends to, with attention ranks in contiguous blocks."""
        a = attention_rank - self.num_ffn_ranks
        if not 0 <= a < self.num_attention_ranks:
            raise ValueError("not an attention rank")
        return a // self.attention_per_ffn()

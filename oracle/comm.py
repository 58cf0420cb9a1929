"""The pages' per-token communication account of an A/F split, as byte counts.

Test infrastructure only (see the package docstring).

Source: A/F 分离 (bowenzhou.top knowledge page), section 深入推导：A/F 分离的流水收益与
通信账, paragraph 通信账.  Per token and layer the attention side dispatches the hidden
state, written there as 2h bytes, to each of the k active experts, and the combine returns
the same amount; for h = 4096, k = 8 at FP8 (1 byte) the page multiplies 2 x 4096 x 8 x 1 B
x 2 and reports about 131 KB per token per layer, and about 10 MB per token over 80 layers.

Reading: the factor "2" in "2h" is not explained at 1 byte per element (an FP8 hidden vector
is h bytes).  ``page_account`` reproduces the page's product literally; ``dispatched_rows``
and ``element_bytes`` give the element-level count of what a dispatch actually moves
(one hidden row per selected (token, expert) pair).
"""
from __future__ import annotations

import numpy as np


def page_account(h: int, k: int, bytes_per_elem: int = 1) -> dict:
    """Bytes per token per layer as the page computes them: 2*h*k*b each way, two ways."""
    per_direction = 2 * h * k * bytes_per_elem
    return {"dispatch": per_direction, "combine": per_direction,
            "total": 2 * per_direction}


def dispatched_rows(topk_idx) -> int:
    """Number of hidden rows a dispatch moves: one per selected (token, expert) pair."""
    idx = np.asarray(topk_idx)
    return int(idx.size)


def element_bytes(topk_idx, h: int, bytes_per_elem: int) -> int:
    """Element-level bytes of one dispatch direction: rows * h * bytes per element."""
    return dispatched_rows(topk_idx) * h * bytes_per_elem

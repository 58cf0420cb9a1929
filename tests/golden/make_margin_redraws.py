"""Write tests/golden/margin_redraws.json: which hidden rows each workload redraws.

Parity of the expert selection is checked bit for bit, which is only meaningful when no two
of a token's top k+1 router logits are closer than the rounding error of an fp32 router.
For every named workload this script draws the hidden states and the router with ``synth``,
evaluates the logits with the fp64 oracle, and for every token whose top-(k+1) logits have
an adjacent gap below 1e-3 tries replacement rows (attempt 1, 2, ...) until the margin
holds.  The result maps token -> attempt; ``synth.gen_hidden`` applies it.

Calls only ``synth`` and ``oracle``.  Run:  python tests/golden/make_margin_redraws.py
"""
from __future__ import annotations

import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402
from oracle import moe  # noqa: E402

MARGIN = 1e-3


def find_redraws(cfg, T=None, margin=MARGIN, max_attempts=1000) -> dict:
    """{token: attempt} that gives every token of ``cfg`` (first T rows) the margin."""
    hidden = synth.gen_hidden(cfg, T=T, redraws={})
    Wr, bias = synth.gen_router(cfg)
    ok = moe.margin_ok(moe.router_logits(hidden, Wr, bias), cfg.k, margin)
    redraws = {}
    for t in np.nonzero(~ok)[0]:
        for attempt in range(1, max_attempts + 1):
            row = synth.redraw_row(cfg, int(t), attempt)[None, :]
            if moe.margin_ok(moe.router_logits(row, Wr, bias), cfg.k, margin)[0]:
                redraws[int(t)] = attempt
                break
        else:
            raise RuntimeError(f"{cfg.name}: token {t} found no row with the margin")
    return redraws


def main():
    table = {}
    for name, cfg in synth.CONFIGS.items():
        table[name] = {str(t): a for t, a in sorted(find_redraws(cfg).items())}
        print(f"{name}: {len(table[name])} of {cfg.T} rows redrawn")
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)), "margin_redraws.json")
    with open(out, "w") as f:
        json.dump({"_about": "token -> redraw attempt giving every adjacent top-(k+1) router "
                             "logit gap >= 1e-3; written by make_margin_redraws.py",
                   **table}, f, indent=1, sort_keys=True)
        f.write("\n")


if __name__ == "__main__":
    main()

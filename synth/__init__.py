"""Seeded synthetic inputs for the MoE FFN-service layer.

Both sides of every parity check -- the fp64 CPU oracle and the CUDA library -- take their
inputs from this module, and nothing else is shared between them.  It draws random tensors
with the distributions of the five workloads and holds none of the layer's arithmetic: no
router, no selection, no expert FFN, no combine.

The one transformation done here is storing the W8A8 workload's expert weights the way they
arrive at the FFN service: e4m3 values with one fp32 scale per output channel.  That packing
uses torch's own float8_e4m3fn conversion on values already inside [-448, 448].

Streams: every tensor has its own numpy PCG64 stream keyed by
``SeedSequence([seed, tensor_id, ...])``, so experts can be drawn lazily, in any order and in
parallel, and a prefix of the hidden rows does not depend on how many rows are drawn.

Workload sources: the pages describe the layer (an MoE FFN with hundreds of experts of which
a few are active per token, DeepSeek-V3 shaped, W8A8 on the serving benchmark) but print no
tensor statistics; the distributions below (hidden ~ N(0,1), router ~ N(0,1/H) in fp32,
expert weights ~ N(0,1/fan_in)) are the stated workload definitions of this library.
"""
from __future__ import annotations

import json
import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, replace

import numpy as np
import torch

__all__ = [
    "MoEConfig", "CONFIGS", "get_config", "rng_for", "gen_experts_on",
    "gen_hidden", "redraw_row", "gen_router", "gen_expert", "gen_experts",
    "load_redraws", "REDRAW_TABLE",
]

# tensor ids of the PCG64 streams
_HIDDEN, _ROUTER_W, _ROUTER_PERM, _W13, _W2, _REDRAW = 0, 1, 2, 3, 4, 99

REDRAW_TABLE = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                            "tests", "golden", "margin_redraws.json")

E4M3_MAX = 448.0


@dataclass(frozen=True)
class MoEConfig:
    """Shape and input recipe of one MoE FFN workload.

    T tokens in the micro-batch, H hidden size, E routed experts, k experts per token,
    I expert intermediate size, S shared experts (0 or 1), dtype of the expert weights and
    activations ("bf16" or "fp8" = e4m3 with per-output-channel / per-token fp32 scales).
    zipf_s > 0 adds the per-expert Zipf bias  b_e = alpha * (-s * ln r_e)  to the router
    logits, r_e being the 1-based rank of expert e under a seeded random permutation.
    """
    name: str
    T: int
    H: int
    E: int
    k: int
    I: int
    S: int = 0
    dtype: str = "bf16"
    seed: int = 0
    zipf_s: float = 0.0
    zipf_alpha: float = 0.0

    @property
    def has_bias(self) -> bool:
        return self.zipf_s > 0.0

    def with_(self, **kw) -> "MoEConfig":
        return replace(self, **kw)

    def weight_bytes_per_expert(self) -> int:
        b = 1 if self.dtype == "fp8" else 2
        scales = (2 * self.I + self.H) * 4 if self.dtype == "fp8" else 0
        return 3 * self.I * self.H * b + scales


CONFIGS = {
    # small case: whole-tensor parity in seconds
    "tiny": MoEConfig("tiny", T=64, H=256, E=8, k=2, I=512, S=0, seed=0),
    # h=4096, k=8 decode micro-batch
    "mid": MoEConfig("mid", T=512, H=4096, E=64, k=8, I=1536, S=0, seed=1),
    # DeepSeek-V3 shaped decode micro-batch, uniform routing
    "dsv3_256": MoEConfig("dsv3_256", T=256, H=7168, E=256, k=8, I=2048, S=1, seed=2),
    # DeepSeek-V3 shaped large micro-batch, Zipf(s=1.1) skewed routing
    "dsv3_4096": MoEConfig("dsv3_4096", T=4096, H=7168, E=256, k=8, I=2048, S=1, seed=3,
                           zipf_s=1.1, zipf_alpha=0.30),
    # W8A8 prefill chunk
    "w8a8_8192": MoEConfig("w8a8_8192", T=8192, H=7168, E=256, k=8, I=2048, S=1,
                           dtype="fp8", seed=4),
    # W8A8 decode micro-batch (the serving benchmark's precision at the decode shape)
    "w8a8_256": MoEConfig("w8a8_256", T=256, H=7168, E=256, k=8, I=2048, S=1,
                          dtype="fp8", seed=5),
}


def get_config(name: str) -> MoEConfig:
    return CONFIGS[name]


def rng_for(*key: int) -> np.random.Generator:
    """The PCG64 stream for one tensor (key = seed, tensor id, then indices)."""
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(list(key))))


def load_redraws(name: str) -> dict:
    """Stored margin redraws {token: attempt} of a named workload (empty when none needed)."""
    with open(REDRAW_TABLE) as f:
        table = json.load(f)
    if name not in table:
        raise KeyError(f"no margin-redraw entry for workload {name!r} in {REDRAW_TABLE}")
    return {int(t): int(a) for t, a in table[name].items()}


def _redraw_f32(cfg: MoEConfig, t: int, attempt: int) -> np.ndarray:
    return rng_for(cfg.seed, _REDRAW, t, attempt).standard_normal(cfg.H, dtype=np.float32)


def redraw_row(cfg: MoEConfig, t: int, attempt: int) -> torch.Tensor:
    """Replacement attempt ``attempt`` (1, 2, ...) for hidden row t, as a bf16 row [H]."""
    return torch.from_numpy(_redraw_f32(cfg, t, attempt)).to(torch.bfloat16)


def gen_hidden(cfg: MoEConfig, T: int | None = None, redraws: dict | None = None) -> torch.Tensor:
    """Post-attention hidden states [T, H], bf16 (N(0,1) draws rounded to nearest even).

    ``redraws`` maps a token to the attempt number of its replacement row; rows are redrawn
    so that the router's top-(k+1) logits of every token are separated by the margin the
    parity checks rely on (the table is computed once by the oracle and stored).
    None -> the stored table of a named workload (or nothing for an unnamed one).
    """
    T = cfg.T if T is None else T
    x = rng_for(cfg.seed, _HIDDEN).standard_normal((T, cfg.H), dtype=np.float32)
    if redraws is None:
        redraws = load_redraws(cfg.name) if cfg.name in CONFIGS else {}
    for t, attempt in redraws.items():
        if t < T:
            x[t] = _redraw_f32(cfg, t, attempt)
    return torch.from_numpy(x).to(torch.bfloat16)


def gen_router(cfg: MoEConfig):
    """Router weight Wr [E, H] fp32 ~ N(0, 1/H) and the optional Zipf bias [E] fp32."""
    w = rng_for(cfg.seed, _ROUTER_W).standard_normal((cfg.E, cfg.H), dtype=np.float32)
    w *= np.float32(1.0 / math.sqrt(cfg.H))
    bias = None
    if cfg.has_bias:
        rank = rng_for(cfg.seed, _ROUTER_PERM).permutation(cfg.E) + 1   # r_e in 1..E
        bias = (cfg.zipf_alpha * (-cfg.zipf_s * np.log(rank.astype(np.float64)))).astype(np.float32)
        bias = torch.from_numpy(bias)
    return torch.from_numpy(w), bias


def _to_e4m3_per_row(w: np.ndarray):
    """Store fp32 rows as e4m3 values times one fp32 scale per row (amax / 448)."""
    amax = np.abs(w).max(axis=1).astype(np.float32)
    scale = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    v = np.clip(w / scale[:, None], -E4M3_MAX, E4M3_MAX).astype(np.float32)
    return torch.from_numpy(v).to(torch.float8_e4m3fn), torch.from_numpy(scale)


def gen_expert(cfg: MoEConfig, e: int) -> dict:
    """Weights of expert e (0..E-1 routed, E = the shared expert).

    w13 [2I, H]: rows 0..I-1 are the gate projection, rows I..2I-1 the up projection, each
    row one output channel over the hidden dimension (K-major).  w2 [H, I]: the down
    projection, one row per hidden output channel.  bf16, or e4m3 plus fp32 scales
    (w13_scale [2I], w2_scale [H]) for the W8A8 workload.
    """
    H, I = cfg.H, cfg.I
    w13 = rng_for(cfg.seed, _W13, e).standard_normal((2 * I, H), dtype=np.float32)
    w13 *= np.float32(1.0 / math.sqrt(H))
    w2 = rng_for(cfg.seed, _W2, e).standard_normal((H, I), dtype=np.float32)
    w2 *= np.float32(1.0 / math.sqrt(I))
    if cfg.dtype == "fp8":
        q13, s13 = _to_e4m3_per_row(w13)
        q2, s2 = _to_e4m3_per_row(w2)
        return {"w13": q13, "w2": q2, "w13_scale": s13, "w2_scale": s2}
    return {"w13": torch.from_numpy(w13).to(torch.bfloat16),
            "w2": torch.from_numpy(w2).to(torch.bfloat16)}


def gen_experts_on(cfg: MoEConfig, device, threads: int | None = None) -> dict:
    """The same stacked experts as gen_experts, written expert by expert into tensors on
    ``device``; the host holds only the experts in flight (a few hundred MB), not the stack."""
    n = cfg.E + cfg.S
    wdt = torch.float8_e4m3fn if cfg.dtype == "fp8" else torch.bfloat16
    out = {"w13": torch.empty((n, 2 * cfg.I, cfg.H), dtype=wdt, device=device),
           "w2": torch.empty((n, cfg.H, cfg.I), dtype=wdt, device=device)}
    if cfg.dtype == "fp8":
        out["w13_scale"] = torch.empty((n, 2 * cfg.I), dtype=torch.float32, device=device)
        out["w2_scale"] = torch.empty((n, cfg.H), dtype=torch.float32, device=device)

    def fill(e):
        d = gen_expert(cfg, e)
        for key, v in d.items():
            out[key][e].copy_(v)

    threads = threads or max(1, min(8, len(os.sched_getaffinity(0))))
    torch_threads = torch.get_num_threads()
    torch.set_num_threads(1)
    try:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(fill, range(n)))
    finally:
        torch.set_num_threads(torch_threads)
    return out


def gen_experts(cfg: MoEConfig, threads: int | None = None, pin: bool = False) -> dict:
    """All E + S experts stacked: w13 [E+S, 2I, H], w2 [E+S, H, I] (+ scales for fp8).

    Experts are drawn on a thread pool (numpy's generators and torch's conversions release
    the GIL).  ``pin`` allocates the stacks in page-locked memory for faster uploads.
    """
    n = cfg.E + cfg.S
    wdt = torch.float8_e4m3fn if cfg.dtype == "fp8" else torch.bfloat16
    out = {"w13": torch.empty((n, 2 * cfg.I, cfg.H), dtype=wdt, pin_memory=pin),
           "w2": torch.empty((n, cfg.H, cfg.I), dtype=wdt, pin_memory=pin)}
    if cfg.dtype == "fp8":
        out["w13_scale"] = torch.empty((n, 2 * cfg.I), dtype=torch.float32)
        out["w2_scale"] = torch.empty((n, cfg.H), dtype=torch.float32)

    def fill(e):
        d = gen_expert(cfg, e)
        for key, v in d.items():
            out[key][e].copy_(v)

    threads = threads or max(1, min(32, len(os.sched_getaffinity(0))))
    torch_threads = torch.get_num_threads()
    torch.set_num_threads(1)      # parallelism comes from the expert pool
    try:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(fill, range(n)))
    finally:
        torch.set_num_threads(torch_threads)
    return out

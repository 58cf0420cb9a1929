"""fp64 CPU oracle of the MoE expert layer that the FFN service runs.

Test infrastructure only (see the package docstring).

What the pages fix (cited by page title and section):
- The FFN service receives hidden states from attention and returns the layer's FFN output
  through compute_ffn_output() (vLLM AFD Plugin, 系統架構 / 2. FFN Service).
- Its work is the routing computation plus dispatch and combine (same page, Attention-FFN
  解耦的原理): a router picks, per token, a few of the layer's many experts (LLM 推理提速:
  Attention与FFN分离AFD方, 一个在啃带宽，一个在吃算力 -- DeepSeek-V3's FFN has hundreds of
  experts and activates a few per token), the hidden state is dispatched to the chosen
  experts, each expert is a large matrix multiplication, and the expert outputs are combined
  back per token (A/F 分离, 为什么要拆 and 机制).

What the pages leave open, and the reading taken here:
- router: logits l = hidden . Wr^T (+ bias), in fp32 on the device, fp64 here; the hidden
  state enters as the bf16 values the device receives.
- selection: the k largest logits, in descending order, ties to the lower expert index.
- gate weights: softmax over the selected logits, which equals the full softmax
  renormalised over the selected experts (both are computed below and must agree).
- expert: SwiGLU FFN  y = (silu(x Wg^T) * (x Wu^T)) W2^T,  silu(z) = z / (1 + e^-z).
- shared expert: applied to every token with weight 1, outside the routing.
- dispatch order: expert-major, ascending token index inside an expert.
- combine: out[t] = sum_j w[t,j] * y_{idx[t,j]}(x_t) + y_shared(x_t), in j order.
- W8A8: the hidden row and each SwiGLU output row are quantised to e4m3 with a per-row
  scale (oracle.fp8.quantize_rows) before the matrix products that consume them; weights
  arrive already as e4m3 values times per-output-channel fp32 scales.

Every matrix product here is one plain float64 numpy product; routing and the dispatch
order are plain loops over tokens.
"""
from __future__ import annotations

import numpy as np

from . import fp8 as _fp8


def _f64(a) -> np.ndarray:
    """Exact float64 copy of a numpy array or a CPU torch tensor (bf16 / fp32 / e4m3)."""
    if hasattr(a, "detach"):                          # torch tensor
        import torch
        a = a.detach().to("cpu")
        if a.dtype in (torch.bfloat16, torch.float16, torch.float8_e4m3fn):
            a = a.to(torch.float32)                    # exact widening
        a = a.numpy()
    return np.asarray(a, dtype=np.float64)


# ----------------------------------------------------------------------------- routing

def router_logits(hidden, Wr, bias=None) -> np.ndarray:
    """l[t, e] = sum_h hidden[t, h] * Wr[e, h] (+ bias[e]), float64."""
    logits = _f64(hidden) @ _f64(Wr).T
    if bias is not None:
        logits = logits + _f64(bias)[None, :]
    return logits


def topk_select(logits, k: int) -> np.ndarray:
    """Indices of the k largest logits per token, descending; equal logits -> lower index."""
    logits = np.asarray(logits, dtype=np.float64)
    order = np.argsort(-logits, axis=1, kind="stable")     # stable keeps lower index first
    return order[:, :k].astype(np.int32)


def gate_weights(logits, idx) -> np.ndarray:
    """Softmax over the selected logits: w[t,j] = exp(l[t,idx_j]) / sum_j' exp(l[t,idx_j'])."""
    sel = np.take_along_axis(np.asarray(logits, dtype=np.float64), idx.astype(np.int64), axis=1)
    z = np.exp(sel - sel.max(axis=1, keepdims=True))
    return z / z.sum(axis=1, keepdims=True)


def gate_weights_renorm(logits, idx) -> np.ndarray:
    """Full softmax over all experts, then renormalised over the selected ones."""
    logits = np.asarray(logits, dtype=np.float64)
    p = np.exp(logits - logits.max(axis=1, keepdims=True))
    p = p / p.sum(axis=1, keepdims=True)
    sel = np.take_along_axis(p, idx.astype(np.int64), axis=1)
    return sel / sel.sum(axis=1, keepdims=True)


def margin_ok(logits, k: int, margin: float = 1e-3) -> np.ndarray:
    """Per token: every adjacent gap among the top k+1 logits (top k when k = E) >= margin.

    When it holds, any evaluation of the logits with error below margin/2 selects the same
    experts in the same order.
    """
    logits = np.asarray(logits, dtype=np.float64)
    n = min(k + 1, logits.shape[1])
    top = -np.sort(-logits, axis=1)[:, :n]
    if n < 2:
        return np.ones(logits.shape[0], dtype=bool)
    return np.all(top[:, :-1] - top[:, 1:] >= margin, axis=1)


# ----------------------------------------------------------------------------- dispatch

def permute(idx, E: int):
    """Expert-major stable order of the (token, slot) pairs.

    counts[e]  = number of pairs with idx = e
    offsets    = exclusive prefix sum of counts, offsets[E] = T*k
    pos[t, j]  = offsets[e] + #{t' < t : token t' selected e}      (e = idx[t, j])
    src[p]     = the token whose row sits at dispatched position p
    A pair whose expert lies outside [0, E) is not dispatched: pos = -1.
    """
    idx = np.asarray(idx)
    T, k = idx.shape
    counts = np.zeros(E, dtype=np.int64)
    for t in range(T):
        for j in range(k):
            e = int(idx[t, j])
            if 0 <= e < E:
                counts[e] += 1
    offsets = np.zeros(E + 1, dtype=np.int64)
    for e in range(E):
        offsets[e + 1] = offsets[e] + counts[e]
    fill = offsets[:-1].copy()
    pos = np.full((T, k), -1, dtype=np.int64)
    src = np.full(int(offsets[E]), -1, dtype=np.int64)
    for t in range(T):                      # ascending t -> stable inside each expert
        for j in range(k):
            e = int(idx[t, j])
            if 0 <= e < E:
                pos[t, j] = fill[e]
                src[fill[e]] = t
                fill[e] += 1
    return (counts.astype(np.int32), offsets.astype(np.int32),
            pos.astype(np.int32), src.astype(np.int32))


# ----------------------------------------------------------------------------- experts

def silu(z) -> np.ndarray:
    """silu(z) = z / (1 + exp(-z))."""
    z = np.asarray(z, dtype=np.float64)
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def expert_weights_f64(expert: dict):
    """(w13, w2) of one expert as exact float64 matrices, scales applied for e4m3."""
    w13 = _f64(expert["w13"])
    w2 = _f64(expert["w2"])
    if "w13_scale" in expert:
        w13 = w13 * _f64(expert["w13_scale"])[:, None]
        w2 = w2 * _f64(expert["w2_scale"])[:, None]
    return w13, w2


def swiglu_ffn(x, w13, w2, quant_act: bool = False):
    """One expert on token rows x [m, H]:  y = (silu(x Wg^T) * (x Wu^T)) W2^T.

    w13 [2I, H] holds the gate rows then the up rows; w2 [H, I].  With ``quant_act`` the
    SwiGLU output is rounded to fp32 and quantised per row to e4m3 (the W8A8 path) before
    the down projection.  Returns (y [m, H], act [m, I] as fed to the down projection).
    """
    x = np.asarray(x, dtype=np.float64)
    I = w13.shape[0] // 2
    g = x @ w13[:I].T
    u = x @ w13[I:].T
    act = silu(g) * u
    if quant_act:
        q, s = _fp8.quantize_rows(act.astype(np.float32))
        act = q * s.astype(np.float64)[:, None]
    return act @ w2.T, act


# ----------------------------------------------------------------------------- the layer

def layer_input(hidden, fp8: bool) -> np.ndarray:
    """Token rows the experts see: the bf16 hidden, or its per-token e4m3 quantisation."""
    if not fp8:
        return _f64(hidden)
    q, s = _fp8.quantize_rows(_f64(hidden).astype(np.float32))
    return q * s.astype(np.float64)[:, None]


def route(hidden, Wr, bias, k: int):
    """Router + selection + gate weights for every token: (logits, idx, w)."""
    logits = router_logits(hidden, Wr, bias)
    idx = topk_select(logits, k)
    return logits, idx, gate_weights(logits, idx)


def forward(hidden, Wr, bias, expert_fn, E: int, k: int, n_shared: int, fp8: bool = False,
            tokens=None, routing=None) -> dict:
    """The MoE layer on the tokens ``tokens`` (all when None).

    expert_fn(e) returns expert e's weights (e = E is the shared expert).  Experts are
    visited one at a time, so only one expert's float64 weights exist at once.
    ``routing`` = (idx, w) reuses a routing already computed for all tokens.
    Returns a dict with logits/idx/w (when routed here), y_routed [n, k, H] (each selected
    expert's output for the token, before weighting), y_shared [n, H] and out [n, H].
    """
    hidden_all = hidden
    T = hidden_all.shape[0]
    tok = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    res = {}
    if routing is None:
        logits, idx, w = route(_f64(hidden_all)[tok], Wr, bias, k)
        res.update(logits=logits, idx=idx, w=w)
    else:
        idx, w = np.asarray(routing[0])[tok], np.asarray(routing[1], dtype=np.float64)[tok]
    x = layer_input(_f64(hidden_all)[tok], fp8)
    n, H = x.shape
    y_routed = np.zeros((n, k, H), dtype=np.float64)
    for e in range(E):
        rows, slots = np.nonzero(idx == e)
        if rows.size == 0:
            continue
        w13, w2 = expert_weights_f64(expert_fn(e))
        y, _ = swiglu_ffn(x[rows], w13, w2, quant_act=fp8)
        y_routed[rows, slots] = y
    y_shared = np.zeros((n, H), dtype=np.float64)
    for s in range(n_shared):
        w13, w2 = expert_weights_f64(expert_fn(E + s))
        y_shared += swiglu_ffn(x, w13, w2, quant_act=fp8)[0]
    res.update(y_routed=y_routed, y_shared=y_shared,
               out=combine(w, y_routed, y_shared))
    return res


def combine(w, y_routed, y_shared) -> np.ndarray:
    """out[t] = sum_j w[t, j] * y_routed[t, j] + y_shared[t]  (j in order)."""
    w = np.asarray(w, dtype=np.float64)
    out = np.array(y_shared, dtype=np.float64, copy=True)
    for j in range(w.shape[1]):
        out += w[:, j:j + 1] * y_routed[:, j]
    return out

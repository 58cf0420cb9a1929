"""Helpers shared by the GPU parity tests: one MoE layer's seeded inputs on the host and the
device, a handle of the CUDA library, and the oracle's answers on the same inputs."""
from __future__ import annotations

import numpy as np
import torch

import ffn_side_expert_b200 as afd
import synth
from oracle import moe

BF16_TOL = 2e-2   # max |err| <= tol x RMS(oracle output), bf16 weights and activations
FP8_TOL = 6e-2    # the same for the W8A8 path
W_TOL = 1e-5      # gate weights: fp32 logits differ from fp64 ones by ~1e-6 (sums of <= 7168 terms)


class Layer:
    """Seeded inputs of ``cfg`` on host and device plus a library handle (T_max = cfg.T)."""

    def __init__(self, cfg: synth.MoEConfig, T_max: int | None = None, hidden=None, bias=None,
                 redraws=None, edit_experts=None):
        self.cfg = cfg
        self.fp8 = cfg.dtype == "fp8"
        self.hidden = synth.gen_hidden(cfg, redraws=redraws) if hidden is None else hidden
        self.Wr, b = synth.gen_router(cfg)
        self.bias = b if bias is None else bias
        self.experts = synth.gen_experts(cfg)
        if edit_experts is not None:            # a test's change to the weights, before upload
            edit_experts(self.experts)
        dev = {k: v.cuda() for k, v in self.experts.items()}
        dev["router_w"] = self.Wr.cuda()
        if self.bias is not None:
            dev["router_bias"] = torch.as_tensor(self.bias, dtype=torch.float32).cuda()
        self.dev = dev
        self.h = self.hidden.cuda()
        self.T_max = T_max or self.hidden.shape[0]
        self.mod = afd.AfdFfn(T_max=self.T_max, H=cfg.H, E=cfg.E, k=cfg.k, I=cfg.I, n_shared=cfg.S,
                              fp8=self.fp8, weights=dev)
        self._oracle = None

    def expert_fn(self, e):
        return {k: v[e] for k, v in self.experts.items()}

    def oracle(self, tokens=None, routing=None):
        if tokens is None and routing is None and self._oracle is not None:
            return self._oracle
        r = moe.forward(self.hidden, self.Wr, self.bias, self.expert_fn, self.cfg.E, self.cfg.k,
                        self.cfg.S, fp8=self.fp8, tokens=tokens, routing=routing)
        if tokens is None and routing is None:
            self._oracle = r
        return r

    def oracle_routing(self):
        return moe.route(self.hidden, self.Wr, self.bias, self.cfg.k)

    # ---------------------------------------------------------------- device calls
    def route(self, T=None):
        T = self.hidden.shape[0] if T is None else T
        k = self.cfg.k
        idx = torch.full((max(T, 1), k), -7, dtype=torch.int32, device="cuda")
        w = torch.full((max(T, 1), k), -7.0, dtype=torch.float32, device="cuda")
        self.mod.route(self.h, T, idx, w)
        return idx[:T], w[:T]

    def permute(self, idx, T=None):
        T = idx.shape[0] if T is None else T
        E, k = self.cfg.E, self.cfg.k
        counts = torch.full((E,), -7, dtype=torch.int32, device="cuda")
        offsets = torch.full((E + 1,), -7, dtype=torch.int32, device="cuda")
        pos = torch.full((max(T, 1), k), -7, dtype=torch.int32, device="cuda")
        src = torch.full((max(T * k, 1),), -7, dtype=torch.int32, device="cuda")
        self.mod.permute(self.h, idx, T, counts, offsets, pos, src)
        return counts, offsets, pos[:T], src[:T * k]

    def expert_gemm(self, offsets, T):
        H, k = self.cfg.H, self.cfg.k
        Y = torch.full((T * k, H), float("nan"), dtype=torch.float32, device="cuda")
        Ys = torch.full((T, H), float("nan"), dtype=torch.float32, device="cuda") if self.cfg.S else None
        self.mod.expert_gemm(offsets, T, Y, Ys)
        return Y, Ys

    def combine(self, w, pos, T):
        out = torch.empty((T, self.cfg.H), dtype=torch.bfloat16, device="cuda")
        self.mod.combine(w, pos, T, out)
        return out

    def forward(self, T=None):
        T = self.hidden.shape[0] if T is None else T
        out = torch.empty((max(T, 1), self.cfg.H), dtype=torch.bfloat16, device="cuda")
        self.mod.forward(self.h, out, T=T)
        return out[:T]

    def close(self):
        self.mod.close()
        self.dev = None
        torch.cuda.empty_cache()


def to64(t) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def rel_max_err(got, ref) -> float:
    """max |got - ref| / RMS(ref)."""
    ref = np.asarray(ref, dtype=np.float64)
    rms = float(np.sqrt(np.mean(ref ** 2)))
    return float(np.max(np.abs(np.asarray(got, dtype=np.float64) - ref))) / rms

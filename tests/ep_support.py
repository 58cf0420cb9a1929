"""CPU stand-in for the library's kernels in expert-parallel tests (test infrastructure).

OracleRowsBackend implements each step of ExpertParallelFfn's per-rank work with the fp64
oracle on CPU tensors, so the exchange (counts, all-to-all-v splits, block regrouping, the
return path) can run on gloo ranks without a GPU.  bf16 mode: rows and outputs stay float64.
fp8 mode (W8A8 experts): each token's row is quantised once with the oracle's per-row e4m3
quantisation and sent as uint8 codes plus a float32 scale per row -- what the CUDA backend
sends -- and the experts apply the oracle's W8A8 mirror to the dequantised rows.
"""
import numpy as np
import torch

from ffn_side_expert_b200.ep import Dispatched
from oracle import fp8 as ofp8
from oracle import moe


class OracleRowsBackend:
    def __init__(self, *, Wr, bias, E, k, local_experts, shared=None, fp8=False):
        self.Wr, self.bias, self.E, self.k, self.fp8 = Wr, bias, E, k, fp8
        self.local = local_experts          # [(w13 f64, w2 f64)] of this rank's expert block
        self.shared = shared                # (w13, w2) or None

    def route(self, hidden, T):
        _, idx, w = moe.route(hidden.numpy(), self.Wr, self.bias, self.k)
        return torch.from_numpy(idx.astype(np.int32)), torch.from_numpy(w)

    def dispatch(self, hidden, idx, T):
        counts, _, pos, src = moe.permute(idx.numpy(), self.E)
        sel = torch.from_numpy(src.astype(np.int64))
        if not self.fp8:
            rows = hidden[sel] if src.size else hidden[:0]
            return Dispatched(torch.from_numpy(counts), torch.from_numpy(pos), rows.contiguous())
        q, s = ofp8.quantize_rows(hidden.numpy().astype(np.float32))
        codes = torch.from_numpy(ofp8.e4m3_encode(q))
        scales = torch.from_numpy(s)
        return Dispatched(torch.from_numpy(counts), torch.from_numpy(pos), codes[sel].contiguous(),
                          scales[sel].contiguous())

    def copy_blocks(self, src, dst, blocks, row_bytes):
        for s, d, n in blocks.tolist():
            dst[d:d + n] = src[s:s + n]

    def experts(self, rows, scales, per_expert, n):
        Y = torch.zeros((max(n, 1), rows.shape[1]), dtype=torch.float64)
        if self.fp8:
            x = ofp8.e4m3_decode(rows[:n].numpy()) * scales[:n].numpy().astype(np.float64)[:, None]
        else:
            x = rows[:n].numpy()
        off = 0
        for e, m in enumerate(per_expert.tolist()):
            if m:
                w13, w2 = self.local[e]
                Y[off:off + m] = torch.from_numpy(moe.swiglu_ffn(x[off:off + m], w13, w2, quant_act=self.fp8)[0])
            off += m
        return Y

    def shared_expert(self, hidden, T, d):
        if self.shared is None:
            return None
        x = moe.layer_input(hidden.numpy(), self.fp8)
        return torch.from_numpy(moe.swiglu_ffn(x, *self.shared, quant_act=self.fp8)[0])

    def combine(self, Y, Ys, w, pos, T):
        out = Ys.clone() if Ys is not None else torch.zeros((T, Y.shape[1]), dtype=torch.float64)
        acc = torch.zeros_like(out)
        for j in range(self.k):
            p = pos[:, j].to(torch.int64)
            ok = p >= 0
            acc[ok] += w[ok, j:j + 1] * Y[p[ok]]
        return acc + out if Ys is not None else acc

"""CPU stand-in for the library's kernels in expert-parallel tests (test infrastructure).

OracleRowsBackend implements each step of ExpertParallelFfn's per-rank work with the fp64
oracle on CPU tensors, so the exchange (counts, all-to-all-v splits, block regrouping, the
return path) can run on gloo ranks without a GPU.  Rows and outputs stay float64.
"""
import numpy as np
import torch

from oracle import moe


class OracleRowsBackend:
    def __init__(self, *, Wr, bias, E, k, local_experts, shared=None):
        self.Wr, self.bias, self.E, self.k = Wr, bias, E, k
        self.local = local_experts          # [(w13 f64, w2 f64)] of this rank's expert block
        self.shared = shared                # (w13, w2) or None

    def route(self, hidden, T):
        _, idx, w = moe.route(hidden.numpy(), self.Wr, self.bias, self.k)
        return torch.from_numpy(idx.astype(np.int32)), torch.from_numpy(w)

    def dispatch(self, hidden, idx, T):
        counts, _, pos, src = moe.permute(idx.numpy(), self.E)
        rows = hidden[torch.from_numpy(src.astype(np.int64))] if src.size else hidden[:0]
        return torch.from_numpy(counts), torch.from_numpy(pos), rows.contiguous()

    def copy_blocks(self, src, dst, blocks, row_bytes):
        for s, d, n in blocks.tolist():
            dst[d:d + n] = src[s:s + n]

    def experts(self, rows, per_expert, n):
        Y = torch.zeros((max(n, 1), rows.shape[1]), dtype=torch.float64)
        off = 0
        for e, m in enumerate(per_expert.tolist()):
            if m:
                w13, w2 = self.local[e]
                Y[off:off + m] = torch.from_numpy(moe.swiglu_ffn(rows[off:off + m].numpy(), w13, w2)[0])
            off += m
        return Y

    def shared_expert(self, hidden, T):
        if self.shared is None:
            return None
        return torch.from_numpy(moe.swiglu_ffn(hidden.numpy(), *self.shared)[0])

    def combine(self, Y, Ys, w, pos, T):
        out = Ys.clone() if Ys is not None else torch.zeros((T, Y.shape[1]), dtype=torch.float64)
        acc = torch.zeros_like(out)
        for j in range(self.k):
            p = pos[:, j].to(torch.int64)
            ok = p >= 0
            acc[ok] += w[ok, j:j + 1] * Y[p[ok]]
        return acc + out if Ys is not None else acc

"""Expert parallelism for the FFN layer across the ranks of a torch.distributed group.

Experts sit in contiguous blocks of E / world per rank; every rank holds a copy of the shared
expert and routes its own micro-batch.  The exchange is the one the A/F split pages describe
for the FFN side (A/F 分离 page, section 机制: each token's hidden state goes to the ranks that
hold its experts, and their outputs come back for the weighted combine; the page's section
通信账 counts those bytes).  Per forward:

  1. route (fp32 router, top-k, renormalised softmax) and dispatch the rows in expert-major
     order -- with experts in contiguous blocks that is also rank-major;
  2. exchange the per-expert row counts, then the rows (all-to-all-v);
  3. regroup the received rows from [source rank][local expert] to [local expert][source rank]
     and run the local experts;
  4. restore the received order and send the outputs back (all-to-all-v);
  5. combine: out[t] = sum_j w[t,j] * Y[pos[t,j]] + shared(hidden[t]).

Precision on the wire: bf16 weights send bf16 rows and get fp32 outputs back.  W8A8 weights
send each dispatched row as its e4m3 codes plus one fp32 scale -- the quantised hidden row
the experts consume anyway, so the exchange adds no error and its dispatch bytes are the
page's FP8 account plus 4 bytes of scale per row -- and get bf16 outputs back.

Every arithmetic step runs in the library's kernels (ExpertParallelFfn's default backend);
torch.distributed moves the bytes (NCCL between GPUs).  The backend is a parameter only so that
the exchange can be exercised on CPU ranks.
"""
from __future__ import annotations

import datetime
from dataclasses import dataclass

import torch
import torch.distributed as dist

from . import (AFD_FFN_ROUTE_STATIC_SCRATCH_FLOATS, AFD_OK, AfdError, AfdFfn, afd_ffn_combine_rows,
               afd_ffn_combine_rows_bf16, afd_ffn_copy_row_blocks, afd_ffn_dispatch_rows, afd_ffn_dispatch_rows_fp8,
               afd_ffn_expert_rows, afd_ffn_expert_rows_fp8, afd_ffn_route_static)


def block_tables(recv_counts: torch.Tensor):
    """Row-block moves between the received order and the per-expert order.

    recv_counts [world][E_local] (host int): rows that source rank s sent for local expert e,
    received as blocks ordered (s, e).  Returns (to_grouped, to_received): int32 [n][3] tables
    of (source row, destination row, rows) for moving (s, e) blocks into (e, s) order and back,
    and the rows per local expert.
    """
    c = recv_counts.to(torch.int64)
    world, el = c.shape
    recv_off = torch.zeros_like(c)
    flat = c.reshape(-1)
    recv_off.view(-1)[1:] = torch.cumsum(flat, 0)[:-1]
    per_expert = c.sum(0)
    grp_off = torch.zeros_like(c)
    expert_base = torch.zeros(el, dtype=torch.int64)
    expert_base[1:] = torch.cumsum(per_expert, 0)[:-1]
    for e in range(el):
        run = int(expert_base[e])
        for s in range(world):
            grp_off[s, e] = run
            run += int(c[s, e])
    fwd, back = [], []
    for s in range(world):
        for e in range(el):
            n = int(c[s, e])
            if n:
                fwd.append((int(recv_off[s, e]), int(grp_off[s, e]), n))
                back.append((int(grp_off[s, e]), int(recv_off[s, e]), n))
    as_t = (lambda rows: torch.tensor(rows, dtype=torch.int32).reshape(-1, 3))
    return as_t(fwd), as_t(back), per_expert.to(torch.int32)


@dataclass
class WireBytes:
    """Bytes one forward moved through the exchange on this rank."""
    dispatch_sent: int      # rows sent for dispatch (to every rank, this one included) x row bytes
                            # (W8A8: e4m3 codes + the fp32 row scale)
    dispatch_remote: int    # ... of which to other ranks
    combine_sent: int       # expert outputs sent back (fp32 rows; bf16 on the W8A8 path)
    combine_remote: int
    tokens: int
    dispatch_rows: int = 0  # rows sent for dispatch (T*k when every pair is valid)


@dataclass
class Dispatched:
    """One rank's dispatch: per-expert counts, each pair's row, the rows to send (expert-major)
    and their per-row scales (W8A8; None otherwise); `shared` is backend data for the shared
    expert (the CUDA W8A8 backend keeps the token-order quantised rows there)."""
    counts: torch.Tensor
    pos: torch.Tensor
    rows: torch.Tensor
    scales: torch.Tensor | None = None
    shared: object = None


class PeerLost(RuntimeError):
    """A rank of the group did not reach this step: found on the host, before any exchange."""

    def __init__(self, step: int, missing: list):
        self.step, self.missing = step, missing
        super().__init__(f"ranks {missing} did not reach step {step}" if missing else
                         f"step {step} was aborted by a rank whose wait for the others ran out")


class CudaRowsBackend:
    """The library's kernels for every step of the expert-parallel forward on one rank.

    fp8: the expert weights are e4m3 (local_w13_scale / local_w2_scale and the shared scales
    hold their per-output-channel fp32 scales); rows travel as e4m3 codes + fp32 row scales and
    outputs as bf16."""

    def __init__(self, *, H, E, k, I, T_max, world, router_w, router_bias, local_w13, local_w2,
                 shared_w13, shared_w2, device, fp8=False, local_w13_scale=None, local_w2_scale=None,
                 shared_w13_scale=None, shared_w2_scale=None):
        self.H, self.E, self.k, self.device, self.fp8 = H, E, k, device, fp8
        self.router_w, self.router_bias = router_w, router_bias
        el = E // world
        dummy_router = torch.zeros((el, H), dtype=torch.float32, device=device)  # unused by expert_rows
        wl = {"router_w": dummy_router, "w13": local_w13, "w2": local_w2}
        if fp8:
            wl.update(w13_scale=local_w13_scale, w2_scale=local_w2_scale)
        self.local = AfdFfn(T_max=world * T_max * k, H=H, E=el, k=1, I=I, n_shared=0, fp8=fp8, weights=wl)
        self.shared = None
        if shared_w13 is not None:
            ws = {"router_w": dummy_router[:1], "w13": shared_w13[None], "w2": shared_w2[None]}
            if fp8:
                ws.update(w13_scale=shared_w13_scale[None], w2_scale=shared_w2_scale[None])
            self.shared = AfdFfn(T_max=T_max, H=H, E=1, k=1, I=I, n_shared=0, fp8=fp8, weights=ws)
        self.scratch = torch.empty(2 * ((T_max + 127) // 128) * E, dtype=torch.int32, device=device)
        self.route_chunk = max(1, AFD_FFN_ROUTE_STATIC_SCRATCH_FLOATS // E)
        self.keep = [dummy_router]

    @staticmethod
    def _ok(st, what):
        if st != AFD_OK:
            raise AfdError(st, what)

    def route(self, hidden, T):
        idx = torch.empty((T, self.k), dtype=torch.int32, device=self.device)
        w = torch.empty((T, self.k), dtype=torch.float32, device=self.device)
        # the allocation-free router holds the partial logits of at most route_chunk tokens,
        # so a larger micro-batch is routed in consecutive chunks on the same stream
        for t0 in range(0, T, self.route_chunk):
            n = min(self.route_chunk, T - t0)
            self._ok(afd_ffn_route_static(hidden[t0:t0 + n], self.router_w, self.router_bias, n, self.H, self.E,
                                          self.k, idx[t0:t0 + n], w[t0:t0 + n]), "afd_ffn_route_static")
        return idx, w

    def dispatch(self, hidden, idx, T) -> Dispatched:
        counts = torch.empty(self.E, dtype=torch.int32, device=self.device)
        offsets = torch.empty(self.E + 1, dtype=torch.int32, device=self.device)
        pos = torch.empty((T, self.k), dtype=torch.int32, device=self.device)
        src = torch.empty(max(T * self.k, 1), dtype=torch.int32, device=self.device)
        if not self.fp8:
            rows = torch.empty((max(T * self.k, 1), self.H), dtype=torch.bfloat16, device=self.device)
            self._ok(afd_ffn_dispatch_rows(hidden, idx, T, self.k, self.E, self.H, counts, offsets, pos, src, rows,
                                           self.scratch), "afd_ffn_dispatch_rows")
            return Dispatched(counts, pos, rows)
        # the T token-order rows of the shared expert follow the dispatched ones
        ws = 1 if self.shared is not None else 0
        n = max(T * (self.k + ws), 1)
        rows = torch.empty((n, self.H), dtype=torch.uint8, device=self.device)
        scales = torch.empty(n, dtype=torch.float32, device=self.device)
        self._ok(afd_ffn_dispatch_rows_fp8(hidden, idx, T, self.k, self.E, self.H, ws, counts, offsets, pos, src,
                                           rows, scales, self.scratch), "afd_ffn_dispatch_rows_fp8")
        tk = T * self.k
        return Dispatched(counts, pos, rows[:max(tk, 1)], scales[:max(tk, 1)],
                          shared=(rows[tk:], scales[tk:]) if ws else None)

    def copy_blocks(self, src, dst, blocks, row_bytes):
        if blocks.shape[0]:
            b = blocks.to(self.device)
            self._ok(afd_ffn_copy_row_blocks(src, dst, b, b.shape[0], row_bytes), "afd_ffn_copy_row_blocks")

    def experts(self, rows, scales, per_expert, n):
        Y = torch.empty((max(n, 1), self.H), dtype=torch.bfloat16 if self.fp8 else torch.float32,
                        device=self.device)
        if n:
            cnt = per_expert.to(self.device)
            if self.fp8:
                self._ok(afd_ffn_expert_rows_fp8(self.local.h, rows, scales, cnt, n, Y), "afd_ffn_expert_rows_fp8")
            else:
                self._ok(afd_ffn_expert_rows(self.local.h, rows, cnt, n, Y), "afd_ffn_expert_rows")
        return Y

    def shared_expert(self, hidden, T, d: Dispatched):
        if self.shared is None:
            return None
        cnt = torch.tensor([T], dtype=torch.int32, device=self.device)
        if self.fp8:
            Ys = torch.empty((max(T, 1), self.H), dtype=torch.bfloat16, device=self.device)
            if T:
                self._ok(afd_ffn_expert_rows_fp8(self.shared.h, d.shared[0], d.shared[1], cnt, T, Ys),
                         "afd_ffn_expert_rows_fp8 (shared)")
            return Ys
        Ys = torch.empty((max(T, 1), self.H), dtype=torch.float32, device=self.device)
        self._ok(afd_ffn_expert_rows(self.shared.h, hidden, cnt, T, Ys), "afd_ffn_expert_rows (shared)")
        return Ys

    def combine(self, Y, Ys, w, pos, T):
        out = torch.empty((max(T, 1), self.H), dtype=torch.bfloat16, device=self.device)
        fn = afd_ffn_combine_rows_bf16 if self.fp8 else afd_ffn_combine_rows
        self._ok(fn(Y, Ys, w, pos, T, self.k, self.H, out), fn.__name__)
        return out[:T]

    def close(self):
        self.local.close()
        if self.shared is not None:
            self.shared.close()


class ExpertParallelFfn:
    """The MoE FFN layer with its routed experts split over the ranks of `group`.

    Every rank calls forward() with its own micro-batch (the same T on all ranks is not
    required).  `backend` defaults to CudaRowsBackend built from the arguments.

    T_max: the largest micro-batch a rank may pass; forward() refuses a larger one with
    ValueError before any device work (the dispatch scratch and the expert handles are sized
    for it).

    liveness: optional torch.distributed Store that every rank of the group reaches.  With it,
    each forward first checks on the host that every rank has reached the same step: each
    rank sets its arrival key, then waits up to liveness_timeout_s for the others'.  The step
    is then decided once, atomically, in the store (compare_set of the step's state key): "go"
    by the first rank that saw every arrival, or "abort" by the first rank whose wait ran out.
    Every rank acts on the decided state, so either all of them run the exchange or all of
    them raise PeerLost -- a rank that arrives after another gave up finds "abort" and raises
    too, instead of entering a collective alone.  A rank that has left, or a store that can no
    longer be reached, is reported as PeerLost before this rank launches any exchange.
    The aborted step stays decided, so a layer that raised PeerLost does not continue: the
    caller rebuilds the group (and the layer) without the lost rank.
    Without a store, a short process-group timeout is the bound.
    """

    def __init__(self, *, H, E, k, I, T_max, router_w=None, router_bias=None, local_w13=None, local_w2=None,
                 shared_w13=None, shared_w2=None, group=None, backend=None, device=None,
                 liveness=None, liveness_timeout_s: float = 5.0, local_w13_scale=None, local_w2_scale=None,
                 shared_w13_scale=None, shared_w2_scale=None):
        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        if E % self.world:
            raise ValueError("E must split evenly over the ranks")
        self.H, self.E, self.k, self.el = H, E, k, E // self.world
        self.T_max = T_max
        self.device = device or (router_w.device if router_w is not None else None)
        if backend is None and (router_w is None or local_w13 is None or local_w2 is None):
            raise ValueError("router_w, local_w13 and local_w2 are required for the library backend")
        fp8 = local_w13 is not None and local_w13.dtype == torch.float8_e4m3fn
        self.backend = backend or CudaRowsBackend(
            H=H, E=E, k=k, I=I, T_max=T_max, world=self.world, router_w=router_w, router_bias=router_bias,
            local_w13=local_w13, local_w2=local_w2, shared_w13=shared_w13, shared_w2=shared_w2, device=self.device,
            fp8=fp8, local_w13_scale=local_w13_scale, local_w2_scale=local_w2_scale,
            shared_w13_scale=shared_w13_scale, shared_w2_scale=shared_w2_scale)
        self.last_wire: WireBytes | None = None
        self.liveness, self.liveness_timeout_s = liveness, liveness_timeout_s
        self.step = 0

    def _key(self, step: int, rank: int) -> str:
        return f"afd_ep/{step}/{rank}"

    def _state_key(self, step: int) -> str:
        return f"afd_ep/{step}/state"

    def _missing(self, step: int) -> list:
        missing = []
        for r in range(self.world):
            try:
                if not self.liveness.check([self._key(step, r)]):
                    missing.append(r)
            except Exception:
                missing.append(r)
        return missing

    def check_peers(self) -> None:
        """Host-side check that every rank reached this step (no-op without a liveness store)."""
        st = self.liveness
        if st is None:
            return
        step = self.step
        keys = [self._key(step, r) for r in range(self.world)]
        try:
            st.set(self._key(step, self.rank), "1")
            try:
                st.wait(keys, datetime.timedelta(seconds=self.liveness_timeout_s))
                arrived = True
            except Exception:
                arrived = False
            # one decision per step, taken by whichever rank gets there first
            state = st.compare_set(self._state_key(step), "", "go" if arrived else "abort")
        except Exception as e:                   # the store itself is gone
            raise PeerLost(step, list(range(self.world))) from e
        if bytes(state) != b"go":
            raise PeerLost(step, self._missing(step))
        if step >= 2:
            # every rank has decided step - 1, so none still reads the keys of step - 2
            for k in (self._key(step - 2, self.rank), self._state_key(step - 2)):
                try:
                    st.delete_key(k)
                except Exception:
                    pass
        self.step = step + 1

    def forward(self, hidden: torch.Tensor) -> torch.Tensor:
        T, H, k = hidden.shape[0], self.H, self.k
        if T > self.T_max:
            raise ValueError(f"micro-batch of {T} tokens exceeds T_max = {self.T_max}")
        self.check_peers()
        b, g = self.backend, self.group
        idx, w = b.route(hidden, T)
        d = b.dispatch(hidden, idx, T)
        rows, scales = d.rows, d.scales
        # 2. per-(rank, local expert) row counts, then the rows (and their scales)
        send_c = d.counts.view(self.world, self.el).contiguous()
        recv_c = torch.empty_like(send_c)
        dist.all_to_all_single(recv_c, send_c, group=g)
        send_c_h, recv_c_h = send_c.cpu(), recv_c.cpu()
        send_split = send_c_h.sum(1).tolist()
        recv_split = recv_c_h.sum(1).tolist()
        n_send, n_recv = sum(send_split), sum(recv_split)
        recv_rows = torch.empty((max(n_recv, 1), H), dtype=rows.dtype, device=rows.device)
        dist.all_to_all_single(recv_rows[:n_recv], rows[:n_send], recv_split, send_split, group=g)
        recv_scales = None
        if scales is not None:
            recv_scales = torch.empty(max(n_recv, 1), dtype=scales.dtype, device=scales.device)
            dist.all_to_all_single(recv_scales[:n_recv], scales[:n_send], recv_split, send_split, group=g)
        # 3. local experts on the rows regrouped by expert
        to_grouped, to_received, per_expert = block_tables(recv_c_h)
        grouped = torch.empty_like(recv_rows)
        b.copy_blocks(recv_rows, grouped, to_grouped, H * rows.element_size())
        grouped_scales = None
        if recv_scales is not None:
            grouped_scales = torch.empty_like(recv_scales)
            b.copy_blocks(recv_scales, grouped_scales, to_grouped, scales.element_size())
        Yg = b.experts(grouped, grouped_scales, per_expert, n_recv)
        # 4. outputs back in the order each source sent its rows
        Yr = torch.empty_like(Yg)
        b.copy_blocks(Yg, Yr, to_received, H * Yg.element_size())
        Yback = torch.empty((max(n_send, 1), H), dtype=Yg.dtype, device=Yg.device)
        dist.all_to_all_single(Yback[:n_send], Yr[:n_recv], send_split, recv_split, group=g)
        # 5. weighted combine with the shared expert
        Ys = b.shared_expert(hidden, T, d)
        out = b.combine(Yback, Ys, w, d.pos, T)
        rb = H * rows.element_size() + (scales.element_size() if scales is not None else 0)
        yb = H * Yg.element_size()
        self.last_wire = WireBytes(
            dispatch_sent=n_send * rb,
            dispatch_remote=(n_send - send_split[self.rank]) * rb,
            combine_sent=n_recv * yb,
            combine_remote=(n_recv - recv_split[self.rank]) * yb,
            tokens=T, dispatch_rows=n_send)
        return out

    def close(self):
        if hasattr(self.backend, "close"):
            self.backend.close()

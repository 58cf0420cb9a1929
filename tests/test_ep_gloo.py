"""Expert parallelism over two gloo ranks on the CPU.

The experts are split in contiguous blocks over the ranks; each rank routes its own
micro-batch (of a different size), exchanges the per-expert row counts and the rows
(all-to-all-v), runs its expert block and sends the outputs back for the combine.  The local
compute here is the fp64 oracle (tests/ep_support.py), so what is checked is the exchange:
every rank's output must equal the single-process oracle layer on its tokens, and the bytes
on the wire must match the per-token account of the A/F split pages (dispatch rows: k per
token; the combine returns the same rows).
"""
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from ffn_side_expert_b200.ep import ExpertParallelFfn, block_tables

H, E, K, I = 16, 8, 2, 24
TOKENS = {0: 12, 1: 9}


def _weights(fp8=False):
    rng = np.random.default_rng(7)
    Wr = rng.normal(0, 1 / np.sqrt(H), (E, H))
    experts = [(rng.normal(0, 1 / np.sqrt(H), (2 * I, H)), rng.normal(0, 1 / np.sqrt(I), (H, I)))
               for _ in range(E + 1)]
    if fp8:   # W8A8 experts: every weight an e4m3 value times its output row's fp32 scale
        from oracle import fp8 as ofp8

        def q(w):
            codes, s = ofp8.quantize_rows(w.astype(np.float32))
            return codes * s.astype(np.float64)[:, None]
        experts = [(q(a), q(b)) for a, b in experts]
    return Wr, experts


def _worker(rank, world, port, q, tokens=TOKENS, fp8=False):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from ep_support import OracleRowsBackend
        from oracle import moe
        Wr, experts = _weights(fp8)
        el = E // world
        hidden = torch.from_numpy(np.random.default_rng(100 + rank).normal(0, 1, (tokens[rank], H)))
        backend = OracleRowsBackend(Wr=Wr, bias=None, E=E, k=K, local_experts=experts[rank * el:(rank + 1) * el],
                                    shared=experts[E], fp8=fp8)
        ep = ExpertParallelFfn(H=H, E=E, k=K, I=I, T_max=16, backend=backend)
        out = ep.forward(hidden)
        from oracle import comm
        if tokens[rank] == 0:                             # an empty micro-batch still takes part
            assert tuple(out.shape) == (0, H)
            q.put((rank, 0.0, 0.0, ep.last_wire, 0))
            return
        idx = moe.route(hidden.numpy(), Wr, None, K)[1]
        # the oracle's per-direction element account: float64 rows, or e4m3 codes + a 4-byte scale
        account = (comm.element_bytes(idx, H, 1) + comm.dispatched_rows(idx) * 4 if fp8
                   else comm.element_bytes(idx, H, 8))
        ref = moe.forward(hidden.numpy(), Wr, None, lambda e: {"w13": experts[e][0], "w2": experts[e][1]},
                          E, K, 1, fp8=fp8)["out"]
        q.put((rank, float(np.max(np.abs(out.numpy() - ref))), float(np.max(np.abs(ref))), ep.last_wire, account))
    finally:
        dist.destroy_process_group()


def _run(tokens, port, fp8=False):
    world = len(tokens)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q, tokens, fp8)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    row_bytes = H + 4 if fp8 else H * 8                                 # e4m3 + scale, or float64
    for rank, err, scale, wire, account in res:
        assert err <= 1e-12 * max(scale, 1.0), (rank, err)
        # every token sends k rows to the experts' ranks and gets k rows back
        assert wire.tokens == tokens[rank]
        assert wire.dispatch_rows == tokens[rank] * K
        assert wire.dispatch_sent == tokens[rank] * K * row_bytes
        assert wire.dispatch_sent == account                           # = the oracle's element account
    sent = sum(r[3].dispatch_rows for r in res)
    back = sum(r[3].combine_sent for r in res) // (H * 8)             # float64 rows back
    assert sent == back                                                # the same rows return


def test_two_ranks_match_the_single_process_layer():
    _run(TOKENS, 29600 + os.getpid() % 1000)


def test_four_ranks_with_an_empty_and_a_one_token_micro_batch():
    _run({0: 7, 1: 0, 2: 13, 3: 1}, 28600 + os.getpid() % 1000)


def test_w8a8_two_ranks_send_e4m3_rows_and_match_the_oracle():
    # the dispatched rows travel as e4m3 codes with their fp32 scale: H + 4 bytes per row,
    # the page's FP8 account (A/F 分离, 通信账) plus the scale; outputs equal the oracle's W8A8 layer
    _run(TOKENS, 21600 + os.getpid() % 1000, fp8=True)


def test_w8a8_four_ranks_with_an_empty_micro_batch():
    _run({0: 5, 1: 11, 2: 0, 3: 3}, 20600 + os.getpid() % 1000, fp8=True)


def test_block_tables_regroup_and_restore():
    # 3 source ranks x 2 local experts: rows arrive (source, expert)-major
    c = torch.tensor([[2, 0], [1, 3], [0, 2]])
    fwd, back, per_expert = block_tables(c)
    assert per_expert.tolist() == [3, 5]
    received = torch.arange(8)
    grouped = torch.empty_like(received)
    for s, d, n in fwd.tolist():
        grouped[d:d + n] = received[s:s + n]
    # expert 0: source 0's 2 rows (0,1), source 1's row (2); expert 1: source 1's 3 (3,4,5), source 2's 2 (6,7)
    assert grouped.tolist() == [0, 1, 2, 3, 4, 5, 6, 7]      # (0,0) (1,0) | (1,1) (2,1)
    restored = torch.empty_like(grouped)
    for s, d, n in back.tolist():
        restored[d:d + n] = grouped[s:s + n]
    assert torch.equal(restored, received)


def test_block_tables_interleave_sources_per_expert():
    c = torch.tensor([[1, 1], [1, 1]])                 # 2 sources x 2 experts, one row each
    fwd, _, per_expert = block_tables(c)
    received = torch.tensor([10, 11, 20, 21])          # (s0,e0) (s0,e1) (s1,e0) (s1,e1)
    grouped = torch.empty_like(received)
    for s, d, n in fwd.tolist():
        grouped[d:d + n] = received[s:s + n]
    assert grouped.tolist() == [10, 20, 11, 21]        # expert 0 rows from both sources first
    assert per_expert.tolist() == [2, 2]


class _CountingBackend:
    """OracleRowsBackend that counts the steps that reached routing."""

    def __init__(self, inner):
        self.inner, self.routed = inner, 0

    def route(self, hidden, T):
        self.routed += 1
        return self.inner.route(hidden, T)

    def __getattr__(self, name):
        return getattr(self.inner, name)


def _leaving_worker(rank, world, port, q, use_store):
    """Both ranks take one step; then rank 1 leaves (between steps) and rank 0 takes the next.
    With a liveness store rank 0 must report PeerLost before it starts any exchange; without one,
    its step must still end (an error from the exchange, or the process ending) rather than hang."""
    import datetime
    import time
    from ep_support import OracleRowsBackend
    from ffn_side_expert_b200.ep import PeerLost
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
    store = None
    if use_store:
        store = dist.TCPStore("127.0.0.1", port + 1, world, is_master=(rank == 0),
                              timeout=datetime.timedelta(seconds=20))
    Wr, experts = _weights()
    el = E // world
    backend = _CountingBackend(OracleRowsBackend(Wr=Wr, bias=None, E=E, k=K,
                                                 local_experts=experts[rank * el:(rank + 1) * el], shared=experts[E]))
    ep = ExpertParallelFfn(H=H, E=E, k=K, I=I, T_max=16, backend=backend, liveness=store, liveness_timeout_s=2.0)
    hidden = torch.from_numpy(np.random.default_rng(3 + rank).normal(0, 1, (6, H)))
    ep.forward(hidden)                                # step 0: everyone is here
    dist.barrier()
    if rank == 1:
        os._exit(0)                                   # leaves between steps
    t0 = time.monotonic()
    try:
        ep.forward(hidden)
        outcome = "no error"
    except PeerLost as e:
        outcome = f"PeerLost {e.missing}"
    except Exception as e:                            # the exchange reports the missing peer
        outcome = type(e).__name__
    q.put((outcome, time.monotonic() - t0, backend.routed))
    q.close()
    q.join_thread()                                   # flush the result before leaving without teardown
    os._exit(0)


def _run_leaving(use_store, port):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_leaving_worker, args=(r, 2, port, q, use_store)) for r in range(2)]
    for p in procs:
        p.start()
    procs[0].join(90)
    still = procs[0].is_alive()
    for p in procs:
        if p.is_alive():
            p.kill()                                  # this test's own child, by handle
        p.join(10)
    assert not still, "rank 0 did not finish its step"
    return None if q.empty() else q.get(timeout=5), procs[0].exitcode


def test_a_rank_that_leaves_is_found_on_the_host_before_the_exchange():
    got, code = _run_leaving(True, 25600 + 2 * (os.getpid() % 500))
    assert code == 0 and got is not None
    outcome, seconds, routed = got
    assert outcome == "PeerLost [1]"
    assert routed == 1                                # the second step stopped before routing
    assert seconds < 10.0


def test_without_a_store_the_step_still_ends():
    got, code = _run_leaving(False, 24600 + 2 * (os.getpid() % 500))
    # gloo reports a vanished peer as an error, or (from its own threads) ends the process
    assert (got is not None and got[0] != "no error") or code != 0, (got, code)


def _steps_worker(rank, world, port, q):
    import datetime
    from ep_support import OracleRowsBackend
    from oracle import moe
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=20))
    try:
        store = dist.TCPStore("127.0.0.1", port + 1, world, is_master=(rank == 0),
                              timeout=datetime.timedelta(seconds=20))
        Wr, experts = _weights()
        el = E // world
        backend = OracleRowsBackend(Wr=Wr, bias=None, E=E, k=K, local_experts=experts[rank * el:(rank + 1) * el],
                                    shared=experts[E])
        ep = ExpertParallelFfn(H=H, E=E, k=K, I=I, T_max=16, backend=backend, liveness=store)
        worst = 0.0
        for step in range(4):
            hidden = torch.from_numpy(np.random.default_rng(50 + 10 * step + rank).normal(0, 1, (5 + step, H)))
            out = ep.forward(hidden)
            ref = moe.forward(hidden.numpy(), Wr, None, lambda e: {"w13": experts[e][0], "w2": experts[e][1]},
                              E, K, 1)["out"]
            worst = max(worst, float(np.max(np.abs(out.numpy() - ref))))
        q.put((rank, worst, ep.step))
    finally:
        dist.destroy_process_group()


def test_liveness_checked_steps_match_the_oracle():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 23600 + 2 * (os.getpid() % 500)
    procs = [ctx.Process(target=_steps_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    for rank, worst, steps in sorted(q.get(timeout=10) for _ in range(2)):
        assert worst <= 1e-12 and steps == 4, (rank, worst, steps)


def _slow_worker(rank, world, port, q):
    """Both ranks take one step; then rank 1 sleeps past rank 0's liveness timeout (alive, only
    slow).  The step must be aborted consistently: rank 0 gives up and reports rank 1 missing,
    rank 1 arrives late, finds the step decided as aborted and raises too -- neither enters the
    exchange, so no rank is left waiting inside a collective."""
    import datetime
    import time
    from ep_support import OracleRowsBackend
    from ffn_side_expert_b200.ep import PeerLost
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=10))
    try:
        store = dist.TCPStore("127.0.0.1", port + 1, world, is_master=(rank == 0),
                              timeout=datetime.timedelta(seconds=20))
        Wr, experts = _weights()
        el = E // world
        backend = _CountingBackend(OracleRowsBackend(Wr=Wr, bias=None, E=E, k=K,
                                                     local_experts=experts[rank * el:(rank + 1) * el],
                                                     shared=experts[E]))
        ep = ExpertParallelFfn(H=H, E=E, k=K, I=I, T_max=16, backend=backend, liveness=store,
                               liveness_timeout_s=1.5)
        hidden = torch.from_numpy(np.random.default_rng(3 + rank).normal(0, 1, (6, H)))
        ep.forward(hidden)
        if rank == 1:
            time.sleep(4.0)
        try:
            ep.forward(hidden)
            outcome = "no error"
        except PeerLost as e:
            outcome = f"PeerLost {e.missing}"
        q.put((rank, outcome, backend.routed))
        dist.barrier()                                 # both ranks are still alive and in step
    finally:
        dist.destroy_process_group()


def test_a_slow_rank_aborts_the_step_on_every_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 22600 + 2 * (os.getpid() % 500)
    procs = [ctx.Process(target=_slow_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(90)
        assert p.exitcode == 0
    res = dict((r, (o, n)) for r, o, n in (q.get(timeout=10) for _ in range(2)))
    assert res[0] == ("PeerLost [1]", 1)               # gave up waiting for rank 1
    assert res[1] == ("PeerLost []", 1)                # arrived late: the step was already aborted


def test_a_micro_batch_above_T_max_is_refused_before_any_work():
    class _Group:
        pass

    class _Never:
        def route(self, *a):
            raise AssertionError("routed a micro-batch above T_max")

    import ffn_side_expert_b200.ep as epmod
    ep = ExpertParallelFfn.__new__(ExpertParallelFfn)
    ep.world, ep.rank, ep.H, ep.E, ep.k, ep.el, ep.T_max = 1, 0, H, E, K, E, 16
    ep.backend, ep.group, ep.liveness, ep.step = _Never(), None, None, 0
    with pytest.raises(ValueError, match="T_max"):
        epmod.ExpertParallelFfn.forward(ep, torch.zeros((17, H), dtype=torch.float64))

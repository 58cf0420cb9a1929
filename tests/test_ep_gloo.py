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


def _weights():
    rng = np.random.default_rng(7)
    Wr = rng.normal(0, 1 / np.sqrt(H), (E, H))
    experts = [(rng.normal(0, 1 / np.sqrt(H), (2 * I, H)), rng.normal(0, 1 / np.sqrt(I), (H, I)))
               for _ in range(E + 1)]
    return Wr, experts


def _worker(rank, world, port, q, tokens=TOKENS):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from ep_support import OracleRowsBackend
        from oracle import moe
        Wr, experts = _weights()
        el = E // world
        hidden = torch.from_numpy(np.random.default_rng(100 + rank).normal(0, 1, (tokens[rank], H)))
        backend = OracleRowsBackend(Wr=Wr, bias=None, E=E, k=K, local_experts=experts[rank * el:(rank + 1) * el],
                                    shared=experts[E])
        ep = ExpertParallelFfn(H=H, E=E, k=K, I=I, T_max=16, backend=backend)
        out = ep.forward(hidden)
        from oracle import comm
        if tokens[rank] == 0:                             # an empty micro-batch still takes part
            assert tuple(out.shape) == (0, H)
            q.put((rank, 0.0, 0.0, ep.last_wire, 0))
            return
        idx = moe.route(hidden.numpy(), Wr, None, K)[1]
        account = comm.element_bytes(idx, H, 8)          # the oracle's per-direction account
        ref = moe.forward(hidden.numpy(), Wr, None, lambda e: {"w13": experts[e][0], "w2": experts[e][1]},
                          E, K, 1)["out"]
        q.put((rank, float(np.max(np.abs(out.numpy() - ref))), float(np.max(np.abs(ref))), ep.last_wire, account))
    finally:
        dist.destroy_process_group()


def _run(tokens, port):
    world = len(tokens)
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q, tokens)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    for rank, err, scale, wire, account in res:
        assert err <= 1e-12 * max(scale, 1.0), (rank, err)
        # every token sends k rows to the experts' ranks and gets k rows back
        assert wire.tokens == tokens[rank]
        assert wire.dispatch_sent == tokens[rank] * K * H * 8          # float64 rows in this test
        assert wire.dispatch_sent == account                           # = the oracle's element account
    sent = sum(r[3].dispatch_sent for r in res)
    back = sum(r[3].combine_sent for r in res)
    assert sent == back                                                # the same rows return


def test_two_ranks_match_the_single_process_layer():
    _run(TOKENS, 29600 + os.getpid() % 1000)


def test_four_ranks_with_an_empty_and_a_one_token_micro_batch():
    _run({0: 7, 1: 0, 2: 13, 3: 1}, 28600 + os.getpid() % 1000)


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


def _leaving_worker(rank, world, port, q):
    """Rank 1 leaves between steps (after the group is up, before the next forward); rank 0's
    next forward must end with an error from the group's short timeout, not hang."""
    import datetime
    import time
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
    dist.barrier()
    if rank == 1:
        os._exit(0)                                   # leaves without taking the next step
    from ep_support import OracleRowsBackend
    Wr, experts = _weights()
    backend = OracleRowsBackend(Wr=Wr, bias=None, E=E, k=K, local_experts=experts[:E // world], shared=experts[E])
    ep = ExpertParallelFfn(H=H, E=E, k=K, I=I, T_max=16, backend=backend)
    hidden = torch.from_numpy(np.random.default_rng(3).normal(0, 1, (6, H)))
    t0 = time.monotonic()
    try:
        ep.forward(hidden)
        q.put(("no error", time.monotonic() - t0))
    except Exception as e:                            # the exchange reports the missing peer
        q.put((type(e).__name__, time.monotonic() - t0))
    os._exit(0)


def test_a_rank_that_leaves_ends_the_others_step_with_an_error():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 27600 + os.getpid() % 1000
    procs = [ctx.Process(target=_leaving_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    try:
        outcome, seconds = q.get(timeout=90)
    finally:
        for p in procs:
            p.join(30)
            if p.is_alive():
                p.kill()                              # this test's own child, by handle
    assert outcome != "no error"
    assert seconds < 60

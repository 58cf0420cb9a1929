"""The FFN-service mailbox on the CPU: the slot protocol (post, take, complete, wait), its
order, its bounded waits and its rejections.  Buffers are ordinary host memory here; the
serving loop itself, which needs a device, is covered by tests/test_gpu_service.py."""
import threading
import time

import pytest
import torch

import ffn_side_expert_b200 as afd
from ffn_side_expert_b200.service import Mailbox


@pytest.fixture
def mb():
    m = Mailbox(3, 16, 64, pinned=False)
    yield m
    m.close()


def test_buffers_are_zeroed_distinct_and_writable(mb):
    views = [mb.input(s) for s in range(3)] + [mb.output(s) for s in range(3)]
    assert all(v.shape == (16, 64) and v.dtype == torch.bfloat16 for v in views)
    assert all(float(v.abs().sum()) == 0.0 for v in views)
    ptrs = {v.data_ptr() for v in views}
    assert len(ptrs) == 6 and all(p % 64 == 0 for p in ptrs)
    mb.input(1).fill_(3.0)
    assert float(mb.input(1).sum()) == 3.0 * 16 * 64 and float(mb.input(0).abs().sum()) == 0.0


def test_slots_are_taken_in_post_order(mb):
    for s, T in ((2, 5), (0, 16), (1, 0)):
        mb.post(s, T)
    got = [mb.take(0.1) for _ in range(3)]
    assert got == [(afd.AFD_OK, 2, 5), (afd.AFD_OK, 0, 16), (afd.AFD_OK, 1, 0)]
    assert mb.take(0.01)[0] == afd.AFD_ERR_TIMEOUT
    for s in (1, 2, 0):
        assert mb.complete(s) == afd.AFD_OK
    for s in range(3):
        mb.wait(s, 0.1)
        post, take, done = mb.times_ns(s)
        assert 0 < post <= take <= done


def test_wait_is_bounded_and_leaves_the_slot(mb):
    mb.post(0, 4)
    t0 = time.perf_counter()
    assert afd.afd_ffn_mailbox_wait(mb.mb, 0, 20000) == afd.AFD_ERR_TIMEOUT   # posted, not taken
    assert 0.015 < time.perf_counter() - t0 < 2.0
    st, slot, T = mb.take(0.1)
    assert (st, slot, T) == (afd.AFD_OK, 0, 4)
    assert afd.afd_ffn_mailbox_wait(mb.mb, 0, 1000) == afd.AFD_ERR_TIMEOUT    # taken, not complete
    assert mb.complete(0) == afd.AFD_OK
    assert afd.afd_ffn_mailbox_wait(mb.mb, 0, 0) == afd.AFD_OK


def test_failed_slot_reports_the_consumer_status(mb):
    mb.post(1, 3)
    _, slot, _ = mb.take(0.1)
    assert mb.complete(slot, afd.AFD_ERR_CUDA) == afd.AFD_OK
    assert afd.afd_ffn_mailbox_wait(mb.mb, 1, 0) == afd.AFD_ERR_CUDA
    with pytest.raises(afd.AfdError):
        mb.wait(1, 0.0)
    mb.post(1, 3)                                   # a failed slot can be posted again
    assert mb.take(0.1) == (afd.AFD_OK, 1, 3)


def test_protocol_violations_are_rejected(mb):
    inv = afd.AFD_ERR_INVALID_ARG
    assert afd.afd_ffn_mailbox_wait(mb.mb, 0, 0) == inv            # never posted
    assert afd.afd_ffn_mailbox_complete(mb.mb, 0, afd.AFD_OK) == inv  # not taken
    assert afd.afd_ffn_mailbox_post(mb.mb, 0, 17) == inv           # T > T_max
    assert afd.afd_ffn_mailbox_post(mb.mb, 0, -1) == inv
    assert afd.afd_ffn_mailbox_post(mb.mb, 3, 1) == inv            # no such slot
    assert afd.afd_ffn_mailbox_input(mb.mb, 3) is None
    mb.post(0, 1)
    assert afd.afd_ffn_mailbox_post(mb.mb, 0, 1) == inv            # already posted
    mb.take(0.1)
    assert afd.afd_ffn_mailbox_post(mb.mb, 0, 1) == inv            # taken
    assert afd.afd_ffn_mailbox_complete(mb.mb, 0, 5) == inv        # status must be <= 0
    assert mb.complete(0) == afd.AFD_OK
    assert mb.complete(0) == inv                                   # completed twice


def test_create_rejects_bad_shapes():
    for args in ((0, 4, 64, 0), (2, 0, 64, 0), (2, 4, 60, 0), (2, 4, 0, 0), (2, 4, 64, 2), (2000, 4, 64, 0)):
        st, m = afd.afd_ffn_mailbox_create(*args)
        assert st == afd.AFD_ERR_INVALID_ARG and m is None
    st, m = afd.afd_ffn_mailbox_create(1, 1, 8, 0)          # the smallest valid mailbox
    assert st == afd.AFD_OK and m is not None
    afd.afd_ffn_mailbox_destroy(m)
    afd.afd_ffn_mailbox_destroy(None)


def test_producer_and_consumer_threads_round_trip():
    """A consumer thread doubles each micro-batch while the producer keeps every slot busy:
    the attention-side / FFN-side hand-off, with the outputs checked slot by slot."""
    n_slots, rounds, T, H = 3, 20, 8, 32
    mb = Mailbox(n_slots, T, H, pinned=False)
    errors = []

    def consumer():
        try:
            for _ in range(n_slots * rounds):
                st, slot, t = mb.take(5.0)
                assert st == afd.AFD_OK, st
                mb.output(slot)[:t].copy_(mb.input(slot)[:t] * 2)
                assert mb.complete(slot) == afd.AFD_OK
        except Exception as e:  # surfaced by the producer's assertion below
            errors.append(e)

    th = threading.Thread(target=consumer)
    th.start()
    try:
        for r in range(rounds):
            for s in range(n_slots):
                if r:
                    mb.wait(s, 5.0)
                    want = 2.0 * ((r - 1) * n_slots + s)
                    assert torch.all(mb.output(s)[: 1 + s] == want)
                mb.input(s)[: 1 + s].fill_(float(r * n_slots + s))
                mb.post(s, 1 + s)
        for s in range(n_slots):
            mb.wait(s, 5.0)
    finally:
        th.join(10.0)
        mb.close()
    assert not errors, errors


def test_write_input_copies_rows_and_checks_them(mb):
    rows = torch.arange(5 * 64, dtype=torch.float32).reshape(5, 64).to(torch.bfloat16)
    mb.write_input(2, rows)
    assert torch.equal(mb.input(2)[:5], rows) and float(mb.input(2)[5:].abs().sum()) == 0.0
    mb.write_input(0, rows[:0])                                     # T = 0 copies nothing
    with pytest.raises(IndexError):
        mb.write_input(3, rows)
    for bad in (rows.float(), rows.t(), rows[:, :32].contiguous(), torch.zeros(17, 64, dtype=torch.bfloat16)):
        with pytest.raises(ValueError):
            mb.write_input(0, bad)


class _NoDeviceLayer(afd.AfdFfn):
    """An AfdFfn shell with a stand-in handle value: only its close guard is exercised."""

    def __init__(self):
        self.h = 99


def test_a_running_service_keeps_its_layer_and_mailbox_open(monkeypatch):
    from ffn_side_expert_b200 import service
    stopped = []
    monkeypatch.setattr(service, "afd_ffn_service_start", lambda h, mb, stream=None: (afd.AFD_OK, 4242))
    monkeypatch.setattr(service, "afd_ffn_service_stop",
                        lambda svc: (stopped.append(svc), (afd.AFD_OK, afd.afd_ffn_service_stats(served=3)))[1])
    layer, m = _NoDeviceLayer(), Mailbox(2, 4, 64, pinned=False)
    try:
        svc = service.FfnService(layer, m)
        with pytest.raises(RuntimeError):
            m.close()
        with pytest.raises(RuntimeError):
            layer.close()
        assert svc.stop().served == 3 and stopped == [4242]
        assert svc.stop().served == 3 and stopped == [4242]          # a second stop does nothing
        assert m._served_by == 0 and layer._served_by == 0
        m.close()                                                      # allowed once stopped
    finally:
        layer.h = None                                                 # nothing real to destroy
        m.close()


def test_a_service_that_fails_to_start_holds_nothing(monkeypatch):
    from ffn_side_expert_b200 import service
    monkeypatch.setattr(service, "afd_ffn_service_start", lambda h, mb, stream=None: (afd.AFD_ERR_INVALID_ARG, None))
    layer, m = _NoDeviceLayer(), Mailbox(2, 4, 64, pinned=False)
    try:
        with pytest.raises(afd.AfdError):
            service.FfnService(layer, m)
        assert m._served_by == 0 and getattr(layer, "_served_by", 0) == 0
        m.close()
        with pytest.raises(ValueError):
            service.FfnService(layer, m)                               # a closed mailbox
    finally:
        layer.h = None
        m.close()

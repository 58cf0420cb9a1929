"""The FFN serving loop on the device: every micro-batch posted to the mailbox comes back equal,
bit for bit, to afd_ffn_forward of the same rows (the loop only moves bytes around the layer),
and within the bf16 bar of the fp64 oracle; the loop's start checks, its stop with slots in
flight, and the micro-pipeline ordering of the period (two slots in flight beat one)."""
import pytest
import torch

import bench
import ffn_side_expert_b200 as afd
import synth
from ffn_side_expert_b200.service import FfnService, Mailbox
from layer_support import BF16_TOL, Layer, rel_max_err, to64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", params=["tiny", "mid"])
def layer(request):
    L = Layer(synth.CONFIGS[request.param])
    yield L
    L.close()


def _forward(L, rows):
    T = rows.shape[0]
    out = torch.empty((max(T, 1), L.cfg.H), dtype=torch.bfloat16, device="cuda")
    L.mod.forward(rows.cuda(), out, T=T)
    torch.cuda.synchronize()
    return out[:T].cpu()


def test_served_outputs_equal_forward(layer):
    L, cfg = layer, layer.cfg
    g = torch.Generator().manual_seed(11)
    sizes = [cfg.T, 37, 0, 1, cfg.T - 3, cfg.T, 5, cfg.T]
    perms = [torch.randperm(cfg.T, generator=g)[:T] for T in sizes]
    batches = [L.hidden[p] for p in perms]
    refs = [_forward(L, b) for b in batches]
    mb = Mailbox(3, cfg.T, cfg.H)
    svc = FfnService(L.mod, mb)
    got = [None] * len(batches)
    try:
        in_slot = {}
        for i, b in enumerate(batches):
            s = i % 3
            if s in in_slot:
                mb.wait(s, 60.0)
                j = in_slot.pop(s)
                got[j] = mb.output(s)[: sizes[j]].clone()
            mb.write_input(s, b)
            mb.post(s, sizes[i])
            in_slot[s] = i
        for s, j in in_slot.items():
            mb.wait(s, 60.0)
            got[j] = mb.output(s)[: sizes[j]].clone()
    finally:
        stats = svc.stop()
        mb.close()
    assert stats.status == afd.AFD_OK and stats.device_status == afd.AFD_OK
    assert stats.served == len(batches)
    for i, (a, b) in enumerate(zip(got, refs)):
        assert torch.equal(a, b), f"micro-batch {i} (T={sizes[i]})"
    # and the first full micro-batch (a permutation of the seeded rows) against the oracle
    i = sizes.index(cfg.T)
    ref = L.oracle(tokens=perms[i].numpy())
    assert rel_max_err(to64(got[i]), ref["out"]) <= BF16_TOL


def test_start_checks(layer):
    L, cfg = layer, layer.cfg
    for T_max, H in ((cfg.T, cfg.H + 8), (cfg.T + 1, cfg.H)):
        m = Mailbox(2, T_max, H)
        try:
            assert afd.afd_ffn_service_start(L.mod.h, m.mb)[0] == afd.AFD_ERR_INVALID_ARG
        finally:
            m.close()
    m = Mailbox(2, cfg.T, cfg.H)
    try:
        svc = FfnService(L.mod, m)
        assert afd.afd_ffn_service_start(L.mod.h, m.mb)[0] == afd.AFD_ERR_INVALID_ARG   # one loop per mailbox
        assert svc.stop().status == afd.AFD_OK
        svc = FfnService(L.mod, m)                                                     # free again after stop
        assert svc.stop().served == 0
    finally:
        m.close()


def test_stop_with_slots_in_flight(layer):
    """Each posted slot either completes or fails with AFD_ERR_STOPPED; none is left hanging."""
    L, cfg = layer, layer.cfg
    m = Mailbox(4, cfg.T, cfg.H)
    svc = FfnService(L.mod, m)
    try:
        for s in range(4):
            m.write_input(s, L.hidden)
            m.post(s, cfg.T)
        stats = svc.stop()
        ends = [afd.afd_ffn_mailbox_wait(m.mb, s, 10_000_000) for s in range(4)]
    finally:
        m.close()
    assert stats.status == afd.AFD_OK
    assert all(e in (afd.AFD_OK, afd.AFD_ERR_STOPPED) for e in ends), ends
    assert stats.served == ends.count(afd.AFD_OK)


def test_two_slots_in_flight_overlap_attention_and_ffn(layer):
    """Attention stub of t_a per micro-batch on the host: with one slot the period is at least
    t_a + t_f; with two, the attention of one micro-batch overlaps the FFN of the other."""
    L, cfg = layer, layer.cfg
    if cfg.name != "mid":
        pytest.skip("timing on the larger workload only")
    ref = _forward(L, L.hidden)
    out = torch.empty_like(L.h)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(10):
        L.mod.forward(L.h, out)
    b.record()
    torch.cuda.synchronize()
    t_f = a.elapsed_time(b) / 10
    t_a = max(t_f, 0.5)
    p1, bad1, s1, _ = bench.pipeline_period(L.mod, L.hidden, cfg.T, t_a, 1, 12, ref)
    p2, bad2, s2, _ = bench.pipeline_period(L.mod, L.hidden, cfg.T, t_a, 2, 12, ref)
    assert bad1 == 0 and bad2 == 0
    assert s1.status == s2.status == afd.AFD_OK
    assert p1 >= 0.95 * (t_a + t_f), (p1, t_a, t_f)
    assert p2 < 0.8 * p1, (p1, p2, t_a, t_f)


def test_slot_timeline_is_ordered(layer):
    """The device timeline of a served micro-batch: H2D, then the layer, then D2H, in order."""
    L, cfg = layer, layer.cfg
    m = Mailbox(1, cfg.T, cfg.H)
    svc = FfnService(L.mod, m)
    try:
        for _ in range(2):
            m.write_input(0, L.hidden)
            m.post(0, cfg.T)
            m.wait(0, 60.0)
            t = svc.timeline(0)
            assert t[0] >= 0.0
            assert 0.0 <= t[1] <= t[2] <= t[3] <= t[4], t
            assert t[3] - t[2] > 0.0
        assert afd.afd_ffn_service_slot_timeline(svc.svc, 1)[0] == afd.AFD_ERR_INVALID_ARG
    finally:
        assert svc.stop().status == afd.AFD_OK
        m.close()

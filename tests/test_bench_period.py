"""The period models that bench.py --period reports beside its measurement (CPU only)."""
import random

import pytest

import bench


def test_one_slot_is_the_serial_sum_in_both_models():
    m = bench.period_models(1.5, 3.5, 0.1, 0.07, 1)
    assert m["page"] == pytest.approx(1.5 + 3.5 + 0.17)
    assert m["cycle"] == pytest.approx(m["page"])
    assert m["colocated"] == pytest.approx(5.0)


def test_two_slots_without_copies_reach_the_longer_stage():
    for t_a, t_f in ((1.0, 3.0), (3.0, 3.0), (4.0, 3.0)):
        m = bench.period_models(t_a, t_f, 0.0, 0.0, 2)
        assert m["page"] == pytest.approx(max(t_a, t_f))
        assert m["cycle"] == pytest.approx(max(t_a, t_f))


def test_balanced_stages_pay_half_the_copies_when_they_overlap():
    t, c = 3.5, 0.3
    m = bench.period_models(t, t, c / 2, c / 2, 2)
    assert m["page"] == pytest.approx(t + c)
    assert m["cycle"] == pytest.approx(t + c / 2)


def test_many_slots_hide_the_copies():
    m = bench.period_models(2.0, 3.0, 0.5, 0.5, 64)
    assert m["cycle"] == pytest.approx(3.0)


def test_cycle_bound_never_exceeds_the_page_model():
    rng = random.Random(5)
    for _ in range(1000):
        t_a, t_f, h, d = (rng.uniform(0, 5) for _ in range(4))
        for slots in (1, 2, 3, 8):
            m = bench.period_models(t_a, t_f, h, d, slots)
            assert m["cycle"] <= m["page"] + 1e-12
            assert m["cycle"] >= max(t_a, t_f) - 1e-12


def test_a_measured_point_carries_its_models():
    # the parts of the balanced two-slot point measured at the T=256 decode shape
    parts = {"post_to_take_ms": 0.0131, "take_to_landed_ms": 3.846, "period_mean_ms": 3.701,
             "h2d_ms": 0.096, "h2d_end_to_layer_ms": 0.008, "layer_ms": 3.501, "layer_gap_ms": 0.1712,
             "d2h_after_layer_ms": 0.079, "host_overhead_ms": 0.012}
    p = bench.period_point(3.4939, 2, 3.697, parts, 3.4939, 0.0842, 0.0705)
    assert p["model_ms"] == pytest.approx(3.4939 + 0.0842 + 0.0705, abs=1e-4)
    assert p["cycle_bound_in_loop_ms"] == pytest.approx((3.4939 + 0.096 + 3.501 + 0.079) / 2, abs=1e-4)
    assert p["colocated_ms"] == pytest.approx(2 * 3.4939, abs=1e-4)
    assert p["period_over_colocated"] == pytest.approx(3.697 / (2 * 3.4939), abs=1e-3)
    assert p["layer_gap_ms"] == 0.1712 and p["slots"] == 2

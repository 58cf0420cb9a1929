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

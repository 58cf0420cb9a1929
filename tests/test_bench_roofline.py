"""Host-side accounting of bench.py (CPU only): which peak bounds each workload's dominant
kernel, its algorithmic bytes and FLOPs, and the library launches per forward."""
import numpy as np

import bench
import synth


def _acct(name):
    cfg = synth.CONFIGS[name]
    counts = np.full(cfg.E, cfg.T * cfg.k // cfg.E)       # every routed expert touched
    return cfg, bench.algorithmic(cfg, counts)


def test_decode_shape_is_hbm_bound_on_the_expert_weights():
    cfg, acct = _acct("dsv3_256")
    assert acct["touched_experts"] == 257
    assert acct["weight_bytes"] == 257 * 3 * 7168 * 2048 * 2
    roof, path = bench.rooflines(cfg, acct, ms=3.5, kernel_ms=3.45)
    assert roof["bound"] == "hbm" and roof["unit"] == "GB/s"
    assert roof["algorithmic_bytes_per_launch"] == acct["weight_bytes"]   # weights only
    assert abs(roof["achieved"] - acct["weight_bytes"] / 3.45e-3 / 1e9) < 0.1
    assert path["t_hbm_ms"] > path["t_tensor_ms"]
    assert bench.launches_per_step(cfg) == 8


def test_w8a8_large_chunk_gate_up_is_tensor_bound():
    cfg, acct = _acct("w8a8_8192")
    roof, path = bench.rooflines(cfg, acct, ms=4.5, kernel_ms=2.3)
    rows = cfg.T * cfg.k + cfg.T
    assert roof["algorithmic_flops_per_launch"] == 4 * cfg.H * cfg.I * rows
    assert roof["bound"] == "tensor" and roof["unit"] == "TFLOP/s"
    assert roof["peak"] == 2 * bench.load_peaks()[0]["bf16_tflops"]         # e4m3 = 2 x bf16
    assert bench.launches_per_step(cfg) == 10


def test_bf16_large_micro_batch_gate_up_is_hbm_bound():
    cfg, acct = _acct("dsv3_4096")
    roof, _ = bench.rooflines(cfg, acct, ms=5.0, kernel_ms=2.7)
    assert roof["bound"] == "hbm"
    assert roof["algorithmic_bytes_per_launch"] == 257 * 2 * 2048 * 7168 * 2
    assert bench.launches_per_step(cfg) == 9


def test_clock_summary_keeps_only_the_timed_window(tmp_path):
    # lines written before the region (the sampler warming up) and after it are left out; the
    # last line before the region stands in when the region is shorter than one period
    import os
    f = open(tmp_path / "clk.csv", "w+")
    idle = "0, 1965, 1965, 200.0, 0x0, Not Active, Not Active, Not Active, Not Active"
    load = "0, 1320, 1965, 995.0, 0x4, Not Active, Not Active, Not Active, Active"
    f.write("\n".join([idle] * 10 + [load] * 3 + [idle] * 4) + "\n")
    f.flush()
    c = bench.ClockSampler(0)
    c.f, c.proc, c.first, c.last = f, object(), 10, 13
    s = c.summary()
    assert s["samples"] == 3 and s["sm_mhz"] == 1320.0 and s["sm_mhz_min"] == 1320.0
    assert s["reasons"] == ["sw_power_cap"] and s["power_w_max"] == 995.0
    assert not os.path.exists(tmp_path / "clk.csv")
    f = open(tmp_path / "clk2.csv", "w+")
    f.write("\n".join([idle] * 5 + [load]) + "\n")
    f.flush()
    c.f, c.first, c.last = f, 6, 6                           # no sample inside a short region
    s2 = c.summary()
    assert s2["samples"] == 1 and s2["sm_mhz"] == 1320.0


def test_shape_entry_carries_its_own_measurement():
    import argparse
    cfg, acct = _acct("w8a8_8192")
    r = {"cfg": cfg, "acct": acct, "ms": 4.3, "kernel_ms": 2.3, "stage_ms": np.linspace(0.01, 0.09, 9),
         "clocks": {"sm_mhz": 1800.0, "sm_max_mhz": 1965.0, "reasons": [], "samples": 5}}
    args = argparse.Namespace(steps=20, warmup=5)
    e = bench.report_shape(args, 1, r)
    assert set(e) >= {"value", "unit", "ms_per_step", "dtype", "config", "roofline", "path_roofline",
                      "stage_ms", "gpu_launches", "clocks"}
    assert abs(e["value"] - cfg.T / 4.3e-3) < 1.0 and e["dtype"] == "fp8_e4m3"
    assert e["config"]["workload"] == "w8a8_8192" and e["gpu_launches"] == 10 * 20
    assert e["roofline"]["bound"] == "tensor" and len(e["stage_ms"]) == 9

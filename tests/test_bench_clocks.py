"""The benchmark's clock evidence and the choice of its peak (CPU): samples
inside the timed window are aggregated (median SM clock, active reasons),
samples outside it are ignored, and a run held below its maximum clock by
the power cap is compared with the sustained bf16 peak, an unthrottled one
with the burst peak."""
import threading

import bench


def _sampler(samples, window, max_mhz=1965):
    s = bench.NvmlClockSampler("GPU-test")
    s.max_mhz = max_mhz
    s.samples = samples
    s.window = list(window)
    s.thread = threading.Thread(target=lambda: None)
    s.thread.start()
    return s


def test_power_capped_run_is_detected():
    # 30 samples at the maximum clock, then the cap (reason bit 0x4) holds
    # the clock at 1650 MHz; idle samples before the window do not count
    idle = [(0.1 + 0.002 * i, 345, 150.0, 0x1) for i in range(20)]
    load = [(1.0 + 0.002 * i, 1965 if i < 30 else 1650, 900.0, 0 if i < 30 else 0x4) for i in range(90)]
    c = _sampler(idle + load, (0.9, 2.0)).stop()
    assert c["samples"] == 90
    assert c["sm_mhz"] == 1650 and c["sm_mhz_min"] == 1650 and c["sm_max_mhz"] == 1965
    assert c["reasons"] == ["sw_power_cap"]
    assert c["sm_mhz_by_quarter"][0] == 1965 and c["sm_mhz_by_quarter"][-1] == 1650
    assert bench.power_capped(c)


def test_unthrottled_run_keeps_the_burst_peak():
    load = [(1.0 + 0.002 * i, 1965, 800.0, 0) for i in range(50)]
    c = _sampler(load, (0.9, 2.0)).stop()
    assert c["reasons"] == [] and not bench.power_capped(c)
    # the cap flagged but the clock still at its maximum: not a capped regime
    assert not bench.power_capped({"reasons": ["sw_power_cap"], "sm_mhz": 1965, "sm_mhz_min": 1965, "sm_max_mhz": 1965})
    assert not bench.power_capped(None)


def test_late_cap_counts_although_the_median_reads_the_maximum():
    # the clock readings trail the steps: three quarters of the samples still
    # read the maximum when the cap has already slowed the steps
    load = [(1.0 + 0.002 * i, 1965 if i < 90 else 1657, 450.0, 0x4 if i >= 80 else 0) for i in range(120)]
    c = _sampler(load, (0.9, 2.0)).stop()
    assert c["sm_mhz"] == 1965 and c["sm_mhz_min"] == 1657
    assert bench.power_capped(c)


def test_thermal_and_slowdown_reasons_are_named():
    load = [(1.0, 1500, 900.0, 0x8 | 0x20 | 0x40)]
    c = _sampler(load, (0.9, 2.0)).stop()
    assert c["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]


def test_no_samples_in_window_gives_none():
    c = _sampler([(0.1, 1965, 100.0, 0)], (0.9, 2.0)).stop()
    assert c is None

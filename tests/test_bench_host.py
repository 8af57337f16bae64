"""Host-side pieces of bench.py that decide whether a run is accepted: the clock / throttle
record taken during the timed region (a run that saw a hardware or thermal slowdown is
rejected, so the parser must report every active reason) and the workload names."""
import bench


class _FakeProc:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


def _sampler(lines):
    s = bench.ClockSampler(0)
    s.proc = _FakeProc()
    s.lines = list(lines)
    return s


def test_clock_record_reports_median_loaded_clock_power_and_active_reasons():
    # index, clocks.sm, clocks.max.sm, power.draw, active mask, hw, hw_thermal, sw_thermal, sw_power
    lines = [
        "0, 345, 1965, 150.2, 0x0, Not Active, Not Active, Not Active, Not Active",   # idle
        "0, 1650, 1965, 990.1, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1700, 1965, 995.0, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1680, 1965, 980.0, 0x0, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
    ]
    rec = _sampler(lines).stop()
    assert rec["sm_max_mhz"] == 1965.0
    assert rec["sm_mhz"] == 1680.0            # median of the loaded samples (idle one dropped)
    assert rec["reasons"] == ["sw_power_cap"]
    assert rec["samples"] == 4
    assert rec["power_w"] == (980.0 + 990.1) / 2


def test_clock_record_flags_hardware_and_thermal_slowdowns():
    lines = ["0, 1200, 1965, 700, 0x8, Active, Not Active, Active, Not Active",
             "0, 1300, 1965, 720, 0x8, Not Active, Active, Not Active, Not Active"]
    rec = _sampler(lines).stop()
    assert rec["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]


def test_clock_record_without_samples_is_none():
    assert _sampler([]).stop() is None
    s = bench.ClockSampler(0)                 # nvidia-smi could not be started
    assert s.stop() is None


def test_workload_names_the_step_it_times():
    w = bench._workload("480x480", 40)
    assert "480x480" in w and "40 layers" in w and "clean" in w

"""Host logic of bench.py that needs no GPU: the clock sampler's window filter."""
import bench


def _line(sm, reasons=("Not Active",) * 4):
    return ", ".join(["0", str(sm), "1965", "700.5", "0x0", *reasons])


def _sampler(samples, t0, t1):
    c = bench.ClockSampler("0")
    c.samples = samples
    c.t0, c.t1 = t0, t1
    return c


def test_clock_summary_keeps_only_the_timed_window():
    s = [(0.9, _line(900)), (1.05, _line(1900)), (1.10, _line(1800)), (1.15, _line(1700)), (1.3, _line(100))]
    out = _sampler(s, 1.0, 1.2).summary()
    assert out["samples"] == 3 and out["sm_mhz"] == 1800 and out["window"] == "inside"
    assert out["sm_max_mhz"] == 1965 and out["reasons"] == []


def test_clock_summary_short_window_takes_the_neighbours():
    s = [(0.9, _line(1950)), (1.5, _line(1930)), (2.0, _line(100))]
    out = _sampler(s, 1.0, 1.01).summary()
    assert out["window"] == "nearest" and out["samples"] == 2 and out["sm_mhz"] == 1940


def test_clock_summary_reports_throttle_reasons():
    active = ("Not Active", "Not Active", "Not Active", "Active")
    s = [(1.05, _line(1800, active)), (1.1, _line(1850))]
    out = _sampler(s, 1.0, 1.2).summary()
    assert out["reasons"] == ["sw_power_cap"]


def test_clock_summary_without_samples():
    out = _sampler([], 1.0, 2.0).summary()
    assert out["samples"] == 0 and out["sm_mhz"] is None and out["reasons"] == ["unavailable"]

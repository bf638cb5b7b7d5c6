"""The benchmark's clock record: median SM clock under load, max clock and
the throttle reasons seen Active, parsed from nvidia-smi's timestamped CSV
lines, restricted to the timed region."""
import time

import bench


LINE = "{ts}, 0, {sm}, 1965, 900.1, 0x{act:x}, {hw}, {hwt}, {swt}, {pc}"
T0 = time.mktime(time.strptime("2026/12/03 10:00:00", "%Y/%m/%d %H:%M:%S"))


def line(sm, hw="Not Active", hwt="Not Active", swt="Not Active", pc="Not Active", act=0, at=0.0):
    ts = time.strftime("%Y/%m/%d %H:%M:%S", time.localtime(T0 + int(at))) + f".{int(round((at % 1) * 1000)):03d}"
    return LINE.format(ts=ts, sm=sm, act=act, hw=hw, hwt=hwt, swt=swt, pc=pc)


def test_median_max_and_reasons():
    text = "\n".join([line(1965), line(1800, pc="Active", act=4), line(1905), line(1500)])
    c = bench.summarise_clocks(text)
    assert c == {"sm_mhz": 1852.5, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"],
                 "samples": 4}


def test_slowdowns_are_reported_and_bad_lines_skipped():
    text = "\n".join([line(1200, hw="Active", hwt="Active"), "garbage", "0, [N/A], 1965, 1, 0, a, b, c, d",
                      line(1300, swt="Active")])
    c = bench.summarise_clocks(text)
    assert c["samples"] == 2 and c["sm_mhz"] == 1250.0
    assert c["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]


def test_no_samples_is_none():
    assert bench.summarise_clocks("") is None
    assert bench.summarise_clocks("no gpu here\n") is None


def test_sampler_without_nvidia_smi_reports_nothing(monkeypatch):
    monkeypatch.setenv("PATH", "/nonexistent")
    s = bench.ClockSampler(0)
    s.start()
    assert s.stop() is None


def test_only_samples_inside_the_timed_region():
    text = "\n".join([line(1965, at=0.0), line(1700, pc="Active", act=4, at=0.52),
                      line(1650, pc="Active", act=4, at=0.54), line(1965, hw="Active", at=0.9)])
    c = bench.summarise_clocks(text, T0 + 0.5, T0 + 0.6)
    assert c == {"sm_mhz": 1675.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 2}


def test_short_region_takes_the_first_sample_after_its_start():
    text = "\n".join([line(1965, at=0.0), line(1800, at=0.30), line(1500, hw="Active", at=0.32)])
    c = bench.summarise_clocks(text, T0 + 0.21, T0 + 0.22)
    assert c["samples"] == 1 and c["sm_mhz"] == 1800.0 and c["reasons"] == []


def test_smi_timestamps():
    assert abs(bench._smi_time("2026/12/03 10:00:00.250") - (T0 + 0.25)) < 1e-6
    assert bench._smi_time("not a time") is None

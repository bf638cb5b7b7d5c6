"""The benchmark's clock record: median SM clock under load, max clock and
the throttle reasons seen Active, parsed from nvidia-smi's CSV lines."""
import bench


LINE = "0, {sm}, 1965, 900.1, 0x{act:x}, {hw}, {hwt}, {swt}, {pc}"


def line(sm, hw="Not Active", hwt="Not Active", swt="Not Active", pc="Not Active", act=0):
    return LINE.format(sm=sm, act=act, hw=hw, hwt=hwt, swt=swt, pc=pc)


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

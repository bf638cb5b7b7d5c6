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


class FakeNvml:
    """Stands in for pynvml: clocks and event-reason masks from a script."""
    NVML_CLOCK_SM = 1

    def __init__(self, samples, fail_init=False):
        self.samples, self.i, self.fail_init, self.shutdown = samples, 0, fail_init, False
        self.handle_by = None

    def nvmlInit(self):
        if self.fail_init:
            raise RuntimeError("no driver")

    def nvmlShutdown(self):
        self.shutdown = True

    def nvmlDeviceGetHandleByPciBusId(self, bus):
        self.handle_by = ("bus", bus)
        return "h"

    def nvmlDeviceGetHandleByIndex(self, idx):
        self.handle_by = ("index", idx)
        return "h"

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        return 1965

    def nvmlDeviceGetClockInfo(self, h, kind):
        return self.samples[min(self.i, len(self.samples) - 1)][0]

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        mask = self.samples[min(self.i, len(self.samples) - 1)][1]
        self.i += 1
        return mask


def test_nvml_sampler_reads_clocks_and_reasons():
    fake = FakeNvml([(1800, 0x4), (1700, 0x4 | 0x1), (1900, 0x0)])
    s = bench.NvmlClockSampler(0, b"00000000:1b:00.0", period=0.001, nvml=fake)
    assert s.start()
    import time
    while fake.i < 3:
        time.sleep(0.001)
    c = s.stop()
    assert fake.handle_by == ("bus", b"00000000:1b:00.0") and fake.shutdown
    assert c["sm_max_mhz"] == 1965.0 and c["reasons"] == ["sw_power_cap"] and c["samples"] >= 3
    assert 1700 <= c["sm_mhz"] <= 1900


def test_nvml_reason_bits():
    rows = [(1500.0, 1965.0, 0x8 | 0x40), (1600.0, 1965.0, 0x20), (1700.0, 1965.0, 0x2 | 0x1)]
    c = bench.summarise_nvml(rows)
    assert c == {"sm_mhz": 1600.0, "sm_max_mhz": 1965.0,
                 "reasons": ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"], "samples": 3}
    assert bench.summarise_nvml([]) is None


def test_nvml_sampler_without_nvml_reports_nothing():
    s = bench.NvmlClockSampler(0, nvml=FakeNvml([], fail_init=True))
    assert not s.start()
    assert s.stop() is None

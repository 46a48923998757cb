"""The bench's clock record against a fake NVML (no GPU, nothing set): samples inside the
timed region decide the median clock and the reasons; with none inside, all samples."""
import time

import bench


class FakeNvml:
    NVML_CLOCK_SM = 1

    def __init__(self, script):
        self.script = list(script)   # (sm MHz, reason bits) returned in turn, last one repeats
        self.i = 0

    def nvmlInit(self):
        pass

    def nvmlDeviceGetHandleByPciBusId(self, bus):
        raise RuntimeError("no such device")

    def nvmlDeviceGetHandleByIndex(self, index):
        return ("gpu", index)

    def nvmlDeviceGetClockInfo(self, handle, kind):
        sm = self.script[min(self.i, len(self.script) - 1)][0]
        return sm

    def nvmlDeviceGetMaxClockInfo(self, handle, kind):
        return 1965

    def nvmlDeviceGetCurrentClocksEventReasons(self, handle):
        bits = self.script[min(self.i, len(self.script) - 1)][1]
        self.i += 1
        return bits


def test_window_median_and_reasons():
    fake = FakeNvml([(1965, 0)] * 5 + [(1400, 0x4)] * 200)
    cs = bench.ClockSampler(0, interval=0.001, nvml=fake)
    while fake.i < 10:               # idle samples before the timed region
        time.sleep(0.001)
    cs.mark_start()
    time.sleep(0.05)
    cs.mark_end()
    rec = cs.stop()
    assert rec["source"] == "nvml" and rec["window"] == "timed region"
    assert rec["sm_mhz"] == 1400 and rec["sm_max_mhz"] == 1965
    assert rec["reasons"] == ["sw_power_cap"]


def test_reason_bits_and_fallback_to_all_samples():
    fake = FakeNvml([(1200, 0x4 | 0x8 | 0x40)])
    cs = bench.ClockSampler(0, interval=0.001, nvml=fake)
    time.sleep(0.02)
    rec = cs.stop()                  # never marked: every sample counts
    assert rec["window"] == "whole sampling period" and rec["samples"] >= 1
    assert rec["reasons"] == ["hw_slowdown", "hw_thermal_slowdown", "sw_power_cap"]

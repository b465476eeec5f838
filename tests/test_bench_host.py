"""Host-side pieces of bench.py that need no GPU.

* the clock sampler keeps only nvidia-smi samples taken inside the timed
  region and reports the throttle reasons seen there;
* the DRAM-traffic record is read from the committed ncu summaries only while
  the kernel's sources hash to the value the summary was taken on;
* the throughput arithmetic of the JSON line.
"""
import datetime
import json
import os
import sys
import time

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


class _FakeSmi:
    def __init__(self, out):
        self.out = out

    def terminate(self):
        pass

    def communicate(self, timeout=None):
        return self.out, None


def _line(t, sm, reasons=("Not Active",) * 4):
    ts = datetime.datetime.fromtimestamp(t).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
    return f"{ts}, 0, {sm}, 1965, 900.0, 0x0, " + ", ".join(reasons)


def test_clock_sampler_keeps_only_the_timed_window():
    now = time.time()
    capped = ("Not Active", "Not Active", "Not Active", "Active")
    lines = [_line(now - 2.0, 600),                  # idle, before the region
             _line(now + 0.1, 1900, capped),
             _line(now + 0.3, 1800, capped),
             _line(now + 0.5, 1700, capped),
             _line(now + 3.0, 300, ("Active", "Not Active", "Not Active", "Not Active"))]  # after it
    cs = bench.ClockSampler(0)
    cs.proc = _FakeSmi("\n".join(lines))
    cs.mark(now, now + 1.0)
    got = cs.stop()
    assert got == {"sm_mhz": 1800.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}


def test_clock_sampler_without_window_keeps_everything_and_flags_slowdown():
    now = time.time()
    lines = [_line(now, 1000, ("Active", "Not Active", "Not Active", "Not Active")), _line(now + 0.1, 1200)]
    cs = bench.ClockSampler(0)
    cs.proc = _FakeSmi("\n".join(lines) + "\nnot a sample line\n")
    got = cs.stop()
    assert got["samples"] == 2 and got["sm_mhz"] == 1100.0 and got["reasons"] == ["hw_slowdown"]


def test_clock_sampler_with_no_process():
    assert bench.ClockSampler(0).stop() is None


class _FakeNvml:
    """Read-only NVML stand-in: a clock that steps through `mhz` and the
    sw_power_cap reason bit from the third sample on."""
    NVML_CLOCK_SM = 1

    def __init__(self, mhz, fail_init=False):
        self.mhz, self.n, self.fail, self.calls = list(mhz), 0, fail_init, []

    def nvmlInit(self):
        if self.fail:
            raise RuntimeError("no NVML")

    def nvmlShutdown(self):
        self.calls.append("shutdown")

    def nvmlDeviceGetHandleByPciBusId(self, bus):
        self.calls.append(bus)
        return "h"

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        return 1965

    def nvmlDeviceGetClockInfo(self, h, kind):
        v = self.mhz[min(self.n, len(self.mhz) - 1)]
        self.n += 1
        return v

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return 0x4 if self.n >= 3 else 0


def test_nvml_clock_sampler_keeps_window_samples_and_reasons():
    nv = _FakeNvml([1965, 1965, 1800, 1700, 1700])
    cs = bench.NvmlClockSampler("00000000:1b:00.0", period_s=0.001, nvml=nv)
    t0 = time.time()
    assert cs.start()
    time.sleep(0.05)
    cs.mark(t0 - 1.0, time.time() + 1.0)
    got = cs.stop()
    assert nv.calls[0] == "00000000:1b:00.0" and nv.calls[-1] == "shutdown"
    assert got["samples"] >= 5 and got["sm_max_mhz"] == 1965.0 and got["sm_mhz"] == 1700.0
    assert got["reasons"] == ["sw_power_cap"] and got["source"].startswith("nvml")
    # a window that holds no sample gives no record
    cs2 = bench.NvmlClockSampler(None, period_s=0.001, nvml=_FakeNvml([1965]))
    cs2.nv.nvmlDeviceGetHandleByIndex = lambda i: "h"
    assert cs2.start()
    time.sleep(0.01)
    cs2.mark(0.0, 1.0)
    assert cs2.stop() is None


def test_nvml_clock_sampler_reports_failure_to_start():
    cs = bench.NvmlClockSampler("x", nvml=_FakeNvml([1], fail_init=True))
    assert cs.start() is False and cs.stop() is None


def test_traffic_record_follows_the_source_hash(tmp_path, monkeypatch):
    k = "fa_fwd_kernel"
    h = bench.kernel_source_hash(k)
    assert len(h) == 16 and h == bench.kernel_source_hash(k)
    rec = tmp_path / "dram_traffic.json"
    rec.write_text(json.dumps({"entries": [
        {"kernel": k, "workload": "wl", "source_hash": h, "read_bytes": 100, "write_bytes": 23},
        {"kernel": k, "workload": "wl2", "source_hash": "0000000000000000", "read_bytes": 1, "write_bytes": 1}]}))
    monkeypatch.setattr(bench, "TRAFFIC_RECORD", str(rec))
    assert bench.recorded_traffic(k, "wl") == 123
    assert bench.recorded_traffic(k, "wl2") is None        # taken on other sources
    assert bench.recorded_traffic(k, "other") is None
    assert bench.recorded_traffic("fa_bwd_dq_kernel", "wl") is None
    monkeypatch.setattr(bench, "TRAFFIC_RECORD", str(tmp_path / "missing.json"))
    assert bench.recorded_traffic(k, "wl") is None


def test_committed_traffic_record_parses():
    # every entry of the committed record names a known kernel and integer byte counts
    with open(os.path.join(ROOT, "profiles", "dram_traffic.json")) as f:
        entries = json.load(f)["entries"]
    for e in entries:
        assert e["kernel"] in bench.KERNEL_FILES and len(e["source_hash"]) == 16
        int(e["read_bytes"]), int(e["write_bytes"])
    assert len(entries) >= 6


@pytest.mark.parametrize("ws", [1, 2, 8])
def test_job_throughput_counts_every_rank(ws):
    # flops of one step on each rank, over the slowest rank's time
    assert bench.job_tflops(2e12, ws, 4.0) == pytest.approx(ws * 2e12 / 4e-3 / 1e12)

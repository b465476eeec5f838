"""Host-side pieces of bench.py that need no GPU.

* the clock sampler keeps only nvidia-smi samples taken inside the timed
  region and reports the throttle reasons seen there;
* the DRAM-traffic record is read from the committed ncu summaries only while
  the kernel's sources hash to the value the summary was taken on;
* the throughput arithmetic of the JSON line.
"""
import datetime
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


def test_traffic_record_follows_the_source_hash(tmp_path, monkeypatch):
    k = "fa_fwd_kernel"
    h = bench.kernel_source_hash(k)
    assert len(h) == 16 and h == bench.kernel_source_hash(k)
    summary = tmp_path / "dram_traffic_x.md"
    summary.write_text("| kernel | workload | source hash | read bytes | write bytes | ns |\n|---|---|---|---|---|---|\n"
                       f"| {k} | wl | {h} | 100 | 23 | 5 |\n| {k} | wl2 | 0000000000000000 | 1 | 1 | 1 |\n")
    monkeypatch.setattr(bench, "TRAFFIC_GLOB", str(tmp_path / "dram_traffic_*.md"))
    assert bench.recorded_traffic(k, "wl") == 123
    assert bench.recorded_traffic(k, "wl2") is None        # taken on other sources
    assert bench.recorded_traffic(k, "other") is None
    assert bench.recorded_traffic("fa_bwd_dq_kernel", "wl") is None


def test_committed_traffic_records_parse():
    # every row of the committed summaries names a known kernel and integer byte counts
    import glob
    rows = 0
    for path in glob.glob(os.path.join(ROOT, "profiles", "dram_traffic_*.md")):
        for line in open(path):
            cells = [c.strip() for c in line.strip().strip("|").split("|")]
            if len(cells) >= 6 and cells[0] in bench.KERNEL_FILES and len(cells[2]) == 16:
                int(cells[3]), int(cells[4])
                rows += 1
    assert rows >= 6


@pytest.mark.parametrize("ws", [1, 2, 8])
def test_job_throughput_counts_every_rank(ws):
    # flops of one step on each rank, over the slowest rank's time
    assert bench.job_tflops(2e12, ws, 4.0) == pytest.approx(ws * 2e12 / 4e-3 / 1e12)

"""bench.py's clock record, on the CPU with a stand-in nvidia-smi: only the
samples taken while the timed region runs count toward the median SM clock
and the throttle reasons; the samples of the idle lead-in before it do not."""

import os
import stat
import sys
import time

import bench

FAKE_SMI = """#!{python}
import os, sys, time
while True:
    busy = os.path.exists({flag!r})
    sys.stdout.write("0, %d, 1965, 500.00, 0x0, Not Active, Not Active, Not Active, %s\\n"
                     % (1700 if busy else 1965, "Active" if busy else "Not Active"))
    sys.stdout.flush()
    time.sleep(0.02)
"""


def _install_fake_smi(tmp_path, monkeypatch, flag):
    path = tmp_path / "nvidia-smi"
    path.write_text(FAKE_SMI.format(python=sys.executable, flag=str(flag)))
    path.chmod(path.stat().st_mode | stat.S_IXUSR)
    monkeypatch.setenv("PATH", str(tmp_path) + os.pathsep + os.environ.get("PATH", ""))


def test_median_and_reasons_come_from_the_timed_region(tmp_path, monkeypatch):
    flag = tmp_path / "busy"
    _install_fake_smi(tmp_path, monkeypatch, flag)
    clocks = bench.ClockSampler(0)
    clocks.start()
    deadline = time.time() + 30
    while len(clocks.lines) < 10 and time.time() < deadline:  # idle samples before the region
        time.sleep(0.02)
    flag.touch()  # the stand-in reports loaded clocks from here on
    time.sleep(0.1)
    clocks.mark_start()
    time.sleep(0.3)
    clocks.mark_stop()
    clk = clocks.stop()
    assert clk["window"] == "samples that arrived during the timed region"
    assert clk["samples"] >= 5 and clk["samples_total"] > clk["samples"] + 5
    assert clk["sm_mhz"] == 1700.0 and clk["sm_max_mhz"] == 1965.0
    assert clk["reasons"] == ["sw_power_cap"]


def test_all_samples_when_none_arrived_in_the_region():
    lines = [(10.0, "0, 1965, 1965, 100.00, 0x0, Not Active, Not Active, Not Active, Not Active"),
             (10.2, "0, 1800, 1965, 900.00, 0x4, Not Active, Not Active, Not Active, Active"),
             (10.4, "0, 1700, 1965, 900.00, 0x4, Not Active, Not Active, Not Active, Active"),
             (10.5, "not a sample line")]
    clk = bench.ClockSampler.summarise(lines, 11.0, 11.1)
    assert clk["window"] == "all samples (none arrived during the timed region)"
    assert clk["samples"] == 3 and clk["sm_mhz"] == 1800.0 and clk["reasons"] == ["sw_power_cap"]
    inside = bench.ClockSampler.summarise(lines, 10.1, 10.45)
    assert inside["samples"] == 2 and inside["sm_mhz"] == 1750.0 and inside["samples_total"] == 3
    empty = bench.ClockSampler.summarise([], None, None)
    assert empty["sm_mhz"] is None and empty["samples"] == 0

"""Host-side pieces of the benchmark that need no GPU: the clock sampler, fed by a fake
nvidia-smi, writes where BITLINEAR_BENCH_OUT points and reports the median SM clock and
the throttle reasons it saw."""
import os
import stat
import sys
import time

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

pytestmark = pytest.mark.cpu

FAKE_SMI = """#!/bin/sh
echo "0, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active"
echo "0, 1800, 1965, 990.5, 0x4, Not Active, Not Active, Not Active, Active"
echo "0, 1900, 1965, 980.0, 0x4, Not Active, Not Active, Not Active, Active"
exec sleep 30
"""


def test_clock_sampler_with_fake_nvidia_smi(tmp_path, monkeypatch):
    import bench
    bindir = tmp_path / "bin"
    bindir.mkdir()
    smi = bindir / "nvidia-smi"
    smi.write_text(FAKE_SMI)
    smi.chmod(smi.stat().st_mode | stat.S_IEXEC)
    out = tmp_path / "out"
    monkeypatch.setenv("PATH", str(bindir) + os.pathsep + os.environ["PATH"])
    monkeypatch.setenv("BITLINEAR_BENCH_OUT", str(out))
    cs = bench.ClockSampler(0)
    cs.start()
    assert cs.path == str(out / "clocks_rank0.csv")
    for _ in range(100):  # wait for the three lines
        if os.path.exists(cs.path) and open(cs.path).read().count("\n") >= 3:
            break
        time.sleep(0.05)
    rec = cs.stop()
    assert rec == {"sm_mhz": 1900.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}


def test_clock_sampler_without_nvidia_smi(tmp_path, monkeypatch):
    import bench
    monkeypatch.setenv("PATH", str(tmp_path))
    monkeypatch.setenv("BITLINEAR_BENCH_OUT", str(tmp_path / "o"))
    cs = bench.ClockSampler(0)
    cs.start()
    assert cs.stop() is None

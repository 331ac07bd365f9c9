"""Host logic of bench.py that needs no GPU: the clock / throttle-reason sampler
that brackets the timed region, driven here by a stand-in `nvidia-smi` that
prints fixed CSV rows in the format the sampler queries."""
import os
import stat
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _fake_smi(tmp_path, rows):
    """A stand-in nvidia-smi that prints `rows` (cycling) every 20 ms until killed."""
    script = tmp_path / "nvidia-smi"
    body = "\n".join(f'  echo "{r}"; sleep 0.02' for r in rows)
    script.write_text(f"#!/bin/bash\nwhile true; do\n{body}\ndone\n")
    script.chmod(script.stat().st_mode | stat.S_IEXEC)
    return str(tmp_path)


def test_sampler_reads_clocks_and_reasons(tmp_path, monkeypatch):
    rows = [
        "0, 1800, 1965, 700.0, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1900, 1965, 650.0, 0x0, Not Active, Not Active, Not Active, Not Active",
        "0, 1700, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active",
    ]
    monkeypatch.setenv("PATH", _fake_smi(tmp_path, rows) + os.pathsep + os.environ["PATH"])
    c = bench.ClockSampler(0)
    t0 = time.perf_counter()
    c.start()
    assert c.lines, "start() returns only once the first sample is in"
    assert time.perf_counter() - t0 < 5.0
    time.sleep(0.3)
    out = c.stop()
    assert out["samples"] >= 3
    assert out["sm_max_mhz"] == 1965.0
    assert out["sm_mhz_min"] == 1700.0
    assert 1700.0 <= out["sm_mhz"] <= 1900.0
    assert out["reasons"] == ["sw_power_cap"]
    assert c.proc.poll() is not None  # the sampler process has ended


def test_sampler_reports_slowdown_reasons(tmp_path, monkeypatch):
    rows = ["0, 1200, 1965, 400.0, 0x48, Active, Active, Not Active, Not Active"]
    monkeypatch.setenv("PATH", _fake_smi(tmp_path, rows) + os.pathsep + os.environ["PATH"])
    c = bench.ClockSampler(0)
    c.start()
    time.sleep(0.1)
    out = c.stop()
    assert out["reasons"] == ["hw_slowdown", "hw_thermal_slowdown"]
    assert out["sm_mhz"] == 1200.0


def test_sampler_without_nvidia_smi(tmp_path, monkeypatch):
    monkeypatch.setenv("PATH", str(tmp_path))  # an empty folder: no nvidia-smi to start
    c = bench.ClockSampler(0)
    c.start(wait_s=0.5)
    out = c.stop()
    assert out["sm_mhz"] is None and out["reasons"] == ["nvidia-smi unavailable"]

"""bench.py's clock record: samples are kept by their nvidia-smi timestamp when
they fall inside the timed region, else the one nearest to it; throttle
reasons are read from the kept samples only."""

import datetime
import os
import sys
import tempfile

sys.path.insert(0, os.path.join(os.path.dirname(__file__), ".."))
import bench  # noqa: E402


class _Done:
    def terminate(self):
        pass

    def wait(self, timeout=None):
        return 0


def _sampler(rows, t0, t1):
    cs = bench.ClockSampler.__new__(bench.ClockSampler)
    cs.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
    for when, mhz, slow, pcap in rows:
        stamp = datetime.datetime.fromtimestamp(when).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
        cs.f.write("%s, 0, %d, 1965, 700.0, 0x0, %s, Not Active, Not Active, %s\n"
                   % (stamp, mhz, slow, pcap))
    cs.f.flush()
    cs.p = _Done()
    cs.t0, cs.t1 = t0, t1
    return cs


def test_samples_inside_the_region():
    T = 1_800_000_000.0
    rows = [(T - 0.10, 900, "Active", "Not Active"),   # before: a slowdown that must not count
            (T + 0.05, 1900, "Not Active", "Active"),
            (T + 0.10, 1880, "Not Active", "Active"),
            (T + 0.15, 1960, "Not Active", "Not Active"),
            (T + 0.40, 700, "Active", "Not Active")]   # after
    out = _sampler(rows, T, T + 0.2).stop()
    assert out["samples"] == 3
    assert out["sm_mhz"] == 1900
    assert out["reasons"] == ["sw_power_cap"]
    assert out["sm_max_mhz"] == 1965
    assert out["window_ms"] == 200.0


def test_nearest_sample_when_the_region_is_short():
    T = 1_800_000_000.0
    rows = [(T - 0.20, 1000, "Not Active", "Not Active"),
            (T + 0.06, 1950, "Not Active", "Not Active"),
            (T + 0.30, 1200, "Active", "Not Active")]
    out = _sampler(rows, T, T + 0.02).stop()
    assert out["samples"] == 0
    assert out["sm_mhz"] == 1950 and out["reasons"] == []


def test_a_short_run_waits_for_the_first_sample(tmp_path, monkeypatch):
    """nvidia-smi can take longer to print its first sample than a short timed run
    lasts: the sampler waits (at most 5 s) for it before the warm-up, so the record
    is never empty."""
    fake = tmp_path / "nvidia-smi"
    fake.write_text("#!/bin/sh\nsleep 0.5\nwhile true; do\n"
                    "  echo '2026/12/03 12:00:00.000, 0, 1965, 1965, 700.0, 0x0, Not Active, Not Active, "
                    "Not Active, Not Active'\n  sleep 0.05\ndone\n")
    fake.chmod(0o755)
    monkeypatch.setenv("PATH", str(tmp_path) + os.pathsep + os.environ.get("PATH", ""))
    cs = bench.ClockSampler("0")
    assert os.path.getsize(cs.f.name) > 0
    cs.begin()
    cs.end()
    out = cs.stop()
    assert out is not None and out["sm_mhz"] == 1965 and out["reasons"] == []

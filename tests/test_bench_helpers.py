"""bench.py's host-side helpers, on the CPU: the clock summary taken from
nvidia-smi samples, and the lookup of the attention kernel's DRAM traffic in the
ncu summaries under profiles/ (valid only for the kernel source it was taken on).
"""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


class _DoneProc:
    def send_signal(self, sig):
        pass

    def wait(self, timeout=None):
        return 0


def _summary(tmp_path, text):
    path = tmp_path / "clocks.csv"
    path.write_text(text)
    s = bench.ClockSampler(0)
    s.proc, s.path = _DoneProc(), str(path)
    return s.stop()


def test_clock_summary_median_max_and_reasons(tmp_path):
    rows = [
        "0, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active",
        "0, 1800, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1900, 1965, 980.0, 0x4, Not Active, Not Active, Not Active, Active",
        "garbage line",
        "0, [N/A], 1965, 0, 0x0, Not Active, Not Active, Not Active, Not Active",
    ]
    c = _summary(tmp_path, "\n".join(rows) + "\n")
    assert c == dict(sm_mhz=1900.0, sm_max_mhz=1965.0, samples=3, reasons=["sw_power_cap"])
    assert not os.path.exists(tmp_path / "clocks.csv")   # the sample file is removed


def test_clock_summary_reports_thermal_slowdown(tmp_path):
    c = _summary(tmp_path, "0, 1500, 1965, 1000, 0x20, Not Active, Active, Not Active, Not Active\n")
    assert c["reasons"] == ["hw_thermal_slowdown"] and c["samples"] == 1


def test_clock_summary_without_samples(tmp_path):
    assert _summary(tmp_path, "") is None
    assert bench.ClockSampler(0).stop() is None   # never started


def test_traffic_is_read_only_for_the_profiled_kernel_source(monkeypatch):
    lines = []
    for name in sorted(os.listdir(os.path.join(ROOT, "profiles"))):
        if name.endswith(".md"):
            lines += bench.TRAFFIC_LINE.findall(open(os.path.join(ROOT, "profiles", name)).read())
    assert lines, "no traffic line under profiles/"
    workload, sha, nbytes = lines[0]
    monkeypatch.setattr(bench, "kernel_sha", lambda: sha)
    assert bench.profiled_traffic(workload) == int(nbytes)
    assert bench.profiled_traffic("no-such-workload") is None
    monkeypatch.setattr(bench, "kernel_sha", lambda: "0" * 16)   # the kernel changed since
    assert bench.profiled_traffic(workload) is None


def test_kernel_sha_follows_the_attention_sources():
    sha = bench.kernel_sha()
    assert len(sha) == 16 and int(sha, 16) >= 0
    assert bench.kernel_sha() == sha

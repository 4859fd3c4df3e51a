"""bench.py end to end on the smallest workload, every selection mode (needs a B200).

Checks that the one JSON line carries the keys the measurement contract asks
for, with sane values; the full-size numbers come from the benchmark itself.
"""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("selection", ["top_p", "eg", "sampled"])
def test_bench_line(selection):
    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--workload", "tiny", "--steps", "2",
           "--warmup", "3", "--no-cpu-baseline", "--selection", selection]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "roofline",
                "gpu_launches", "clocks", "e2e"):
        assert key in line, key
    assert line["value"] > 0 and line["ms_per_step"] > 0
    assert line["roofline"]["bound"] == "tensor" and line["roofline"]["achieved"] > 0
    assert 0 < line["config"]["density"] <= 1
    assert line["gpu_launches"] == 2 * {"top_p": 5, "eg": 9, "sampled": 4}[selection]
    if selection == "top_p":
        assert line["e2e"]["value"] > 0 and line["e2e"]["h2d_bytes_per_step"] > 0
    doms = line["competition_domains"]
    assert set(doms) == {"per_row", "per_head", "grouped", "all_head", "eg_sparse", "call"}
    for name in ("per_row", "per_head", "grouped", "all_head", "eg_sparse"):
        assert doms[name]["ms"] > 0 and 0 < doms[name]["density"] <= 1
    assert doms["per_row"]["pooled_heads"] == 0 and doms["all_head"]["pooled_heads"] == line["config"]["heads"]

"""The benchmark's JSON line on a real GPU: one line from `python bench.py` with
the keys the measurement contract names (metric, value, roofline of the decode
kernel, end-to-end throughput with host buffers, the CPU oracle's baseline,
clock samples from inside the timed region), on the small fp32 workload so the
run takes seconds."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_bench_prints_one_complete_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--config", "1", "--steps", "3", "--warmup",
                        "3", "--no-sweep", "--no-diagnostics", "--cpu-groups", "2"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "dtype", "data", "config", "roofline", "e2e", "cpu_baseline", "clocks", "gpu_launches"):
        assert key in d, key
    assert d["steps"] == 3 and d["warmup"] == 3 and d["n_gpus"] == 1 and d["value"] > 0
    assert d["config"]["workload"] == "tiny-f32-mha2-d64-n1024-b16"
    roof = d["roofline"]
    assert roof["bound"] == "hbm" and roof["unit"] == "GB/s" and roof["achieved"] > 0
    assert roof["frac"] == pytest.approx(roof["achieved"] / roof["peak"])
    e2e = d["e2e"]
    assert e2e["value"] > 0 and e2e["h2d_bytes_per_step"] > 0 and e2e["d2h_bytes_per_step"] > 0
    cpu = d["cpu_baseline"]
    assert cpu["kind"] == "oracle" and cpu["cores"] >= 1 and cpu["value"] > 0
    assert d["clocks"] is not None and d["clocks"]["samples"] >= 1
    assert d["gpu_launches"] == 2 * d["steps"]

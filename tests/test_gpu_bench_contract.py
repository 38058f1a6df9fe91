"""bench.py on a GPU prints exactly one JSON line with the keys and types the
benchmark contract asks for (small workload, a few steps)."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_bench(*args):
    out = subprocess.run([sys.executable, "bench.py", *args], cwd=ROOT, capture_output=True,
                         text=True, timeout=600, check=True)
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1, out.stdout
    return json.loads(lines[0])


@pytest.mark.parametrize("launch", ["graph", "eager"])
def test_bench_line_keeps_the_contract(launch):
    d = run_bench("--workload", "1", "--steps", "4", "--warmup", "3", "--launch", launch,
                  "--cpu-seconds", "1")
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "roofline", "e2e", "gpu_launches", "clocks", "cpu_baseline"):
        assert key in d, key
    assert d["n_gpus"] == 1 and d["steps"] == 4 and d["warmup"] == 3
    assert d["value"] > 0 and d["unit"] == "tokens/s" and d["higher_is_better"] is True
    assert d["scaling"] == "weak" and d["vs_baseline"] is None
    assert d["gpu_launches"] == 2 * 4   # origin scan + rotation per step
    assert d["config"]["step"] == "one-call" and d["positions_avg_ms"] is None
    assert "workload" in d["config"]
    r = d["roofline"]
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["peak"] > 0
    assert abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-9
    assert r["kernel"] == "rotate_qk_kernel" and r["spec_peak"] == 8000.0
    e = d["e2e"]
    assert e["value"] > 0 and e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
    c = d["cpu_baseline"]
    assert c["kind"] == "oracle" and c["cores"] >= 1 and c["value"] > 0
    assert set(d["clocks"]) >= {"sm_mhz", "sm_max_mhz", "reasons"}


def test_decode_and_cache_forms():
    d = run_bench("--workload", "4", "--steps", "4", "--warmup", "3", "--no-cpu-baseline")
    assert d["gpu_launches"] == 4 and d["value"] > 0    # one launch per decode step
    d = run_bench("--workload", "2", "--op", "cache", "--steps", "4", "--warmup", "3",
                  "--no-cpu-baseline")
    assert d["roofline"]["kernel"] == "rotate_qk_cache_kernel" and "skipped" in d["e2e"]


def test_separate_step_and_the_copy_pattern_probe():
    d = run_bench("--workload", "2", "--step", "separate", "--steps", "4", "--warmup", "3",
                  "--no-cpu-baseline")
    assert d["config"]["step"] == "separate" and d["gpu_launches"] == 3 * 4
    assert d["positions_avg_ms"] > 0
    d = run_bench("--probe", "copy-pattern", "--workload", "2", "--steps", "5", "--warmup", "3")
    assert d["probe"] == "copy-pattern" and d["gbs"] > 0 and d["launches"] == 5

"""bench.py on a GPU prints exactly one JSON line with the keys and types the
benchmark contract asks for (small workload, a few steps)."""
import json
import os
import subprocess
import sys

import pytest

import bench

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


@pytest.mark.parametrize("op", ["frames", "chunk"])
def test_planes_ops(op):
    d = run_bench("--op", op, "--prompts", "16", "--rule", "qwen_vl", "--steps", "4",
                  "--warmup", "3", "--cpu-seconds", "1")
    assert d["value"] > 0 and d["config"]["op"] == op and d["config"]["global_batch"] == 16 * 65536
    assert d["gpu_launches"] == (2 if op == "frames" else 2 * 4) * 4
    r = d["roofline"]
    assert r["bound"] == "hbm" and abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-9
    assert "skipped" in d["e2e"] and d["cpu_baseline"]["kind"] == "oracle"
    assert r["same_size_fill_gbs"] > 0 and r["planes_store_gbs"] > 0
    assert abs(r["planes_frac_of_fill"] - r["planes_store_gbs"] / r["same_size_fill_gbs"]) < 1e-9
    if op == "chunk":
        # planes, the ids up to each prompt's first marker (one thumbnail each), the state
        n = 16 * 65536
        assert bench.chunk_bytes(n, 16, 4, 16) < r["algorithmic_bytes_per_launch"]
        assert r["algorithmic_bytes_per_launch"] < bench.chunk_bytes(n, 16, 4, n)


@pytest.mark.parametrize("rule", ["canvas", "qwen_vl", "planes_1d"])
def test_the_chunk_step_equals_the_oracle(cuda_device, rule):
    # the chunk op's calls as bench.py makes them (no offset or state for the
    # first chunk, two state buffers in turn): every plane and the state after
    # each chunk equal the oracle's, bit for bit
    import numpy as np
    import torch

    import oracle
    from vlm_decoder_positional_b200 import cmr, inputs
    dev = cuda_device
    wl = inputs.make_frames_workload(num_prompts=16, frames=1, seed=77)
    pieces = bench.chunk_pieces(wl.ids, wl.cu_seqlens, 8)
    states = [(torch.empty(16, dtype=torch.int32, device=dev),
               torch.empty(16, dtype=torch.int32, device=dev)) for _ in range(2)]
    o_state = (None, None)
    for c, (ids_c, cu_c, off_c) in enumerate(pieces):
        g = [torch.from_numpy(a).to(dev) for a in (ids_c, cu_c, off_c)]
        pos = torch.empty((3, ids_c.shape[0]), dtype=torch.int32, device=dev)
        cmr.positions_chunk(g[0], g[1], pos_offset=g[2] if c else None,
                            state=states[(c + 1) % 2] if c else None, rule=rule,
                            out=(pos, *states[c % 2]))
        torch.cuda.synchronize()
        want, ws, wa = oracle.positions_chunk(ids_c, cu_c, wl.image_token_id, rule, off_c,
                                              *o_state)
        np.testing.assert_array_equal(pos.cpu().numpy(), want)
        np.testing.assert_array_equal(states[c % 2][0].cpu().numpy(), ws)
        np.testing.assert_array_equal(states[c % 2][1].cpu().numpy(), wa)
        o_state = (ws, wa)

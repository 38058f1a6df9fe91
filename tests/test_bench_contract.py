"""bench.py's host-side pieces: algorithmic byte counts, the traffic record,
and the reference (oracle) arm's JSON line, all on CPU."""
import json
import os
import subprocess
import sys

import bench
from vlm_decoder_positional_b200 import inputs

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_algorithmic_bytes_match_the_hand_count():
    # 2,560 B per token-layer for 8 Q + 2 K heads x 64 dims x bf16 x (read + write)
    assert bench.rotate_bytes(1, 1, 8, 2, 64) == 2560 + 12
    assert bench.rotate_bytes(262144, 6, 8, 2, 64) == 4_026_531_840 + 3_145_728
    assert bench.positions_bytes(262144, 32) == 262144 * 16 + 32 * 12
    # rotate + KV cache, 8 Q + 2 KV heads of 256: Q's 64 dims read and written
    # (2,048 B), K and V rows read (2,048 B), their cache rows written (2,048 B)
    assert bench.cache_bytes(1, 1, 8, 2, 64, 256) == 6144
    assert bench.cache_bytes(262144, 6, 8, 2, 64, 256) == 9_663_676_416


def test_traffic_record_is_tied_to_the_kernel_source_and_workload():
    t = bench.recorded_traffic("c5_6layers_32x8192", "rotate_qk_staged_kernel")
    assert t is None or 3.5e9 < t < 4.5e9
    assert bench.recorded_traffic("some_other_workload") is None
    assert bench.recorded_traffic("c5_6layers_32x8192", "rotate_qk_kernel") is None


def test_source_hash_ignores_comments_but_not_code():
    src = {rel: open(os.path.join(bench.ROOT, rel)).read() for rel in bench.ROTATE_SOURCES}
    base = bench.rotate_source_hash(src.__getitem__)
    assert base == bench.rotate_source_hash()
    rel = "vlm_decoder_positional_b200/csrc/rotate.cu"
    commented = dict(src)
    commented[rel] = "// a new remark\n" + src[rel].replace("\n", "\n  /* note */\n", 3)
    assert bench.rotate_source_hash(commented.__getitem__) == base
    changed = dict(src)
    changed[rel] = src[rel].replace("kOneShotRows = 16", "kOneShotRows = 17")
    assert changed[rel] != src[rel]
    assert bench.rotate_source_hash(changed.__getitem__) != base
    # a "//" inside a string literal is code, not a comment
    assert bench.code_tokens('f("a//b"); // c') == 'f("a//b");'


def test_host_cpu_record():
    h = bench.host_cpu()
    assert h["nproc"] == os.cpu_count() and h["threads_allowed"] == bench.host_cores()
    assert h["cpu_model"] is None or isinstance(h["cpu_model"], str)


def test_oracle_sample_step_threads_agree():
    wl = inputs.make_config(2)
    wl_cpu = bench.cpu_sample_inputs(wl, 600)
    assert bench.oracle_sample_step(wl_cpu, 600, threads=1) == 600
    assert bench.oracle_sample_step(wl_cpu, 600, threads=4) == 600
    assert "16 prompts" not in bench.sample_label(wl, 600)


def test_reference_arm_prints_one_json_line():
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--workload", "1",
                          "--steps", "3", "--warmup", "3", "--reference-budget-s", "2"],
                         cwd=ROOT, capture_output=True, text=True, timeout=300, check=True)
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["metric"] == bench.METRIC and d["higher_is_better"] is True
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    host = d["cpu_baseline"]["host"]
    assert host["nproc"] >= 1 and host["threads_allowed"] >= 1 and "cpu_model" in host
    # the same config keys (and workload) as the GPU arm's line
    assert set(d["config"]) == {"workload", "global_batch", "launch", "op", "step", "seq_len",
                                "parallelism", "l2"}
    assert d["config"]["workload"].startswith("c1_single_prompt_80: 1 prompts x 80 tokens")
    assert d["config"]["global_batch"] == 80

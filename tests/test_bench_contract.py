"""bench.py's host-side pieces: algorithmic byte counts, the traffic record,
and the reference (oracle) arm's JSON line, all on CPU."""
import json
import os
import subprocess
import sys

import numpy as np
import pytest

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


def test_chunk_bytes_hand_count():
    # 12 B of planes per token, 4 B per id the rule reads; per prompt 12 B for
    # the first call and 24 B for each later one
    assert bench.chunk_bytes(1000, 2, 1, 1000) == bench.positions_bytes(1000, 2)
    assert bench.chunk_bytes(262144, 4, 4, 0) == 262144 * 12 + 4 * (12 + 3 * 24)
    assert bench.chunk_bytes(262144, 4, 4, 10) == 262144 * 12 + 40 + 4 * (12 + 3 * 24)


def test_first_marker_reads():
    m = inputs.IMAGE_TOKEN_ID
    ids = np.array([1, 2, m, 3, m,   m, 5,   7, 8, 9,   4], np.int32)
    cu = np.array([0, 5, 7, 10, 10, 11], np.int32)   # marker at 2; at 0; none; empty; none
    assert bench.first_marker_reads(ids, cu, m, "canvas") == 3 + 1 + 3 + 0 + 1
    assert bench.first_marker_reads(ids, cu, m, "qwen_vl") == 8
    assert bench.first_marker_reads(ids, cu, m, "planes_1d") == 0


def test_chunk_pieces_cover_every_token_once():
    rng = np.random.default_rng(5)
    ids = rng.integers(0, 1000, size=4 * 96).astype(np.int32)
    cu = np.arange(5, dtype=np.int32) * 96
    pieces = bench.chunk_pieces(ids, cu, 3)
    assert len(pieces) == 3
    back = np.stack([p[0].reshape(4, 32) for p in pieces], axis=1).reshape(-1)
    np.testing.assert_array_equal(back, ids)
    for c, (_, cu_c, off_c) in enumerate(pieces):
        np.testing.assert_array_equal(cu_c, np.arange(5) * 32)
        np.testing.assert_array_equal(off_c, np.full(4, 32 * c))
    with pytest.raises(ValueError):
        bench.chunk_pieces(ids, cu, 5)                       # 5 does not divide 96
    with pytest.raises(ValueError):
        bench.chunk_pieces(ids[:-1], np.array([0, 96, 191], np.int32), 1)  # unequal prompts


def test_chunked_oracle_step_equals_whole_prompts():
    # the chunk op's step under the canvas rule gives each prompt the planes of
    # its whole-prompt canvas (the marker in any chunk, or across a chunk edge)
    import oracle
    wl = inputs.make_frames_workload(num_prompts=6, length=4096, frames=1, seed=11)
    want, want_s, want_a = oracle.positions(wl.ids, wl.cu_seqlens)
    for chunks in (1, 2, 8):
        pieces = bench.chunk_pieces(wl.ids, wl.cu_seqlens, chunks)
        state = (None, None)
        got = []
        for ids_c, cu_c, off_c in pieces:
            pos, st, am = oracle.positions_chunk(ids_c, cu_c, pos_offset=off_c,
                                                 in_start=state[0], in_amount=state[1])
            got.append(pos.reshape(3, 6, -1))
            state = (st, am)
        np.testing.assert_array_equal(np.concatenate(got, axis=2).reshape(3, -1), want)
        np.testing.assert_array_equal(state[0], want_s)
        np.testing.assert_array_equal(state[1], want_a)


@pytest.mark.parametrize("op", ["frames", "chunk"])
def test_planes_reference_arm_prints_one_json_line(op):
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--op", op,
                          "--prompts", "4", "--rule", "qwen_vl", "--steps", "3", "--warmup", "3",
                          "--reference-budget-s", "2"],
                         cwd=ROOT, capture_output=True, text=True, timeout=300, check=True)
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["config"]["op"] == op
    assert d["config"]["global_batch"] == 4 * 65536
    assert d["cpu_baseline"]["kind"] == "oracle"
    if op == "chunk":
        assert "4 chunks per prompt, rule qwen_vl" in d["config"]["workload"]
        assert "rule qwen_vl" in d["cpu_baseline"]["sample"]

"""Benchmark of the canvas M-RoPE hot path on B200.

One step = the whole path over one batch: the planes from the ids, then the
fused cos/sin + rotate of Q and K (every layer), through the one-call entry
point cmr_positions_rotate_qk (the rotation launched to overlap the positions
kernels), on the 6-layer workload: 32 prompts x 8192 tokens with one image
frame each, Q [6, 262144, 8, 256] and K [6, 262144, 2, 256] bf16, rot_dim 64,
theta 1e7, sections [11, 11, 10].  The rotate kernel touches 4.03 GB per step,
far more than the 126 MB L2, so no L2 flush is needed between steps.
--step separate calls cmr_positions and cmr_rotate_qk one after the other
instead, and times the rotate launch on its own.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    torchrun --nproc-per-node N bench.py --gpus N ...   (weak scaling: one batch per GPU)
    python bench.py --probe copy-pattern   (the staged copy-pattern ceiling alone)
    python bench.py --op frames            (multi-frame planes, 256 x 65,536 tokens)
    python bench.py --op chunk [--chunks C] [--rule canvas|qwen_vl|planes_1d]
                                           (chunked prefill planes on the same prompts)

Prints one JSON line on rank 0.  --impl reference times the fp64 CPU oracle on
all host cores (a thread pool over token ranges) on a bounded sample of the
same workload.
"""
import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from vlm_decoder_positional_b200 import cmr, inputs, pipeline, shard  # noqa: E402

METRIC = "canvas M-RoPE tokens/s and achieved HBM GB/s (% of B200 peak), bf16 Q/K, 1 GPU"
UNIT = "tokens/s"
FALLBACK_HBM_GBS = 6650.0
SPEC_HBM_GBS = 8000.0  # B200 HBM3e specification (DGX figure)
PLANES_OPS = ("frames", "chunk")  # planes-only steps on 65,536-token prompts
ROTATE_SOURCES = ["vlm_decoder_positional_b200/csrc/rotate.cu",
                  "vlm_decoder_positional_b200/csrc/rotate_staged.cu",
                  "vlm_decoder_positional_b200/csrc/tma.cuh",
                  "vlm_decoder_positional_b200/csrc/pdl.cuh",
                  "vlm_decoder_positional_b200/csrc/tensor_map.cu",
                  "vlm_decoder_positional_b200/csrc/rotate_common.cuh",
                  "vlm_decoder_positional_b200/csrc/canvas.cuh",
                  "vlm_decoder_positional_b200/csrc/cmr_internal.cuh",
                  "include/cmr.h"]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "rotate_qk_traffic.txt")

# Algorithmic bytes: rotate reads and writes the rot_dim dims of every Q and K
# head of every layer (2,560 B per token-layer here) and reads pos once (12 B
# per token); positions reads 4 B of ids and writes 12 B of planes per token.
def rotate_bytes(n_tokens, layers, hq, hk, rot_dim):
    return n_tokens * layers * (hq + hk) * rot_dim * 2 * 2 + n_tokens * 12


def cache_bytes(n_tokens, layers, hq, hk, rot_dim, head_dim):
    """Rotate + KV-cache write: Q's rotated dims read and written, K and V rows
    read and their cache rows written."""
    return n_tokens * layers * (hq * rot_dim * 2 * 2 + hk * head_dim * 2 * 4)


def positions_bytes(n_tokens, num_seqs):
    return n_tokens * 16 + num_seqs * 12


def workload_label(wl):
    t = wl.num_seqs if wl.cache_len is not None else wl.n_tokens  # Q/K tokens of the workload
    return (f"{wl.name}: {wl.num_seqs} prompts x {wl.n_tokens // max(wl.num_seqs, 1)} tokens, "
            f"{wl.num_layers} layers, Q [{wl.num_layers},{t},{wl.hq},{wl.head_dim}] "
            f"K [{wl.num_layers},{t},{wl.hk},{wl.head_dim}] bf16, rot_dim "
            f"{wl.rot_dim}, theta {wl.theta:g}, sections {list(wl.sections)}")


def config_dict(args, wl, tokens_all, world, rot_b):
    """The workload's config, the same for both arms of the benchmark."""
    return {"workload": workload_label(wl), "global_batch": tokens_all,
            "launch": args.launch, "op": args.op, "step": step_kind(args, wl),
            "seq_len": wl.n_tokens // max(wl.num_seqs, 1),
            "parallelism": f"dp{world} ({'independent batches' if args.scaling == 'weak' else 'whole prompts split over ranks'}, no data-path collective)",
            "l2": "inputs larger than L2 (rotate touches %.2f GB per step, L2 126 MB);"
                  " no flush" % (rot_b / 1e9)}


def step_kind(args, wl):
    """'one-call' when a prefill step runs the positions + rotate entry point."""
    if args.op == "rotate" and wl.cache_len is None and args.step == "fused":
        return "one-call"
    return "separate"


def measured_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


_C_TOKENS = re.compile(r'//[^\n]*|/\*.*?\*/|"(?:\\.|[^"\\\n])*"|\'(?:\\.|[^\'\\\n])*\'|\s+|[^\s"\'/]+|/',
                       re.S)


def code_tokens(text):
    """The source with comments dropped and every run of whitespace folded to one
    space (string and character literals kept as written), so that a comment
    edit does not count as a change of the kernel."""
    out = []
    for m in _C_TOKENS.finditer(text):
        tok = m.group(0)
        if tok.startswith("//") or tok.startswith("/*") or tok.isspace():
            if out and out[-1] != " ":
                out.append(" ")
        else:
            out.append(tok)
    return "".join(out).strip()


def rotate_source_hash(read=None):
    """SHA-256 of the code (comments and layout aside) of every source the
    rotate kernel compiles; `read(rel)` returns a file's text (default: this
    checkout)."""
    if read is None:
        def read(rel):
            with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
                return f.read()
    h = hashlib.sha256()
    for rel in ROTATE_SOURCES:
        h.update(rel.encode() + b"\0" + code_tokens(read(rel)).encode() + b"\0")
    return h.hexdigest()


def recorded_traffic(workload_name, kernel=None):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    this exact kernel source, workload and kernel; otherwise None."""
    try:
        rec = {}
        with open(TRAFFIC_FILE) as f:
            for line in f:
                if ":" in line and not line.startswith("#"):
                    k, v = line.split(":", 1)
                    rec[k.strip()] = v.strip()
        if rec.get("kernel_source_sha256") != rotate_source_hash():
            return None
        if rec.get("workload") != workload_name:
            return None
        if kernel is not None and rec.get("kernel") != kernel:
            return None
        return int(rec["dram_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        return None


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML (read-only) while running."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
        "display_clock_setting": 0x100,
    }

    def __init__(self, device_index, interval=0.005):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.interval = interval
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nvml = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # noqa: BLE001
            self._nvml = None
            self.error = str(e)

    def _sample(self):
        n = self._nvml
        self.samples.append(n.nvmlDeviceGetClockInfo(self._h, n.NVML_CLOCK_SM))
        mask = n.nvmlDeviceGetCurrentClocksEventReasons(self._h)
        for name, bit in self.REASONS.items():
            if mask & bit:
                self.reasons.add(name)

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.interval)

    def __enter__(self):
        if self._nvml:
            self._sample()
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        if self._thread:
            self._stop.set()
            self._thread.join()
            self._sample()

    def summary(self):
        if not self._nvml:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": self.error}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples),
                "source": "nvml"}


# ---------------------------------------------------------------------------
# CPU side: the oracle on a bounded sample (baseline and reference arm)
# ---------------------------------------------------------------------------

def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def host_cpu():
    """The host's CPU model (first /proc/cpuinfo entry) and logical core count."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"cpu_model": model, "nproc": os.cpu_count(), "threads_allowed": host_cores()}


def oracle_sample_step(wl_cpu, n, threads=1):
    """One oracle pass over a sample: the planes of the prompts that hold the
    first n tokens (decode: of the first n prompts, then their new token),
    then the rotation of those n tokens' Q/K rows, every layer and head.  With
    threads > 1 the rotation's token range is split over a thread pool (the
    oracle is C called through ctypes, which releases the GIL)."""
    import oracle
    cu = wl_cpu["cu"]
    if wl_cpu["cache_len"] is None:
        b = int(np.searchsorted(cu, n, side="left"))
        pos, _, _ = oracle.positions(wl_cpu["ids"][: cu[b]], cu[: b + 1], inputs.IMAGE_TOKEN_ID)
        pos = np.ascontiguousarray(pos[:, :n])
    else:
        _, start, amount = oracle.positions(wl_cpu["ids"][: cu[n]], cu[: n + 1],
                                            inputs.IMAGE_TOKEN_ID)
        pos = oracle.positions_step(wl_cpu["cache_len"][:n], start, amount)

    def rotate(lo, hi):
        p = np.ascontiguousarray(pos[:, lo:hi])
        oracle.rotate_bf16(wl_cpu["q"][:, lo:hi], p)
        oracle.rotate_bf16(wl_cpu["k"][:, lo:hi], p)

    if threads <= 1:
        rotate(0, n)
    else:
        from concurrent.futures import ThreadPoolExecutor
        cuts = np.linspace(0, n, threads + 1).astype(int)
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(lambda i: rotate(cuts[i], cuts[i + 1]), range(threads)))
    return n


def cpu_sample_inputs(wl, n_max):
    def bits(t):
        return t[:, :n_max].detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    return {"ids": wl.ids, "cu": wl.cu_seqlens, "q": bits(wl.q), "k": bits(wl.k),
            "cache_len": wl.cache_len}


def calibrate_sample(wl_cpu, seconds, n_max, threads=1):
    """Tokens whose oracle pass takes about `seconds` on this host (at most n_max),
    estimated from a probe on the tokens wl_cpu holds."""
    probe = min(256 * threads, n_max, wl_cpu["q"].shape[1])
    t0 = time.perf_counter()
    oracle_sample_step(wl_cpu, probe, threads)
    dt = time.perf_counter() - t0
    return int(max(probe, min(n_max, probe * seconds / max(dt, 1e-6))))


def sample_label(wl, n, threads=1):
    tail = f"fp64, {threads} thread{'s' if threads > 1 else ''}"
    if wl.cache_len is not None:
        return (f"planes of the first {n} prompts + their new token, rotation of those {n} "
                f"tokens x {wl.num_layers} layers x {wl.hq + wl.hk} heads, {tail}")
    b = int(np.searchsorted(wl.cu_seqlens, n, side="left"))
    return (f"planes of the first {b} prompts ({wl.cu_seqlens[b]} tokens) + rotation of the "
            f"first {n} tokens x {wl.num_layers} layers x {wl.hq + wl.hk} heads, {tail}")


def run_cpu_baseline(wl, seconds):
    """The oracle on all host cores (and on one, for reference) over a bounded
    sample of the workload, about `seconds` of work each."""
    cores = host_cores()
    n_cap = min(wl.qk_tokens, 200_000)
    probe_inputs = cpu_sample_inputs(wl, min(n_cap, 256 * cores))
    out = {}
    for threads in sorted({1, cores}, reverse=True):
        n = calibrate_sample(probe_inputs, seconds, n_cap, threads)
        wl_cpu = cpu_sample_inputs(wl, n) if n > probe_inputs["q"].shape[1] else probe_inputs
        t0 = time.perf_counter()
        oracle_sample_step(wl_cpu, n, threads)
        dt = time.perf_counter() - t0
        out[threads] = (n / dt, sample_label(wl, n, threads) + f", {dt:.1f} s")
        del wl_cpu
    value, sample = out[cores]
    res = {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample,
           "host": host_cpu()}
    if cores > 1:
        res["single_thread"] = {"value": out[1][0], "sample": out[1][1]}
    return res


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    # the same prompts (ids); Q/K drawn only for the sampled tokens
    wl = inputs.make_config(args.workload, device="cpu", with_qk=False)
    if args.layers is not None:
        wl.num_layers = args.layers
    full_tokens = wl.num_seqs if wl.cache_len is not None else wl.n_tokens
    cores = host_cores()
    per_step = max(1.0, args.reference_budget_s / (args.steps + args.warmup))
    n_max = min(wl.num_seqs if wl.cache_len is not None else wl.n_tokens, 200_000)
    wl.q = inputs.random_qk((wl.num_layers, n_max, wl.hq, wl.head_dim), wl.seed + 1)
    wl.k = inputs.random_qk((wl.num_layers, n_max, wl.hk, wl.head_dim), wl.seed + 2)
    wl_cpu = cpu_sample_inputs(wl, n_max)
    n = calibrate_sample(wl_cpu, per_step, n_max, cores)
    for _ in range(args.warmup):
        oracle_sample_step(wl_cpu, n, cores)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_sample_step(wl_cpu, n, cores)
    dt = time.perf_counter() - t0
    value = n * args.steps / dt
    sample = "per step: " + sample_label(wl, n, cores)
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
        "config": config_dict(args, wl, full_tokens * args.gpus if args.scaling == "weak"
                              else full_tokens, args.gpus,
                              rotate_bytes(full_tokens, wl.num_layers, wl.hq, wl.hk,
                                           wl.rot_dim) if args.op != "cache" else
                              cache_bytes(full_tokens, wl.num_layers, wl.hq, wl.hk, wl.rot_dim,
                                          wl.head_dim)),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample + f", the fp64 oracle on {cores} host threads",
                         "host": host_cpu()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }), flush=True)
    return 0


# ---------------------------------------------------------------------------
# GPU side
# ---------------------------------------------------------------------------

def run_ours(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    cmr.lib()

    if args.scaling == "weak":
        # every rank rotates a full batch of its own (a different seed per rank)
        seed = shard.rank_seed(inputs.BASE_SEED + args.workload, rank)
        wl = inputs.make_config(args.workload, device=dev, seed=seed,
                                with_qk=args.layers is None)
        if args.layers is not None:
            # the workload's prompts with another number of attention layers
            wl.num_layers = args.layers
            rows = wl.n_tokens if wl.cache_len is None else wl.num_seqs
            wl.q = inputs.random_qk((args.layers, rows, wl.hq, wl.head_dim), seed + 1, dev)
            wl.k = inputs.random_qk((args.layers, rows, wl.hk, wl.head_dim), seed + 2, dev)
    else:
        # one batch split by whole prompts; each rank draws only its own Q/K rows
        wl = inputs.make_config(args.workload, device=dev, with_qk=False)
        if args.layers is not None:
            wl.num_layers = args.layers
        if wl.cache_len is not None:
            raise SystemExit("--scaling strong covers prefill workloads only")
        global_tokens = wl.n_tokens
        sh = shard.shard_sequences(wl.cu_seqlens, world, rank)
        wl.ids, wl.cu_seqlens = shard.local_batch(wl.ids, wl.cu_seqlens, sh)
        wl.frame_origin = wl.frame_origin[sh.seq_lo:sh.seq_hi]
        seed = shard.rank_seed(wl.seed, rank)
        wl.q = inputs.random_qk((wl.num_layers, sh.n_tokens, wl.hq, wl.head_dim), seed + 1, dev)
        wl.k = inputs.random_qk((wl.num_layers, sh.n_tokens, wl.hk, wl.head_dim), seed + 2, dev)
    ids = torch.from_numpy(wl.ids).to(dev)
    cu = torch.from_numpy(wl.cu_seqlens).to(dev)
    n, b, L = wl.n_tokens, wl.num_seqs, wl.num_layers
    pos = torch.empty((3, n), dtype=torch.int32, device=dev)
    start = torch.empty(b, dtype=torch.int32, device=dev)
    amount = torch.empty(b, dtype=torch.int32, device=dev)
    decode = wl.cache_len is not None
    cache_len = torch.from_numpy(wl.cache_len).to(dev) if decode else None
    stream = torch.cuda.current_stream(dev)
    tokens_per_step = wl.qk_tokens
    rot_b = rotate_bytes(wl.qk_tokens, L, wl.hq, wl.hk, wl.rot_dim)
    # the kernel the library picks for this shape (staged or register-resident)
    kernel = cmr.rotate_qk_kernel(wl.qk_tokens, L, wl.hq, wl.hk, wl.head_dim, wl.rot_dim)
    rope = dict(theta=wl.theta, sections=wl.sections, rot_dim=wl.rot_dim)

    if args.op == "cache":
        # rotate Q and write rotated K and V rows into [L, B, hk, ctx, D] caches
        v = inputs.random_qk(tuple(wl.k.shape), wl.seed + 3, dev)
        ctx = int(wl.cache_len.max()) + 1 if decode else int(np.diff(wl.cu_seqlens).max())
        k_cache = torch.zeros((L, b, wl.hk, ctx, wl.head_dim), dtype=torch.bfloat16, device=dev)
        v_cache = torch.zeros_like(k_cache)
        rot_b = cache_bytes(wl.qk_tokens, L, wl.hq, wl.hk, wl.rot_dim, wl.head_dim)
        kernel = cmr.rotate_qk_cache_kernel(wl.qk_tokens, L, wl.hq, wl.hk, wl.head_dim,
                                            wl.rot_dim)
    if decode:
        # The prompts' (start, amount) come from their prefill, once; a decode
        # step is one launch that derives each new token's planes in the
        # kernel from (cache_len, start, amount) and rotates it.
        cmr.positions(ids, cu, wl.image_token_id, out=(pos, start, amount))
        if args.op == "cache":
            plan = [("rotate", lambda: cmr.rotate_qk_cache(
                wl.q, wl.k, v, start, amount, k_cache, v_cache, pos_offset=cache_len, **rope))]
        else:
            plan = [("rotate", lambda: cmr.rotate_qk_shift(wl.q, wl.k, start, amount,
                                                           pos_offset=cache_len, **rope))]
    elif step_kind(args, wl) == "one-call":
        plan = [("rotate", lambda: cmr.positions_rotate_qk(
            ids, cu, wl.q, wl.k, wl.theta, wl.sections, wl.rot_dim, wl.image_token_id,
            out=(pos, start, amount)))]
    else:
        plan = [("positions", lambda: cmr.positions(ids, cu, wl.image_token_id,
                                                    out=(pos, start, amount)))]
        if args.op == "rotate":
            plan.append(("rotate", lambda: cmr.rotate_qk(wl.q, wl.k, pos, wl.theta, wl.sections,
                                                         wl.rot_dim)))
        elif args.op == "shift":
            plan.append(("rotate", lambda: cmr.rotate_qk_shift(wl.q, wl.k, start, amount,
                                                               cu_seqlens=cu, **rope)))
        else:
            plan.append(("rotate", lambda: cmr.rotate_qk_cache(
                wl.q, wl.k, v, start, amount, k_cache, v_cache, cu_seqlens=cu, **rope)))
    calls = dict(plan)
    if args.launch == "graph":
        # one CUDA graph per call: a rotate form's single kernel, or the
        # positions form's memset and two kernels (the one-call step also holds
        # the rotation, behind a programmatic edge)
        for fn in calls.values():
            fn()
        torch.cuda.synchronize(dev)
        graphs = {}
        for name, fn in plan:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                fn()
            graphs[name] = g
        calls = {name: g.replay for name, g in graphs.items()}

    def step(ev=None):
        if ev is not None:
            ev[2].record(stream)
        if "positions" in calls:
            calls["positions"]()
        if ev is not None:
            ev[0].record(stream)
        calls["rotate"]()
        if ev is not None:
            ev[1].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    # the rotate kernel the library actually launched (recorded at the launch
    # or at its capture into the graph)
    kernel_ran = cmr.last_rotate_kernel() or kernel

    # A step of one call is timed by the two events around the K steps alone
    # (events recorded between graph launches cost about a microsecond each);
    # a step of two calls also gets events around each call.
    single = "positions" not in calls
    rot_events = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3))
                  for _ in range(args.steps)]
    t_begin = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local_rank) as clocks:
        t_begin.record(stream)
        for i in range(args.steps):
            step(None if single else rot_events[i])
        t_end.record(stream)
        torch.cuda.synchronize(dev)
    if dist:
        dist.barrier()
    ms = t_begin.elapsed_time(t_end)
    if single:
        rot_ms = [ms / args.steps]
        pos_ms = [0.0]
    else:
        rot_ms = [a.elapsed_time(z) for a, z, _ in rot_events]
        pos_ms = [p.elapsed_time(a) for a, _, p in rot_events]
    ms_max = shard.max_over_ranks(ms, dist, dev)
    # tokens processed by all ranks in one step
    tokens_all = tokens_per_step * world if args.scaling == "weak" else global_tokens
    # kernels per step: the positions form launches two (origin scan, planes),
    # each rotate form one, the one-call path two (origin scan, rotation)
    per_step = {"positions": 2, "rotate": 1}
    launches = args.steps * sum(per_step[name] for name, _ in plan)
    if step_kind(args, wl) == "one-call":
        launches = args.steps * 2

    # end to end through the public API from pinned host memory
    if args.op == "rotate":
        if wl.cache_len is not None:
            e2e = run_e2e(args, wl, dev, stream, dist, tokens_all)
        else:
            # both prefill paths of the public API, the faster one as the record
            runs = [run_e2e(args, wl, dev, stream, dist, tokens_all, path)
                    for path in ("native", "pipeline")]
            runs.sort(key=lambda r: -r["value"])
            e2e = dict(runs[0])
            e2e["other_path"] = {k: runs[1][k] for k in ("value", "ms_per_step", "path")}
    else:
        e2e = {"skipped": f"--op {args.op} times the device step only; the end-to-end path "
                          "is measured with --op rotate"}

    # the two ceilings of an HBM-bound launch (the staged kernel's batches are
    # larger than L2; the small workloads are bound by launch latency)
    ceiling = same_size_copy = None
    if args.op == "rotate" and kernel_ran == "rotate_qk_staged_kernel":
        ceiling = run_copy_pattern_probe(wl, dev, stream)
        same_size_copy = run_plain_copy_probe(rot_b, dev, stream)

    if rank == 0:
        peak, peak_src = measured_peak()
        rot_avg_s = statistics.mean(rot_ms) / 1e3
        achieved = rot_b / rot_avg_s / 1e9
        traffic = recorded_traffic(wl.name, kernel_ran) if args.op == "rotate" else None
        value = tokens_all * args.steps / (ms_max / 1e3)
        one_call = step_kind(args, wl) == "one-call"
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            cpu = run_cpu_baseline(wl, args.cpu_seconds)
        roofline = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                    "frac": achieved / peak, "traffic": traffic,
                    "kernel": kernel_ran,
                    "algorithmic_bytes_per_launch": rot_b,
                    "avg_launch_ms": rot_avg_s * 1e3,
                    "timed": ("the one-call step (CUDA events around the K steps, divided by "
                              "K): the origin scan and the rotation overlapping it, an upper "
                              "bound of the rotate kernel's own duration" if one_call else
                              "the rotate call alone (events around it)" if not single else
                              "the rotate call (CUDA events around the K steps, divided by K)"),
                    "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)"
                    if peak_src == "measured" else "fallback 6650 GB/s",
                    "spec_peak": SPEC_HBM_GBS, "frac_of_spec": achieved / SPEC_HBM_GBS}
        if ceiling is not None:
            roofline["ceiling"] = ceiling["gbs"]
            roofline["frac_of_ceiling"] = achieved / ceiling["gbs"]
            roofline["ceiling_source"] = ceiling["what"]
        if same_size_copy is not None:
            roofline["same_size_copy"] = same_size_copy["gbs"]
            roofline["frac_of_same_size_copy"] = achieved / same_size_copy["gbs"]
            roofline["same_size_copy_source"] = same_size_copy["what"]
        out = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max / args.steps,
            "higher_is_better": True, "scaling": args.scaling, "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) bf16 Q/K, uniform text ids, one 448x448 frame "
                    "per prompt)",
            "config": config_dict(args, wl, tokens_all, world, rot_b),
            "hbm_gbs": achieved, "pct_of_peak": 100.0 * achieved / peak,
            "pct_of_spec_peak": 100.0 * achieved / SPEC_HBM_GBS,
            "token_layers_per_s": value * L,
            "roofline": roofline,
            "positions_bytes_per_step": positions_bytes(n, b),
            "positions_avg_ms": None if one_call else statistics.mean(pos_ms),
            "e2e": e2e, "gpu_launches": launches, "clocks": clocks.summary(),
            "cpu_baseline": cpu, "impl": "ours",
        }
        print(json.dumps(out), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def probe_lib():
    import ctypes
    from vlm_decoder_positional_b200 import build as libbuild
    libbuild.build()
    lib = ctypes.CDLL(libbuild.PROBE_LIB)
    f = lib.cmr_probe_copy_pattern_tiles
    f.restype = ctypes.c_int
    f.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32,
                  ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                  ctypes.c_void_p, ctypes.c_void_p]
    return f


def run_copy_pattern_probe(wl, dev, stream, launches=10, warmup=3, tiles_per_cta=1):
    """The ceiling of the staged rotation's access pattern: copy_pattern_kernel
    moves the same rotated dims of Q and K through the same TMA staging with no
    math (an identity copy), timed like the rotate launch (CUDA events around
    each of `launches` launches).  tiles_per_cta > 1: each CTA walks that many
    consecutive tiles through one ring.  Returns GB/s over the Q/K bytes it
    moves."""
    f = probe_lib()
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    n = wl.q.shape[1]
    args = (wl.q.data_ptr(), wl.k.data_ptr(), n, wl.num_layers, wl.hq, wl.hk, wl.head_dim,
            int(tiles_per_cta), status.data_ptr(), stream.cuda_stream)
    for _ in range(warmup):
        if f(*args) != 0:
            raise RuntimeError("copy-pattern probe: launch refused")
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(launches)]
    torch.cuda.synchronize(dev)
    for a, z in ev:
        a.record(stream)
        f(*args)
        z.record(stream)
    torch.cuda.synchronize(dev)
    if int(status.item()) != 0:
        raise RuntimeError("copy-pattern probe: a bounded wait gave up")
    ms = statistics.mean(a.elapsed_time(z) for a, z in ev)
    moved = n * wl.num_layers * (wl.hq + wl.hk) * 64 * 2 * 2
    return {"gbs": moved / (ms / 1e3) / 1e9, "ms": ms, "bytes": moved,
            "what": "copy_pattern_kernel (libcmr_probe.so): the staged rotation's TMA boxes "
                    "loaded and stored back unchanged, no math; mean of %d launches" % launches}


def run_plain_copy_probe(moved, dev, stream, launches=10, warmup=3):
    """A plain device-to-device copy (torch copy_, read + write bytes) of the
    same total bytes as the rotation moves, timed the same way: the copy peak
    at this launch size, which includes the start and drain one launch of
    this size cannot hide."""
    half = (moved // 2 + 15) // 16 * 16
    src = torch.empty(half, dtype=torch.uint8, device=dev)
    dst = torch.empty(half, dtype=torch.uint8, device=dev)
    src.fill_(1)
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            dst.copy_(src)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(launches)]
        torch.cuda.synchronize(dev)
        for a, z in ev:
            a.record(stream)
            dst.copy_(src)
            z.record(stream)
    torch.cuda.synchronize(dev)
    ms = statistics.mean(a.elapsed_time(z) for a, z in ev)
    del src, dst
    return {"gbs": 2 * half / (ms / 1e3) / 1e9, "ms": ms, "bytes": 2 * half,
            "what": "torch copy_ of the same read + write bytes as one launch moves (two "
                    "contiguous buffers); mean of %d copies" % launches}


def run_plain_fill_probe(nbytes, dev, stream, launches=10, warmup=3):
    """A store-only stream (torch fill_) of ``nbytes``, timed the same way as
    the copy probe: the ceiling of a launch that only writes, as the planes
    kernels mostly do."""
    buf = torch.empty((nbytes + 15) // 16 * 4, dtype=torch.int32, device=dev)
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            buf.fill_(7)
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(launches)]
        torch.cuda.synchronize(dev)
        for a, z in ev:
            a.record(stream)
            buf.fill_(7)
            z.record(stream)
    torch.cuda.synchronize(dev)
    ms = statistics.mean(a.elapsed_time(z) for a, z in ev)
    size = buf.numel() * 4
    del buf
    return {"gbs": size / (ms / 1e3) / 1e9, "ms": ms, "bytes": size,
            "what": "torch fill_ of a buffer the size of the planes (stores only); mean of "
                    "%d fills" % launches}


def run_probe_only(args):
    """--probe copy-pattern: the ceiling probe alone on the workload's Q/K."""
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", "0")))
    torch.cuda.set_device(dev)
    wl = inputs.make_config(args.workload, device=dev)
    stream = torch.cuda.current_stream(dev)
    if args.layers is not None:
        wl.num_layers = args.layers
        wl.q = inputs.random_qk((args.layers, wl.n_tokens, wl.hq, wl.head_dim), 11, dev)
        wl.k = inputs.random_qk((args.layers, wl.n_tokens, wl.hk, wl.head_dim), 12, dev)
    res = run_copy_pattern_probe(wl, dev, stream, launches=args.steps, warmup=args.warmup,
                                 tiles_per_cta=args.tiles_per_cta)
    plain = run_plain_copy_probe(res["bytes"], dev, stream, launches=args.steps,
                                 warmup=args.warmup)
    peak, src = measured_peak()
    print(json.dumps({"probe": "copy-pattern", "workload": workload_label(wl),
                      "tiles_per_cta": args.tiles_per_cta, "layers": wl.num_layers,
                      "gbs": res["gbs"], "ms_per_launch": res["ms"], "bytes": res["bytes"],
                      "peak": peak, "peak_source": src, "frac_of_peak": res["gbs"] / peak,
                      "launches": args.steps, "what": res["what"],
                      "same_size_copy_gbs": plain["gbs"],
                      "same_size_copy_frac_of_peak": plain["gbs"] / peak,
                      "same_size_copy_what": plain["what"]}), flush=True)
    return 0


def chunk_bytes(n_tokens, num_seqs, chunks, id_reads):
    """Chunked prefill planes, one cmr_positions_chunk call per chunk: 12 B of
    planes per token; the ids the rule has to read (``id_reads`` in all, see
    first_marker_reads), 4 B each; per prompt and call cu_seqlens and the
    outgoing state (12 B), and from the second chunk on the offset and the
    incoming state (12 B more).  The planes themselves follow from each
    token's absolute index and the state, so no other id is needed."""
    return n_tokens * 12 + id_reads * 4 + num_seqs * (12 * chunks + 12 * (chunks - 1))


def first_marker_reads(ids, cu_seqlens, marker, rule):
    """Ids a rule must read to fix every prompt's state: up to and including
    the prompt's first marker, or all of it when it holds none (canvas and
    Qwen-VL rules); none under planes_1d, which never shifts."""
    if rule == "planes_1d":
        return 0
    total = 0
    for b in range(cu_seqlens.shape[0] - 1):
        seg = ids[cu_seqlens[b]:cu_seqlens[b + 1]]
        hit = np.flatnonzero(seg == marker)
        total += int(hit[0]) + 1 if hit.size else int(seg.shape[0])
    return total


def planes_workload(args, seed=None):
    """The planes-only workloads: --op frames, prompts of 65,536 tokens with
    --frames-per-prompt frames on a --grid-side grid; --op chunk, the same
    prompts with one thumbnail each (grid side 8) at a random origin."""
    if args.op == "frames":
        return inputs.make_frames_workload(num_prompts=args.prompts,
                                           frames=args.frames_per_prompt,
                                           grid_side=args.grid_side, seed=seed)
    return inputs.make_frames_workload(num_prompts=args.prompts, frames=1, grid_side=8,
                                       seed=seed)


def chunk_pieces(ids, cu_seqlens, chunks):
    """Cuts every prompt of an equal-length batch into ``chunks`` equal pieces:
    piece c of all prompts is one cmr_positions_chunk call.  Returns a list of
    (ids, cu_seqlens, pos_offset) numpy arrays, one per call."""
    b = cu_seqlens.shape[0] - 1
    length = int(cu_seqlens[1] - cu_seqlens[0]) if b else 0
    if b == 0 or not np.array_equal(cu_seqlens, np.arange(b + 1, dtype=np.int64) * length):
        raise ValueError("chunked prefill needs prompts of one length")
    if chunks < 1 or length % chunks:
        raise ValueError(f"{chunks} chunks do not divide prompts of {length} tokens")
    lc = length // chunks
    blocks = np.asarray(ids, np.int32).reshape(b, chunks, lc)
    cu = (np.arange(b + 1) * lc).astype(np.int32)
    return [(np.ascontiguousarray(blocks[:, c, :]).reshape(-1), cu,
             np.full(b, c * lc, np.int32)) for c in range(chunks)]


def oracle_planes_work(args, wl):
    """The oracle's planes of the first ``take`` prompts of a planes workload:
    run(take) -> tokens covered (the frames reading, or the chunked prefill
    carrying each prompt's state from chunk to chunk)."""
    import oracle
    cu = wl.cu_seqlens
    if args.op == "frames":
        def run(lo, hi):
            oracle.positions_frames(wl.ids[cu[lo]:cu[hi]], cu[lo:hi + 1] - cu[lo],
                                    wl.image_token_id, args.grid_side)
            return int(cu[hi] - cu[lo])
        return run

    def run(lo, hi):
        pieces = chunk_pieces(wl.ids[cu[lo]:cu[hi]], cu[lo:hi + 1] - cu[lo], args.chunks)
        state = (None, None)
        for ids_c, cu_c, off_c in pieces:
            _, st, am = oracle.positions_chunk(ids_c, cu_c, wl.image_token_id, args.rule,
                                               off_c, *state)
            state = (st, am)
        return int(cu[hi] - cu[lo])
    return run


def planes_config(args, wl, world):
    n, b = wl.n_tokens, wl.num_seqs
    if args.op == "frames":
        what = (f"{wl.name}: {b} prompts x {n // b} tokens, "
                f"{args.frames_per_prompt} frames each, grid side {args.grid_side}")
        moved = positions_bytes(n, b)
    else:
        what = (f"chunked_prefill_{b}x{n // b}: {b} prompts x {n // b} tokens, one 448x448 "
                f"thumbnail each, {args.chunks} chunks per prompt, rule {args.rule}")
        moved = chunk_bytes(n, b, args.chunks, first_marker_reads(
            wl.ids, wl.cu_seqlens, wl.image_token_id, args.rule))
    return {"workload": what, "global_batch": n * world, "launch": args.launch, "op": args.op,
            "step": "separate" if args.op == "frames" else
                    f"{args.chunks} chunk call{'s' if args.chunks != 1 else ''}",
            "seq_len": n // b,
            "parallelism": f"dp{world} (independent batches, no data-path collective)",
            "l2": "inputs larger than L2 (%.0f MB of ids and planes per step, L2 126 MB); no "
                  "flush" % (moved / 1e6) if moved > 126e6 else
                  "ids and planes (%.0f MB) fit in L2; no flush" % (moved / 1e6)}


def run_planes_reference(args):
    """--impl reference --op frames|chunk: the oracle's planes on all host
    cores (whole prompts split over a thread pool), on a bounded sample of the
    workload per step."""
    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    from concurrent.futures import ThreadPoolExecutor
    wl = planes_workload(args)
    work = oracle_planes_work(args, wl)
    cores = host_cores()
    cu = wl.cu_seqlens

    def run(take):
        cuts = np.linspace(0, take, cores + 1).astype(int)

        def part(i):
            if cuts[i + 1] > cuts[i]:
                work(cuts[i], cuts[i + 1])
        with ThreadPoolExecutor(cores) as ex:
            list(ex.map(part, range(cores)))

    per_step = max(0.5, args.reference_budget_s / (args.steps + args.warmup))
    take = 1
    while take < wl.num_seqs:
        t0 = time.perf_counter()
        run(take)
        if time.perf_counter() - t0 > per_step / 2:
            break
        take = min(wl.num_seqs, take * 2)
    for _ in range(args.warmup):
        run(take)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run(take)
    dt = time.perf_counter() - t0
    n = int(cu[take])
    value = n * args.steps / dt
    what = ("multi-frame planes" if args.op == "frames" else
            f"planes in {args.chunks} chunks per prompt (rule {args.rule})")
    sample = (f"per step: {what} of the first {take} prompts ({n} tokens), "
              f"the oracle (integer arithmetic) on {cores} host threads")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int32", "data": "synthetic (seeded)",
        "config": planes_config(args, wl, args.gpus),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample, "host": host_cpu()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }), flush=True)
    return 0


def run_planes(args):
    """--op frames: one step = cmr_positions_frames (multi-frame canvas planes)
    on 65,536-token prompts with --frames-per-prompt frames on a --grid-side
    grid.  --op chunk: one step = the chunked prefill of every prompt, --chunks
    cmr_positions_chunk calls (chunk c of all prompts per call, each carrying
    the state of the call before it) under --rule.  Graph-replayed, CUDA events
    around the K steps."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    cmr.lib()
    seed = shard.rank_seed(inputs.BASE_SEED + 6, rank)
    wl = planes_workload(args, seed=seed)
    n, b = wl.n_tokens, wl.num_seqs
    stream = torch.cuda.current_stream(dev)
    if args.op == "frames":
        ids = torch.from_numpy(wl.ids).to(dev)
        cu = torch.from_numpy(wl.cu_seqlens).to(dev)
        pos = torch.empty((3, n), dtype=torch.int32, device=dev)
        start = torch.empty(b, dtype=torch.int32, device=dev)
        amount = torch.empty(b, dtype=torch.int32, device=dev)
        ws = torch.empty(cmr.positions_frames_workspace_bytes(b, n), dtype=torch.uint8,
                         device=dev)

        def call():
            cmr.positions_frames(ids, cu, args.grid_side, out=(pos, start, amount),
                                 workspace=ws)
        moved, launches = positions_bytes(n, b), 2
        kernel = "frames_positions_kernel (+ frames_summary_kernel)"
        timed = "the summary and planes kernels"
    else:
        pieces = [tuple(torch.from_numpy(a).to(dev) for a in p)
                  for p in chunk_pieces(wl.ids, wl.cu_seqlens, args.chunks)]
        outs = [torch.empty((3, p[0].numel()), dtype=torch.int32, device=dev) for p in pieces]
        states = [(torch.empty(b, dtype=torch.int32, device=dev),
                   torch.empty(b, dtype=torch.int32, device=dev)) for _ in range(2)]

        def call():
            for c, (ids_c, cu_c, off_c) in enumerate(pieces):
                cmr.positions_chunk(ids_c, cu_c, pos_offset=off_c if c else None,
                                    state=states[(c + 1) % 2] if c else None, rule=args.rule,
                                    out=(outs[c], *states[c % 2]))
        moved = chunk_bytes(n, b, args.chunks, first_marker_reads(
            wl.ids, wl.cu_seqlens, wl.image_token_id, args.rule))
        launches = 2 * args.chunks
        kernel = "canvas_positions_kernel (+ canvas_origin_kernel), per chunk"
        timed = f"the {args.chunks} chunk calls (origin scan and planes kernels each)"

    call()
    torch.cuda.synchronize(dev)
    if args.launch == "graph":
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            call()
        call = g.replay
    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize(dev)
    t_begin = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local_rank) as clocks:
        t_begin.record(stream)
        for _ in range(args.steps):
            call()
        t_end.record(stream)
        torch.cuda.synchronize(dev)
    if dist:
        dist.barrier()
    ms_local = t_begin.elapsed_time(t_end)
    ms_max = shard.max_over_ranks(ms_local, dist, dev)
    step_ms = ms_local / args.steps
    if rank == 0:
        peak, peak_src = measured_peak()
        achieved = moved / (step_ms / 1e3) / 1e9
        # the planes' stores against a store-only stream of the same size
        fill = run_plain_fill_probe(12 * n, dev, stream)
        planes_gbs = 12 * n / (step_ms / 1e3) / 1e9
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            work = oracle_planes_work(args, wl)
            take = 1
            t0 = time.perf_counter()
            while True:  # whole prompts, about --cpu-seconds of oracle work
                tokens = work(0, take)
                dt = time.perf_counter() - t0
                if dt > args.cpu_seconds or take == b:
                    break
                take = min(b, take * 2)
                t0 = time.perf_counter()
            what = ("multi-frame planes" if args.op == "frames" else
                    f"planes in {args.chunks} chunks per prompt (rule {args.rule})")
            cpu = {"value": tokens / dt, "unit": UNIT, "cores": 1, "kind": "oracle",
                   "host": host_cpu(),
                   "sample": f"{what} of the first {take} prompts ({tokens} tokens), "
                             f"1 thread, {dt:.2f} s"}
        tokens_all = n * world
        out = {
            "metric": METRIC, "value": tokens_all * args.steps / (ms_max / 1e3), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms_max / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int32",
            "data": "synthetic (seeded uniform text ids, frames on a grid_side x grid_side grid)",
            "config": planes_config(args, wl, world),
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": None, "kernel": kernel,
                         "algorithmic_bytes_per_launch": moved, "avg_launch_ms": step_ms,
                         "timed": f"the step (CUDA events around the K steps, divided by K): "
                                  f"{timed}",
                         "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)"
                         if peak_src == "measured" else "fallback 6650 GB/s",
                         "spec_peak": SPEC_HBM_GBS, "frac_of_spec": achieved / SPEC_HBM_GBS,
                         "planes_store_gbs": planes_gbs, "same_size_fill_gbs": fill["gbs"],
                         "planes_frac_of_fill": planes_gbs / fill["gbs"],
                         "same_size_fill_what": fill["what"]},
            "e2e": {"skipped": f"--op {args.op} times the device step only"},
            "gpu_launches": launches * args.steps, "clocks": clocks.summary(),
            "cpu_baseline": cpu, "impl": "ours",
        }
        print(json.dumps(out), flush=True)
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_e2e(args, wl, dev, stream, dist, tokens_all, path="pipeline"):
    """Same metric through the public API, the batch in pinned host memory:
    every step moves the inputs from the host, runs positions + rotate, and
    moves the results back.  Prefill paths: "native" is one
    cmr_positions_rotate_qk_host call (the kernels read and write the host
    buffers over PCIe); "pipeline" is pipeline.HostPipeline (copies of whole-
    prompt chunks overlapped with the kernels on three streams)."""
    decode = wl.cache_len is not None
    # a decode step moves a few MB: time as many steps as the device loop
    steps = args.steps if decode else max(2, min(args.steps, args.e2e_steps))
    h_ids = torch.from_numpy(wl.ids).pin_memory()
    h_cu = torch.from_numpy(wl.cu_seqlens).pin_memory()
    h_q = torch.empty(wl.q.shape, dtype=wl.q.dtype, pin_memory=True)
    h_k = torch.empty(wl.k.shape, dtype=wl.k.dtype, pin_memory=True)
    h_q.copy_(wl.q)
    h_k.copy_(wl.k)
    decode = wl.cache_len is not None
    npos = wl.qk_tokens
    h_pos = torch.empty((3, npos), dtype=torch.int32, pin_memory=True)
    h_start = torch.empty(wl.num_seqs, dtype=torch.int32, pin_memory=True)
    h_amount = torch.empty(wl.num_seqs, dtype=torch.int32, pin_memory=True)
    if decode:
        # per decode step the host sends the new tokens' Q/K and each
        # sequence's length and (start, amount) state, known from its prefill
        _, s, a = cmr.positions(h_ids.to(dev), h_cu.to(dev), wl.image_token_id)
        h_start.copy_(s)
        h_amount.copy_(a)
        h_cl = torch.from_numpy(wl.cache_len).pin_memory()
        # device buffers for the step; only the rotated dims of each head row
        # cross PCIe (cmr_copy_rotated_dims), as in the prefill pipeline
        d_q, d_k = torch.empty_like(wl.q), torch.empty_like(wl.k)
        d_cl = torch.empty_like(h_cl, device=dev)
        d_start = torch.empty_like(h_start, device=dev)
        d_amount = torch.empty_like(h_amount, device=dev)

    elif path == "pipeline":
        # prefill: chunks of whole prompts through a ring of device buffers,
        # host-to-device, kernels and device-to-host overlapped
        longest = int(np.diff(wl.cu_seqlens).max())
        chunk = max(longest, -(-wl.n_tokens // 16))
        pipe = pipeline.HostPipeline(dev, wl.num_layers, wl.hq, wl.hk, wl.head_dim, chunk,
                                     wl.num_seqs, depth=3)

    def step():
        if decode:
            for l in range(wl.num_layers):
                cmr.copy_rotated_dims(d_q[l], h_q[l], wl.rot_dim, stream)
                cmr.copy_rotated_dims(d_k[l], h_k[l], wl.rot_dim, stream)
            d_cl.copy_(h_cl, non_blocking=True)
            d_start.copy_(h_start, non_blocking=True)
            d_amount.copy_(h_amount, non_blocking=True)
            cmr.rotate_qk_shift(d_q, d_k, d_start, d_amount, pos_offset=d_cl, theta=wl.theta,
                                sections=wl.sections, rot_dim=wl.rot_dim)
            for l in range(wl.num_layers):
                cmr.copy_rotated_dims(h_q[l], d_q[l], wl.rot_dim, stream)
                cmr.copy_rotated_dims(h_k[l], d_k[l], wl.rot_dim, stream)
        elif path == "pipeline":
            pipe.run(h_ids, wl.cu_seqlens, h_q, h_k, h_pos, h_start, h_amount, wl.theta,
                     wl.sections, wl.rot_dim, wl.image_token_id, chunk_tokens=chunk)
        else:
            cmr.positions_rotate_qk_host(h_ids, h_cu, h_q, h_k, wl.theta, wl.sections,
                                         wl.rot_dim, wl.image_token_id,
                                         out=(h_pos, h_start, h_amount), device=dev,
                                         stream=stream)

    step()
    torch.cuda.synchronize(dev)
    if dist:
        dist.barrier()
    a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        step()
    z.record(stream)
    torch.cuda.synchronize(dev)
    ms = shard.max_over_ranks(a.elapsed_time(z), dist, dev)
    rot = (h_q.numel() + h_k.numel()) // wl.head_dim * wl.rot_dim * 2
    if decode:
        h2d = rot + 12 * wl.num_seqs
        d2h = rot
    else:
        # both prefill paths move only the rotated dims of every head row
        h2d = h_ids.numel() * 4 + h_cu.numel() * 4 + rot
        d2h = rot + h_pos.numel() * 4 + 8 * wl.num_seqs
    if decode:
        desc = ("pinned host -> rotated dims in (pitched copies), cmr.rotate_qk_shift, "
                "rotated dims out -> pinned host")
    elif path == "pipeline":
        desc = ("pinned host -> HostPipeline: chunks of whole prompts, rotated dims in "
                "(pitched copies), cmr.positions_rotate_qk, rotated dims out, on three "
                "streams -> pinned host")
    else:
        desc = ("pinned host -> cmr_positions_rotate_qk_host: the origin scan and the register "
                "rotate kernel read ids and the rotated dims of Q/K from the mapped pinned "
                "buffers over PCIe and write the rotated dims, planes and state back (zero-"
                "copy, no device buffers) -> pinned host")
    return {"value": tokens_all * steps / (ms / 1e3), "unit": UNIT,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "ms_per_step": ms / steps, "path": desc}


def build_parser():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", type=int, default=5, choices=[1, 2, 3, 4, 5],
                    help="1..5: single 80-token prompt, varlen 16, 64x4096 outliers, "
                         "decode 1024, 6 layers x 32 x 8192 (default)")
    ap.add_argument("--scaling", choices=["weak", "strong"], default="weak",
                    help="weak: a full batch per GPU (default); strong: one batch split by "
                         "whole prompts")
    ap.add_argument("--op", choices=["rotate", "shift", "cache", *PLANES_OPS], default="rotate",
                    help="rotate: planes from pos (default); shift: planes derived in the "
                         "rotate kernel; cache: rotate + KV-cache write; frames: the "
                         "multi-frame planes alone on their own workload; chunk: the planes "
                         "of a chunked prefill (cmr_positions_chunk) on that workload's "
                         "prompts with one thumbnail each")
    ap.add_argument("--prompts", type=int, default=256,
                    help="--op frames|chunk: prompts of 65,536 tokens in the batch")
    ap.add_argument("--chunks", type=int, default=4,
                    help="--op chunk: equal chunks per prompt, one call each")
    ap.add_argument("--rule", choices=sorted(cmr.RULES), default="canvas",
                    help="--op chunk: the position rule of cmr_positions_chunk")
    ap.add_argument("--grid-side", type=int, default=8,
                    help="--op frames: side of each frame's grid (8: 448x448 thumbnail)")
    ap.add_argument("--frames-per-prompt", type=int, default=32,
                    help="--op frames: frames in each of the 256 x 65,536-token prompts")
    ap.add_argument("--step", choices=["fused", "separate"], default="fused",
                    help="fused: a prefill rotate step is one cmr_positions_rotate_qk call "
                         "(default); separate: cmr_positions then cmr_rotate_qk, the rotate "
                         "launch timed on its own")
    ap.add_argument("--probe", choices=["copy-pattern"], default=None,
                    help="run only the copy-pattern ceiling probe (--steps launches)")
    ap.add_argument("--tiles-per-cta", type=int, default=1,
                    help="--probe copy-pattern: consecutive 8-token tiles per CTA (1: the "
                         "rotation's staging)")
    ap.add_argument("--launch", choices=["graph", "eager"], default="graph",
                    help="graph: replay a captured CUDA graph per call (default); eager: "
                         "launch through the Python binding every step")
    ap.add_argument("--layers", type=int, default=None,
                    help="override the workload's number of attention layers (Q/K redrawn)")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--reference-budget-s", type=float, default=150.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap


def main():
    args = build_parser().parse_args()
    args.warmup = max(3, args.warmup)  # at least 3 untimed warm-up steps
    if args.impl == "reference":
        return run_planes_reference(args) if args.op in PLANES_OPS else run_reference(args)
    if args.probe:
        return run_probe_only(args)
    if args.op in PLANES_OPS:
        return run_planes(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())

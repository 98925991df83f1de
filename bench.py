#!/usr/bin/env python3
"""Benchmark: MLA decode over a paged latent KV cache on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

--workload append_fp8_b64_t1 | append_fp8_bulk | append_bf16_bulk times the
latent-cache append kernel alone instead, and --workload proj_h128_n64 |
proj_h64_n4 the absorbed-MLA projections, and --workload agentic | prefix_h16
--cascade the prefix-shared (cascade) step beside the ordinary one (each its
own JSON line).

One step = one whole decode attention of the workload: the device planner
(K0), the main tcgen05 kernel (K1) and the split combine (K2), captured in a
CUDA graph. The default workload is the largest single-GPU configuration,
speculative decoding at a 1,048,576-token context: batch 1, 64 heads, q_len 4
(1 verified + 3 draft tokens, causal among the drafts), bf16 latent cache
~N(0, 0.5) in randomly permuted 64-token pages, q ~N(0, 1). The other
workloads (--workload kimi_50k, spec_128k, spec_256k, agentic, fp8, tiny) use
the same harness. Inputs are seeded synthetic data of those shapes (no
weights or datasets are involved).

L2: a step whose cache is smaller than 4 x L2 (126 MB) gets its page pool
replicated R times (R x step bytes >= 4 x L2), and step k reads replica k % R,
so every timed step reads its KV from HBM. The 1M step reads 1.2 GB: R = 1.

Prints one JSON line (rank 0). With --gpus N > 1 (torchrun) every rank runs an
independent replica of the step ("replicas only": the path has no exchange
step); the step time is the max over ranks.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "MLA decode µs/step, achieved HBM TB/s & fraction of roofline on 1 B200"
UNIT = "us/step"


# ---------------------------------------------------------------------------
# workload arithmetic (algorithmic bytes and flops of one step)
# ---------------------------------------------------------------------------

def step_work(w):
    """Algorithmic HBM bytes and tensor flops of one decode step."""
    L = w.seqlens.astype(np.int64)
    B, T, H = w.batch, w.q_len, w.heads
    c_kv = 1152 if w.kv_dtype == "bf16" else 580
    n_pages = (L + 63) // 64
    kv_bytes = int(L.sum()) * c_kv
    row_bytes = B * T * H * (1152 + 1024 + 4)
    meta_bytes = 4 * int(n_pages.sum()) + 4 * B
    vis = sum(int(Lb) - T + t + 1 for Lb in L for t in range(T))
    flops = 2 * H * (576 + 512) * vis
    # KV bytes with every physical page slot counted once (sequences that share
    # prefix pages read them once each in the per-sequence sum above)
    used = {}
    for b in range(B):
        n = int(n_pages[b])
        for i in range(n):
            slots = 64 if i < n - 1 else int(L[b]) - 64 * (n - 1)
            page = int(w.block_table[b, i])
            used[page] = max(used.get(page, 0), slots)
    unique_kv = sum(used.values()) * c_kv
    return {"bytes": kv_bytes + row_bytes + meta_bytes, "kv_bytes": kv_bytes, "flops": flops,
            "tokens": int(L.sum()), "unique_kv_bytes": unique_kv}


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# The sources that make up the decode kernel (K1); its recorded DRAM traffic
# stays valid while these are unchanged.
K1_SOURCES = ("mla_common.cuh", "mla_decode_kernel.cu", "mla_launch.h", "mla_ptx.cuh")


def kernel_source_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "mla_paged_kv_05_b200", "csrc")
    for name in K1_SOURCES:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload):
    """DRAM bytes per K1 launch from the committed ncu summary, if it was taken
    on the current kernel sources; else None. An entry may be scaled from a
    capture of a smaller case of the same kernel ("scaled_from": name, "scale":
    units of this launch / units of the captured one), where the full launch is
    too large to capture."""
    path = os.path.join(ROOT, "profiles", "k1_dram_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(workload)
    if not e:
        return None
    scale = 1.0
    if "scaled_from" in e:
        scale = float(e["scale"])
        e = d.get(e["scaled_from"])
        if not e:
            return None
    if e.get("kernel_sources") != kernel_source_hash():
        return None
    return int(round(e["dram_bytes_per_launch"] * scale))


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "50",
                 "-i", str(self.gpu)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=2)

    def summary(self, t0=None, t1=None):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ts, line in self.lines:
            if t0 is not None and (ts < t0 or ts > t1):
                continue
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# CPU oracle timing (baseline / reference arm)
# ---------------------------------------------------------------------------

# Both CPU legs (the cpu_baseline of our arm and the --impl reference arm) time
# the oracle on the same sample: the first ORACLE_SAMPLE_TOKENS tokens of every
# sequence. Every workload but the 128K-1M speculative steps fits in it whole.
ORACLE_SAMPLE_TOKENS = 65536


def time_oracle(w, budget_s: float, sample_tokens: int = ORACLE_SAMPLE_TOKENS):
    """Time the fp64 oracle, as it stands, on the first `sample_tokens` tokens
    of every sequence (all heads, all query tokens), repeated until the budget
    is spent (at least once). Returns (us per full step, sample text, cores):
    when a sequence is longer than the sample the time is extrapolated linearly
    in context tokens."""
    import oracle
    Ls = np.minimum(w.seqlens.astype(np.int64), sample_tokens)
    Ls = np.maximum(Ls, w.q_len)
    frac = float(w.seqlens.astype(np.int64).sum()) / float(Ls.sum())
    t_start = time.perf_counter()
    reps = 0
    while True:
        oracle.mla_decode_ref(w.q_bits, w.cache, w.kv_dtype, w.block_table, Ls.astype(np.int32), w.scale)
        reps += 1
        if time.perf_counter() - t_start >= budget_s:
            break
    per_sample = (time.perf_counter() - t_start) / reps
    cores = len(os.sched_getaffinity(0))
    if frac == 1.0:
        sample = (f"oracle (numpy fp64) on the whole step: {w.batch} sequence(s), all {w.q_len * w.heads} query "
                  f"rows, x{reps}")
    else:
        sample = (f"oracle (numpy fp64) on the first {int(Ls.max())} tokens of each sequence, all "
                  f"{w.q_len * w.heads} query rows, x{reps}; extrapolated x{frac:.2f} (linear in tokens) to the "
                  f"full step")
    return per_sample * frac * 1e6, sample, cores


# ---------------------------------------------------------------------------
# main
# ---------------------------------------------------------------------------

def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="spec_1m")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=None)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cascade", action="store_true", help="time the prefix-shared (cascade) step of the workload")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--clock-soak", type=float, default=1.0, help="seconds of untimed replays sampled for clocks")
    return ap.parse_args()


def max_over_ranks(values, device):
    """Each value's maximum over all ranks (the slowest replica's device time).
    Without an initialised process group of more than one rank the values come
    back unchanged."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t]


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def reference_arm(args, world, rank):
    from mla_paged_kv_05_b200 import inputs
    if rank != 0:
        return
    w = inputs.WORKLOADS[args.workload]()
    budget = max(1.0, min(120.0, 1.5 * (args.steps + args.warmup)))
    per_step_us, sample, cores = time_oracle(w, budget)
    ms = per_step_us / 1e3
    line = {
        "metric": METRIC, "value": per_step_us, "unit": UNIT, "impl": "reference", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {**w.describe(), "parallelism": "replicas only (rank 0 runs the oracle)"},
        "cpu_baseline": {"value": per_step_us, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": per_step_us, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# the latent-cache append (the write before a decode step), measured on its own
# ---------------------------------------------------------------------------

APPEND_WORKLOADS = {
    # name: (kv_dtype, batch, q_len, pages per sequence) - the fp8 batch's decode
    # step (64 sequences, one new token each) and bulk appends of 65,536 rows
    "append_fp8_b64_t1": ("fp8", 64, 1, 1024),
    "append_fp8_bulk": ("fp8", 16384, 4, 1),
    "append_bf16_bulk": ("bf16", 16384, 4, 1),
}


PROJ_WORKLOADS = {
    # name: (n_tokens, heads) - the absorbed projections around the 128-head
    # fp8 batch step (64 tokens) and the 64-head speculative step (4 tokens)
    "proj_h128_n64": (64, 128),
    "proj_h64_n4": (4, 64),
}


def proj_arm(args, world, rank, local):
    """Times the two absorbed-MLA projections (mla_absorb_q then
    mla_project_out) of one step: K pairs of launches in one CUDA graph, the
    weights rotating over replicas whose total exceeds 4 x L2. One JSON line."""
    import torch
    import torch.distributed as dist
    import mla_paged_kv_05_b200 as mla
    from mla_paged_kv_05_b200 import inputs

    N, H = PROJ_WORKLOADS[args.workload]
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", device_id=dev, timeout=__import__("datetime").timedelta(seconds=120))
    rng = np.random.default_rng(8)
    l2 = int(getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 126 * 2 ** 20))
    w_bytes = 2 * H * 128 * 512 * 2
    R = max(1, min(32, int(math.ceil(4 * l2 / w_bytes))))

    def bf16(shape, std):
        return torch.from_numpy(inputs.f32_to_bf16_bits(rng.standard_normal(shape).astype(np.float32) * std)
                                .view(np.int16)).view(torch.bfloat16).to(dev)

    w_uk = [bf16((H, 128, 512), 0.05) for _ in range(R)]
    w_uv = [bf16((H, 128, 512), 0.05) for _ in range(R)]
    q = bf16((N, H, 192), 1.0)
    o = bf16((N, H, 512), 0.3)
    q_out = torch.empty((N, H, 576), dtype=torch.bfloat16, device=dev)
    y = torch.empty((N, H, 128), dtype=torch.bfloat16, device=dev)
    flag = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        mla.absorb_q(q, w_uk[0], q_out, flag=flag, stream=stream)
        mla.project_out(o, w_uv[0], y, flag=flag, stream=stream)
    stream.synchronize()
    K, W = args.steps, args.warmup
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for k in range(K):
            mla.absorb_q(q, w_uk[k % R], q_out, flag=flag, stream=stream)
            mla.project_out(o, w_uv[k % R], y, flag=flag, stream=stream)
    with torch.cuda.stream(stream):
        for _ in range(max(W, 3)):
            g.replay()
    stream.synchronize()
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.2)
    t0 = time.time()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with torch.cuda.stream(stream):
        e0.record(stream)
        g.replay()
        e1.record(stream)
    torch.cuda.synchronize(dev)
    t1 = time.time()
    time.sleep(0.1)
    sampler.stop()
    clocks = sampler.summary(t0 - 0.1, t1 + 0.1)
    (ms,) = max_over_ranks([e0.elapsed_time(e1) / K], dev)
    nbytes = w_bytes + N * H * (192 + 576 + 512 + 128) * 2
    flops = 2 * 2 * N * H * 128 * 512
    peaks = load_peaks()
    achieved = nbytes / (ms / 1e3) / 1e9
    if rank == 0:
        print(json.dumps({
            "metric": "absorbed-MLA projections us/step (absorb + project)", "value": ms * 1e3, "unit": "us/step",
            "n_gpus": world, "steps": K, "warmup": W, "ms_per_step": ms, "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": args.workload, "n_tokens": N, "heads": H,
                       "l2": f"weights rotate over {R} replicas ({R * w_bytes / 2**20:.0f} MiB)",
                       "graph": "K (absorb, project) pairs captured in one CUDA graph"},
            "achieved_tflops": flops / (ms / 1e3) / 1e12,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / peaks["hbm_gbs"], "traffic": None,
                         "peak_source": f"{peaks['source']} (MEASURED_PEAKS.json)", "bytes_per_step": nbytes,
                         "flops_per_step": flops},
            "gpu_launches": 2 * K,
            "clocks": {k: clocks[k] for k in ("sm_mhz", "sm_max_mhz", "reasons")},
            "device_flag": int(flag.item()),
        }), flush=True)
    del g
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def cascade_arm(args, world, rank, local):
    """Times the prefix-shared (cascade) decode step of a workload whose
    sequences share a page-aligned prefix (--workload agentic | prefix_h16 with
    --cascade): K cascade steps in one CUDA graph against K ordinary steps of
    the same inputs. The page pool is replicated as in the ordinary bench so
    that every step reads HBM. One JSON line; value = the cascade step."""
    import torch
    import torch.distributed as dist
    import mla_paged_kv_05_b200 as mla
    from mla_paged_kv_05_b200 import inputs

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", device_id=dev, timeout=__import__("datetime").timedelta(seconds=120))
    w = inputs.WORKLOADS[args.workload]()
    prefix = inputs.cascade_prefix_len(w)
    if prefix == 0:
        raise SystemExit(f"{args.workload}: no shared prefix for a cascade step")
    work = step_work(w)
    peaks = load_peaks()
    l2 = int(getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 126 * 2 ** 20))
    R = 1 if work["unique_kv_bytes"] >= 4 * l2 else int(math.ceil(4 * l2 / max(work["unique_kv_bytes"], 1))) + 1
    R = max(1, min(R, 32))
    q = torch.from_numpy(w.q_bits.view(np.int16).copy()).view(torch.bfloat16).to(dev)
    base = (torch.from_numpy(w.cache.view(np.int16)).view(torch.bfloat16) if w.kv_dtype == "bf16"
            else torch.from_numpy(w.cache)).to(dev)
    P = base.shape[0]
    pool = torch.empty((R * P,) + tuple(base.shape[1:]), dtype=base.dtype, device=dev)
    for r in range(R):
        pool[r * P:(r + 1) * P].copy_(base)
    del base
    bt0 = torch.from_numpy(w.block_table).to(dev)
    bts = [(bt0 + r * P).contiguous() for r in range(R)]
    sl = torch.from_numpy(w.seqlens).to(dev)
    out = torch.empty((w.batch, w.q_len, w.heads, 512), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.batch, w.q_len, w.heads), dtype=torch.float32, device=dev)
    ws = torch.empty(mla.cascade_workspace_size(w.batch, w.max_pages, w.q_len, w.heads, w.kv_dtype),
                     dtype=torch.uint8, device=dev)
    dec = mla.MlaDecoder(w.batch, w.max_pages, w.q_len, w.heads, w.kv_dtype, device=dev)
    stream = torch.cuda.Stream(device=dev)

    def cascade_step(r):
        mla.cascade(q, pool, bts[r], sl, prefix, out, lse, ws, w.kv_dtype, w.scale, stream=stream)

    def plain_step(r):
        dec.plan(sl, stream=stream, block_table=bts[r], num_pages=int(pool.shape[0]))
        dec.run(q, pool, bts[r], sl, scale=w.scale, stream=stream)

    with torch.cuda.stream(stream):
        cascade_step(0)
        plain_step(0)
    stream.synchronize()
    flag = mla.read_device_flag(ws, stream)
    if flag != 0:
        raise RuntimeError(f"device flag {flag:#x} after the first cascade step")
    K, W = args.steps, args.warmup
    graphs = {}
    for name, fn in (("cascade", cascade_step), ("plain", plain_step)):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for k in range(K):
                fn(k % R)
        graphs[name] = g
    with torch.cuda.stream(stream):
        for _ in range(max(W, 3)):
            graphs["cascade"].replay()
            graphs["plain"].replay()
    stream.synchronize()
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.2)
    t0 = time.time()
    ms = {}
    for name in ("cascade", "plain"):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        with torch.cuda.stream(stream):
            e0.record(stream)
            graphs[name].replay()
            e1.record(stream)
        torch.cuda.synchronize(dev)
        ms[name] = e0.elapsed_time(e1) / K
    t1 = time.time()
    time.sleep(0.1)
    sampler.stop()
    clocks = sampler.summary(t0 - 0.1, t1 + 0.1)
    ms_c, ms_p = max_over_ranks([ms["cascade"], ms["plain"]], dev)
    ubytes = work["unique_kv_bytes"] + work["bytes"] - work["kv_bytes"]
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    bound = "hbm" if work["flops"] / ubytes < ridge else "tensor"
    if bound == "hbm":
        achieved, peak, unit = ubytes / (ms_c / 1e3) / 1e9, peaks["hbm_gbs"], "GB/s"
    else:
        achieved, peak, unit = work["flops"] / (ms_c / 1e3) / 1e12, peaks["bf16_tflops"], "TFLOP/s"
    if rank == 0:
        print(json.dumps({
            "metric": METRIC + " (prefix-shared cascade step)", "value": ms_c * 1e3, "unit": UNIT, "n_gpus": world,
            "steps": K, "warmup": W, "ms_per_step": ms_c, "higher_is_better": False, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16" if w.kv_dtype == "bf16" else "fp8-e4m3 cache, bf16 mma",
            "data": "synthetic",
            "config": {**w.describe(), "cascade_prefix_tokens": prefix,
                       "l2": f"inputs rotate over {R} page-pool replicas", "graph": "K steps in one CUDA graph"},
            "plain_step_us": ms_p * 1e3, "speedup_vs_plain": ms_p / ms_c,
            "unique_kv_bytes": work["unique_kv_bytes"], "algorithmic_bytes_unique": ubytes,
            "algorithmic_flops": work["flops"],
            "roofline": {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit, "frac": achieved / peak,
                         "traffic": None, "peak_source": f"{peaks['source']} (MEASURED_PEAKS.json, burst)",
                         "kernel": "whole cascade step (prep, prefix pass, suffix pass, merge), unique KV bytes"},
            "gpu_launches": 9 * K,
            "clocks": {k: clocks[k] for k in ("sm_mhz", "sm_max_mhz", "reasons")},
            "device_flag": flag,
        }), flush=True)
    del graphs
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def append_arm(args, world, rank, local):
    """Times mla_cache_append alone: K launches captured in one CUDA graph, new
    rows rotating over replicas whose total exceeds 4 x L2, page ids drawn from
    a shuffled pool. One JSON line (rank 0)."""
    import torch
    import torch.distributed as dist
    import mla_paged_kv_05_b200 as mla
    from mla_paged_kv_05_b200 import inputs

    kv_dtype, B, T, maxp = APPEND_WORKLOADS[args.workload]
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", device_id=dev, timeout=__import__("datetime").timedelta(seconds=120))
    rng = np.random.default_rng(7)
    rows = B * T
    row_in, row_out = 1152, (1152 if kv_dtype == "bf16" else 580)
    l2 = int(getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 126 * 2 ** 20))
    R = max(1, min(32, int(math.ceil(4 * l2 / (rows * row_in)))))
    pages = B * maxp + 1
    # every replica has its own shuffled block table, so successive launches
    # write different pages of the pool
    bts = [torch.from_numpy(rng.permutation(pages).astype(np.int32)[:B * maxp].reshape(B, maxp).copy()).to(dev)
           for _ in range(R)]
    bt = bts[0]
    lens = rng.integers(T, maxp * 64 + 1, size=B).astype(np.int32)
    sl = torch.from_numpy(lens).to(dev)
    if kv_dtype == "bf16":
        cache = torch.zeros((pages, 64, 576), dtype=torch.bfloat16, device=dev)
    else:
        cache = torch.zeros((pages, inputs.FP8_PAGE_BYTES), dtype=torch.uint8, device=dev)
    new = [torch.from_numpy(inputs.f32_to_bf16_bits(rng.standard_normal((B, T, 576)).astype(np.float32) * 0.5)
                            .view(np.int16)).view(torch.bfloat16).to(dev) for _ in range(R)]
    flag = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        mla.append(new[0], cache, bt, sl, kv_dtype, flag=flag, stream=stream)
    stream.synchronize()
    K, W = args.steps, args.warmup
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for k in range(K):
            mla.append(new[k % R], cache, bts[k % R], sl, kv_dtype, flag=flag, stream=stream)
    with torch.cuda.stream(stream):
        for _ in range(max(W, 3)):
            g.replay()
    stream.synchronize()
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.2)
    t0 = time.time()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with torch.cuda.stream(stream):
        e0.record(stream)
        g.replay()
        e1.record(stream)
    torch.cuda.synchronize(dev)
    t1 = time.time()
    time.sleep(0.1)
    sampler.stop()
    clocks = sampler.summary(t0 - 0.1, t1 + 0.1)
    (ms,) = max_over_ranks([e0.elapsed_time(e1) / K], dev)
    nbytes = rows * (row_in + row_out) + rows * 4 + B * 4
    peaks = load_peaks()
    achieved = nbytes / (ms / 1e3) / 1e9
    if rank == 0:
        print(json.dumps({
            "metric": "latent-cache append us/launch", "value": ms * 1e3, "unit": "us/launch", "n_gpus": world,
            "steps": K, "warmup": W, "ms_per_step": ms, "higher_is_better": False, "scaling": "weak",
            "vs_baseline": None, "dtype": f"bf16 in, {kv_dtype} cache", "data": "synthetic",
            "config": {"workload": args.workload, "batch": B, "q_len": T, "rows": rows, "kv_dtype": kv_dtype,
                       "l2": f"new rows and block tables rotate over {R} replicas ({R * rows * row_in / 2**20:.0f} "
                             f"MiB of rows)",
                       "graph": "K launches captured in one CUDA graph"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / peaks["hbm_gbs"], "traffic": None,
                         "peak_source": f"{peaks['source']} (MEASURED_PEAKS.json)",
                         "bytes_per_launch": nbytes},
            "gpu_launches": K,
            "clocks": {k: clocks[k] for k in ("sm_mhz", "sm_max_mhz", "reasons")},
            "device_flag": int(flag.item()),
        }), flush=True)
    del g
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    args = parse()
    world, rank, local = dist_setup(args)
    if args.workload in PROJ_WORKLOADS:
        if args.impl == "reference":
            if rank == 0:
                print(json.dumps({"impl": "reference", "unavailable": "the projections are measured on the GPU only"}))
            return
        proj_arm(args, world, rank, local)
        return
    if args.cascade:
        if args.impl == "reference":
            reference_arm(args, world, rank)
        else:
            cascade_arm(args, world, rank, local)
        return
    if args.workload in APPEND_WORKLOADS:
        if args.impl == "reference":
            if rank == 0:
                print(json.dumps({"impl": "reference", "unavailable": "the append is measured on the GPU only"}))
            return
        append_arm(args, world, rank, local)
        return
    if args.impl == "reference":
        reference_arm(args, world, rank)
        return

    import torch
    import torch.distributed as dist
    from cuda.bindings import runtime as cudart

    import mla_paged_kv_05_b200 as mla
    from mla_paged_kv_05_b200 import inputs

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", device_id=dev, timeout=__import__("datetime").timedelta(seconds=120))

    w = inputs.WORKLOADS[args.workload]()
    work = step_work(w)
    peaks = load_peaks()
    props = torch.cuda.get_device_properties(dev)
    l2 = int(getattr(props, "L2_cache_size", 126 * 2 ** 20))

    # ---- device inputs, R page-pool replicas so that every step misses L2
    kv_step_bytes = work["kv_bytes"]
    R = 1 if kv_step_bytes >= 4 * l2 else int(math.ceil(4 * l2 / max(kv_step_bytes, 1))) + 1
    R = max(1, min(R, 64))
    q = torch.from_numpy(w.q_bits.view(np.int16).copy()).view(torch.bfloat16).to(dev)
    if w.kv_dtype == "bf16":
        base = torch.from_numpy(w.cache.view(np.int16)).view(torch.bfloat16).to(dev)
    else:
        base = torch.from_numpy(w.cache).to(dev)
    P = base.shape[0]
    pool = torch.empty((R * P,) + tuple(base.shape[1:]), dtype=base.dtype, device=dev)
    for r in range(R):
        pool[r * P:(r + 1) * P].copy_(base)
    del base
    bt0 = torch.from_numpy(w.block_table).to(dev)
    bts = [(bt0 + r * P).contiguous() for r in range(R)]
    sl = torch.from_numpy(w.seqlens).to(dev)
    dec = mla.MlaDecoder(w.batch, w.max_pages, w.q_len, w.heads, w.kv_dtype, device=dev)
    stream = torch.cuda.Stream(device=dev)

    NP = int(pool.shape[0])

    def step(r, evs=None):
        dec.plan(sl, stream=stream, block_table=bts[r], num_pages=NP)
        if evs is None:
            dec.run(q, pool, bts[r], sl, scale=w.scale, stream=stream)
        else:
            s = cudart.cudaStream_t(stream.cuda_stream)
            cudart.cudaEventRecordWithFlags(evs[0], s, cudart.cudaEventRecordExternal)
            mla.run(q, pool, bts[r], sl, dec.out, dec.lse, dec.workspace, w.kv_dtype, w.scale,
                    stream=stream, phases=mla.PHASE_ATTEND)
            cudart.cudaEventRecordWithFlags(evs[1], s, cudart.cudaEventRecordExternal)
            mla.run(q, pool, bts[r], sl, dec.out, dec.lse, dec.workspace, w.kv_dtype, w.scale,
                    stream=stream, phases=mla.PHASE_COMBINE)
            cudart.cudaEventRecordWithFlags(evs[2], s, cudart.cudaEventRecordExternal)

    # eager run once: correctness flag + lazy init outside capture
    with torch.cuda.stream(stream):
        step(0)
    stream.synchronize()
    flag = dec.device_flag(stream)
    if flag != 0:
        raise RuntimeError(f"device flag {flag:#x} after the first step")

    # ---- graphs: one single-step graph per replica (warm-up, clock soak) and
    # one graph holding exactly K steps with external event nodes around K1.
    K, W = args.steps, args.warmup
    ev_k1 = []
    for _ in range(K):
        ev_k1.append(tuple(cudart.cudaEventCreate()[1] for _ in range(3)))
    single = []
    for r in range(R):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            step(r)
        single.append(g)
    gK = torch.cuda.CUDAGraph()            # exactly K steps: the timed region
    with torch.cuda.graph(gK, stream=stream):
        for k in range(K):
            step(k % R)
    gK_ev = torch.cuda.CUDAGraph()         # the same K steps with event nodes around K1 and K2
    with torch.cuda.graph(gK_ev, stream=stream):
        for k in range(K):
            step(k % R, ev_k1[k])

    gK1 = torch.cuda.CUDAGraph()           # K back-to-back K1 launches (the period)
    with torch.cuda.graph(gK1, stream=stream):
        for k in range(K):
            mla.run(q, pool, bts[k % R], sl, dec.out, dec.lse, dec.workspace, w.kv_dtype, w.scale,
                    stream=stream, phases=mla.PHASE_ATTEND)
    k1_s0 = torch.cuda.Event(enable_timing=True)
    k1_s1 = torch.cuda.Event(enable_timing=True)

    with torch.cuda.stream(stream):
        for i in range(max(W, 3)):
            single[i % R].replay()
    stream.synchronize()

    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    t_soak = time.time()
    with torch.cuda.stream(stream):
        n = 0
        while time.time() - t_soak < args.clock_soak:
            for _ in range(50):
                single[n % R].replay()
                n += 1
            stream.synchronize()
    # One untimed replay of each graph timed below: a graph's first launch also
    # uploads it to the device, a one-time cost a serving loop does not pay per step.
    with torch.cuda.stream(stream):
        gK.replay()
        gK_ev.replay()
    stream.synchronize()
    # ---- timed region: exactly K steps
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    t_wall0 = time.time()
    with torch.cuda.stream(stream):       # CUDAGraph.replay() launches on the current stream
        start.record(stream)
        gK.replay()
        end.record(stream)
    torch.cuda.synchronize(dev)
    t_wall1 = time.time()
    # Per-kernel durations from a replay of the event-instrumented graph right
    # after the timed one, in the same thermal and power state (the clock
    # sampler still runs). The event nodes between a step's kernels also stop
    # the launch overlap between them, so each K1 here runs on its own, set-up
    # included: the roofline's kernel time.
    with torch.cuda.stream(stream):
        gK_ev.replay()
    stream.synchronize()
    # K1's period back to back: K launches of the decode kernel (same plan,
    # rotating replicas) in one graph, each launch's set-up overlapping the
    # previous one's tail. Reported beside the isolated time.
    with torch.cuda.stream(stream):
        gK1.replay()
        k1_s0.record(stream)
        gK1.replay()
        k1_s1.record(stream)
    stream.synchronize()
    k1_b2b_ms = k1_s0.elapsed_time(k1_s1) / K
    t_wall2 = time.time()
    if world > 1:
        dist.barrier()

    ms_total = start.elapsed_time(end)
    k1_ms, k2_ms = [], []
    for a, b, c in ev_k1:
        k1_ms.append(float(cudart.cudaEventElapsedTime(a, b)[1]))
        k2_ms.append(float(cudart.cudaEventElapsedTime(b, c)[1]))
    k1_avg_ms = float(np.mean(k1_ms))
    k2_avg_ms = float(np.mean(k2_ms))
    ms_total, k1_avg_ms, k2_avg_ms, k1_b2b_ms = max_over_ranks([ms_total, k1_avg_ms, k2_avg_ms, k1_b2b_ms], dev)
    ms_step = ms_total / K
    us_step = ms_step * 1e3
    flag = dec.device_flag(stream)

    # ---- end to end through the public API with host buffers. The step's
    # inputs (q, seqlens, block table) sit in one pinned host buffer and go over
    # in one copy into one device buffer; out and lse come back the same way.
    E = args.e2e_steps or max(20, min(K, 200))
    q_bytes, sl_bytes, bt_bytes = q.numel() * 2, sl.numel() * 4, bts[0].numel() * 4
    off_sl = (q_bytes + 255) // 256 * 256
    off_bt = off_sl + (sl_bytes + 255) // 256 * 256
    in_bytes = off_bt + bt_bytes
    out_bytes = dec.out.numel() * 2
    off_lse = (out_bytes + 255) // 256 * 256
    res_bytes = off_lse + dec.lse.numel() * 4
    in_h = [torch.empty(in_bytes, dtype=torch.uint8).pin_memory() for _ in range(R)]
    for r in range(R):
        in_h[r][:q_bytes].copy_(q.view(torch.uint8).reshape(-1).cpu())
        in_h[r][off_sl:off_sl + sl_bytes].copy_(sl.view(torch.uint8).reshape(-1).cpu())
        in_h[r][off_bt:off_bt + bt_bytes].copy_(bts[r].view(torch.uint8).reshape(-1).cpu())
    # Two device copies of the step's buffers (and of the pinned result buffer):
    # step n uses set n % 2, so that step n + 1's inputs can go over while step n
    # computes, and step n's results come back while step n + 1 computes.
    res_h = [torch.empty(res_bytes, dtype=torch.uint8).pin_memory() for _ in range(2)]
    in_d = [torch.empty(in_bytes, dtype=torch.uint8, device=dev) for _ in range(2)]
    res_d = [torch.empty(res_bytes, dtype=torch.uint8, device=dev) for _ in range(2)]
    q_d = [x[:q_bytes].view(torch.bfloat16).view(q.shape) for x in in_d]
    sl_d = [x[off_sl:off_sl + sl_bytes].view(torch.int32) for x in in_d]
    bt_d = [x[off_bt:off_bt + bt_bytes].view(torch.int32).view(bts[0].shape) for x in in_d]
    out_d = [x[:out_bytes].view(torch.bfloat16).view(dec.out.shape) for x in res_d]
    lse_d = [x[off_lse:off_lse + dec.lse.numel() * 4].view(torch.float32).view(dec.lse.shape) for x in res_d]
    h2d = q_bytes + sl_bytes + bt_bytes
    d2h = out_bytes + dec.lse.numel() * 4
    s_in = torch.cuda.Stream(device=dev)    # host -> device copies
    s_out = torch.cuda.Stream(device=dev)   # device -> host copies

    def compute(n):
        b = n % 2
        mla.plan(sl_d[b], w.max_pages, w.q_len, w.heads, dec.workspace, w.kv_dtype, stream=stream,
                 block_table=bt_d[b], num_pages=NP)
        mla.run(q_d[b], pool, bt_d[b], sl_d[b], out_d[b], lse_d[b], dec.workspace, w.kv_dtype, w.scale,
                stream=stream)

    def pipeline(n_steps):
        """n_steps end-to-end steps on `stream`, as a serving loop runs them: every
        step copies its inputs in from pinned host memory, plans, runs, and copies
        its results out; the copies run on their own streams (copy engines), step
        n + 1's input copy beside step n's kernels."""
        ev_in = [torch.cuda.Event() for _ in range(n_steps)]
        ev_done = [torch.cuda.Event() for _ in range(n_steps)]
        ev_out = [torch.cuda.Event() for _ in range(n_steps)]
        s_in.wait_stream(stream)
        s_out.wait_stream(stream)
        for n in range(n_steps):
            b = n % 2
            if n >= 2:
                s_in.wait_event(ev_done[n - 2])      # step n - 2 has finished with set b's inputs
            with torch.cuda.stream(s_in):
                in_d[b].copy_(in_h[n % R], non_blocking=True)
            ev_in[n].record(s_in)
            stream.wait_event(ev_in[n])
            if n >= 2:
                stream.wait_event(ev_out[n - 2])     # step n - 2's results have left set b
            compute(n)
            ev_done[n].record(stream)
            s_out.wait_event(ev_done[n])
            with torch.cuda.stream(s_out):
                res_h[b].copy_(res_d[b], non_blocking=True)
            ev_out[n].record(s_out)
        stream.wait_stream(s_in)
        stream.wait_stream(s_out)

    with torch.cuda.stream(stream):
        pipeline(2)                           # lazy set-up outside capture
    stream.synchronize()
    g_e2e = torch.cuda.CUDAGraph()            # exactly E end-to-end steps
    with torch.cuda.graph(g_e2e, stream=stream):
        pipeline(E)
    # The same soak as the device-resident leg before the timed replay, so that
    # both legs are timed in the same power state (the sampler still runs); the
    # soak's first replay also uploads the graph.
    t_e0 = time.time()
    with torch.cuda.stream(stream):
        n = 0
        while n < 2 or time.time() - t_e0 < args.clock_soak:
            g_e2e.replay()
            stream.synchronize()
            n += 1
        if world > 1:
            dist.barrier()
        s0 = torch.cuda.Event(enable_timing=True)
        s1 = torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        g_e2e.replay()
        s1.record(stream)
        stream.synchronize()
    t_e1 = time.time()
    e2e_ms = s0.elapsed_time(s1) / E
    del g_e2e
    (e2e_ms,) = max_over_ranks([e2e_ms], dev)
    time.sleep(0.2)
    sampler.stop()
    clocks = sampler.summary(t_soak, t_wall2 + 0.1)
    e2e_clocks = sampler.summary(t_e0, t_e1 + 0.1)

    # ---- roofline of the dominant kernel (K1, timed on its own) and of the whole step
    k1_s = k1_avg_ms / 1e3
    intensity = work["flops"] / work["bytes"]
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    bound = "hbm" if intensity < ridge else "tensor"
    # A tensor-bound K1 timed while the clock record shows the power cap is a
    # kernel inside a sustained load: its denominator is the sustained bf16
    # figure; otherwise the burst one.
    capped = "sw_power_cap" in clocks["reasons"]
    tflops_peak = peaks["bf16_tflops_sustained"] if capped else peaks["bf16_tflops"]
    if bound == "hbm":
        achieved, peak, unit = work["bytes"] / k1_s / 1e9, peaks["hbm_gbs"], "GB/s"
        peak_kind = "HBM copy"
    else:
        achieved, peak, unit = work["flops"] / k1_s / 1e12, tflops_peak, "TFLOP/s"
        peak_kind = "bf16 sustained (power-capped run)" if capped else "bf16 burst"
    t_roof = max(work["bytes"] / (peaks["hbm_gbs"] * 1e9), work["flops"] / (tflops_peak * 1e12))
    traffic = recorded_traffic(args.workload)

    if rank == 0:
        cpu = None
        if not args.no_cpu_baseline and world == 1:
            us, sample, cores = time_oracle(w, args.cpu_budget)
            cpu = {"value": us, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample}
        line = {
            "metric": METRIC, "value": us_step, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": W,
            "ms_per_step": ms_step, "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if w.kv_dtype == "bf16" else "fp8-e4m3 cache, bf16 mma", "data": "synthetic",
            "config": {**w.describe(), "parallelism": "replicas only" if world > 1 else "single GPU",
                       "l2": f"inputs rotate over {R} page-pool replicas ({R * kv_step_bytes / 2**20:.0f} MiB "
                             f"of KV, L2 {l2 / 2**20:.0f} MiB)",
                       "graph": "K steps captured in one CUDA graph (kernel_us from an event-instrumented replay "
                                "right after it, same clock record)"},
            "achieved_tbs": work["bytes"] / (ms_step / 1e3) / 1e12,
            "achieved_tflops": work["flops"] / (ms_step / 1e3) / 1e12,
            "roofline_frac_step": t_roof / (ms_step / 1e3),
            "algorithmic_bytes": work["bytes"], "algorithmic_flops": work["flops"],
            "unique_kv_bytes": work["unique_kv_bytes"],
            "kernel_us": {"k1_attend": k1_avg_ms * 1e3, "k2_combine": k2_avg_ms * 1e3,
                          "k1_back_to_back_period": k1_b2b_ms * 1e3,
                          "note": "k1/k2: event nodes between each step's kernels (no launch overlap); "
                                  "period: K back-to-back K1 launches, set-up overlapping the previous tail"},
            "roofline": {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
                         "frac": achieved / peak, "traffic": traffic,
                         "peak_source": f"{peaks['source']} (MEASURED_PEAKS.json, {peak_kind})",
                         "kernel": "K1 decode kernel, isolated launch (kernel_us.k1_attend)"},
            "e2e": {"value": e2e_ms * 1e3, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "how": ("pinned H2D copy + plan + run + D2H copy per step; E steps in one CUDA graph, pipelined "
                            "as a serving loop runs them (step n+1's input copy and step n-1's result copy on "
                            "their own streams beside step n's kernels)"),
                    "steps": E,
                    "sm_mhz": e2e_clocks["sm_mhz"], "reasons": e2e_clocks["reasons"]},
            "gpu_launches": 3 * K,
            "clocks": {k: clocks[k] for k in ("sm_mhz", "sm_max_mhz", "reasons")},
            "clock_samples": clocks["samples"],
            "device_flag": flag,
        }
        if cpu is not None:
            line["cpu_baseline"] = cpu
        print(json.dumps(line), flush=True)

    for evs in ev_k1:
        for e in evs:
            cudart.cudaEventDestroy(e)
    del gK, gK_ev, gK1, single
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

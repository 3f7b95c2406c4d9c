#!/usr/bin/env python
"""Benchmark of the gated local/full decode-attention step on B200.

Workloads (--workload):
  ctx128k (default, the headline): batch 1, 28 layers of GQA attention (16
      query / 8 KV heads, head_dim 128, bf16), context t = 131072 at the first
      step and growing by one per step, s = 4 sinks + w = 2048 window for
      Local, Full recomputation on a Bernoulli(0.125) draw per step;
  ctx16k: batch 8, one layer, t = 16384, Full calls Bernoulli(0.41) per row,
      one planted needle per flagged row;
  mixed: batch 32, one layer, t uniform in [4096, 65536] per row, Full calls
      Bernoulli(--rate) per row;
  recall: batch 16, one layer, t = --context (4096 or 131072) for every row,
      the recall head's own scores decide the gate (theta = 0).
Every workload runs the 6144 -> 4096 -> 1 recall head each step. One "step"
= one decode step of the whole path (append, Local per layer, recall head with
the gate, Full per layer when a row is flagged) replayed from a captured CUDA
graph; inputs are resident in HBM and fed with one device copy per step.
Workloads whose per-step reads would fit the 126 MB L2 rotate through
--copies independently allocated copies of the KV state.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl oda|reference]
                    [--workload ctx128k|ctx16k|mixed|recall] [--rate R] [--context T]

Prints one JSON line (rank 0). Under torchrun every rank runs an independent
replica (the path has no cross-request exchange) and the time is the max
over ranks.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "decode-attn tokens/s & KV GB/s vs HBM roofline, 128K ctx, 12.5% full calls"
UNIT = "tokens/s"
KV_BYTES_PER_TOKEN_LAYER = 2 * 8 * 128 * 2      # K and V, 8 KV heads, d=128, bf16
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0                        # B200 HBM3e, nominal
WORKLOADS = ("ctx128k", "ctx16k", "mixed", "recall")


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1024)
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--impl", choices=["oda", "reference"], default="oda")
    ap.add_argument("--workload", choices=WORKLOADS, default="ctx128k")
    ap.add_argument("--layers", type=int, default=28, help="layers of the ctx128k workload")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--cpu-steps", type=int, default=4,
                    help="decode steps in the oracle's bounded sample (a quarter flagged)")
    ap.add_argument("--cpu-workers", type=int, default=0,
                    help="oracle worker processes (0: every core this process may use)")
    ap.add_argument("--copies", type=int, default=0,
                    help="independent KV-state copies the steps rotate through "
                         "(0: 1 for ctx128k, 3 otherwise)")
    ap.add_argument("--launch", choices=["graph", "plain"], default="graph",
                    help="graph: captured step with the IF node; plain: the same kernels "
                         "launched one by one (visible to ncu)")
    ap.add_argument("--context", type=int, default=None,
                    help="context length t at the first step (ctx128k: 131072; recall: "
                         "131072 or 4096)")
    ap.add_argument("--rate", type=float, default=None,
                    help="Full-call rate (ctx128k: Bernoulli per step, default 0.125; mixed: "
                         "Bernoulli per row, default 0.125)")
    ap.add_argument("--mode", choices=["oda", "full-only", "recall-loss"], default="oda",
                    help="full-only: every step appends and runs Full attention in every "
                         "layer, no Local, recall head or gate (dense decode, for the "
                         "speedup and the short-context crossover; ctx128k only); recall-loss: "
                         "the recall head's training objective over --positions positions")
    ap.add_argument("--positions", type=int, default=1 << 24,
                    help="positions per recall-loss call (--mode recall-loss)")
    a = ap.parse_args(argv)
    if a.context is None:
        a.context = 131072
    if a.rate is None and a.workload in ("ctx128k", "mixed"):
        a.rate = 0.125
    if a.mode == "full-only" and a.workload != "ctx128k":
        ap.error("--mode full-only runs the ctx128k request only")
    return a


# ----------------------------------------------------------------------------
# distributed plumbing (replicas only; the collectives here are for timing)
# ----------------------------------------------------------------------------

def dist_init(backend: str = "nccl"):
    """(rank, world_size, local_rank) from the torchrun environment; NCCL on
    GPUs, gloo for the CPU tests of this plumbing."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws <= 1:
        return 0, 1, 0
    import datetime
    import torch
    import torch.distributed as dist
    local = int(os.environ.get("LOCAL_RANK", "0"))
    kw = {}
    if backend == "nccl":
        torch.cuda.set_device(local)
        kw["device_id"] = torch.device("cuda", local)
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120), **kw)
    return dist.get_rank(), ws, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, ws: int) -> float:
    """Max of a per-rank time over all ranks (the job's time)."""
    if ws <= 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: int, ws: int, seconds_max: float) -> float:
    """Whole-job units per second: all ranks' units over the slowest rank's time."""
    return units_per_rank * ws / seconds_max


# ----------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.samples = []
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", gpu_id, f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()
        t0 = time.time()
        while not self.samples and time.time() - t0 < 5:
            time.sleep(0.05)

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), line.strip()))

    def stop(self):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0: float, t1: float) -> dict:
        rows = [s for (ts, s) in self.samples if t0 - 0.15 <= ts <= t1 + 0.15] or \
               [s for (_, s) in self.samples]
        sm, mx, reasons = [], 0.0, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for r in rows:
            p = [x.strip() for x in r.split(",")]
            if len(p) < 8:
                continue
            try:
                sm.append(float(p[0]))
                mx = max(mx, float(p[1]))
            except ValueError:
                continue
            for name, v in zip(names, p[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": mx or None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------------------
# workloads and their algorithmic bytes (KV actually read + KV written)
# ----------------------------------------------------------------------------

def make_workload(args, n_steps: int):
    """(Workload, external_scores) for --workload with n_steps decode steps.
    external_scores: the gate reads the workload's drawn flags (as +-1
    scores) instead of the recall head's output."""
    import synth
    wl = getattr(args, "workload", "ctx128k")
    rate = getattr(args, "rate", None)
    if wl == "ctx128k":
        w = synth.ctx128k(steps=n_steps, layers=getattr(args, "layers", 28),
                          context=getattr(args, "context", None) or 131072,
                          rate=0.125 if rate is None else rate)
    elif wl == "ctx16k":
        w = synth.ctx16k(steps=n_steps)
    elif wl == "mixed":
        w = synth.mixed_batch(0.125 if rate is None else rate, steps=n_steps)
    elif wl == "recall":
        w = synth.recall_step(getattr(args, "context", None) or 131072, steps=n_steps)
        return w, False
    else:
        raise ValueError(wl)
    w.recall = True                  # the recall head runs every step
    return w, True


def step_kv_bytes(t: int, flagged: bool, layers: int, s=4, w=2048) -> int:
    """One row's algorithmic KV bytes of one step at context t."""
    local = min(t, s + w)
    full = t if flagged else 0
    return layers * (local + full + 2) * KV_BYTES_PER_TOKEN_LAYER


def model_speedup(t: int, rho: float, s=4, w=2048) -> float:
    """Dense decode's KV bytes per step over ODA's at Full-call rate rho (both
    append the token; ODA reads the Local set every step and the whole
    history on a fraction rho of steps). It tends to 1/rho as t grows."""
    dense = t + 2
    oda = min(t, s + w) + rho * t + 2
    return dense / oda


def batch_step_bytes(w, j: int, flags_j) -> int:
    """All rows of step j: Local reads, Full reads of flagged rows, appended K/V."""
    return sum(step_kv_bytes(int(w.t0[b]) + j, bool(flags_j[b]), w.layers, w.sink, w.window)
               for b in range(w.batch))


def gpu_id(local: int) -> str:
    """nvidia-smi id of this process's GPU (UUID when torch exposes it)."""
    import torch
    try:
        u = str(torch.cuda.get_device_properties(local).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
        return vis.split(",")[local] if vis else str(local)


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


KERNEL_SOURCES = ("attn.cu", "plan.cuh", "oda_internal.cuh")


def _code_only(text: str) -> str:
    """C++ source without // and /* */ comments or blank space, so that an
    edit of comments alone keeps the digest (the kernel is unchanged)."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    return "\n".join(" ".join(line.split()) for line in text.splitlines() if line.strip())


def kernel_src_sha1() -> str:
    """Digest of the attention kernel's code (what the ncu counters were taken on)."""
    h = hashlib.sha1()
    for f in KERNEL_SOURCES:
        src = open(os.path.join(ROOT, "gated_local_full_b200", "csrc", f)).read()
        h.update(_code_only(src).encode())
    return h.hexdigest()


def replay_seconds(torch, fn, stream) -> float:
    """Device time of the launches `fn` makes: captured once in a CUDA graph,
    replayed once to warm up, then timed between CUDA events on `stream`."""
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        fn()
    stream.wait_stream(side)
    with torch.cuda.stream(stream):
        g.replay()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        g.replay()
        b.record(stream)
    torch.cuda.synchronize()
    del g
    return a.elapsed_time(b) / 1000.0


def recorded_traffic():
    """Per-launch DRAM traffic of the Full-attention kernel from the committed
    ncu summary, if it was taken on the current kernel source."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    if not os.path.exists(p):
        return None, None
    d = json.load(open(p))
    if d.get("kernel_src_sha1") != kernel_src_sha1():
        return None, d
    return d.get("full_attn_traffic_bytes_per_launch_128k"), d


# ----------------------------------------------------------------------------
# the CPU oracle on a bounded sample (cpu_baseline leg and --impl reference)
#
# A sample of (kind, row, layer, KV head) tasks of a few decode steps is split
# over a pool of worker processes (started with spawn, one BLAS thread each).
# Each worker generates its tasks' inputs first; then all pass a barrier and
# the parent times the oracle calls alone, from the barrier to the last
# worker's end. A full step's time is extrapolated from the per-task means
# and the measured parallel speedup, and every factor is reported.
# ----------------------------------------------------------------------------

def _wl_spec(args) -> dict:
    return {"workload": getattr(args, "workload", "ctx128k"), "layers": getattr(args, "layers", 28),
            "context": getattr(args, "context", None), "rate": getattr(args, "rate", None)}


def _kv_rows(w, layer, row, g, positions):
    """float64 K, V [1][t][d] of one (layer, row, KV head) holding the listed
    positions (others 0), from the shared seeded generator."""
    from synth.gen import table_values
    pos = sorted(positions)
    t = pos[-1]
    K = np.zeros((1, t, w.d))
    V = np.zeros((1, t, w.d))
    tab = w.kv_table()
    runs, start, prev = [], pos[0], pos[0]
    for p in pos[1:]:
        if p != prev + 1:
            runs.append((start, prev))
            start = p
        prev = p
    runs.append((start, prev))
    for kv, dst in ((0, K), (1, V)):
        key = w.kv_key(layer, row, g, kv)
        for a, b in runs:
            vals = table_values(key, (a - 1) * w.d, (b - a + 1) * w.d, tab).reshape(-1, w.d)
            dst[0, a - 1:b] = w.to_f64(vals)
        if kv == 0:
            for n in w.needles:
                if (n.layer, n.row, n.kv_head) == (layer, row, g) and n.position <= t:
                    dst[0, n.position - 1] = w.to_f64(n.key)
    return K, V


def _prepare_task(w, task, cache):
    import oracle as O  # test infrastructure; only the baseline leg runs it
    kind, j, layer, row, g = task
    if kind == "recall":
        from synth import bf16_bits_to_f32
        if "W" not in cache:
            W1, b1, w2, b2 = w.recall_weights()
            cache["W"] = (bf16_bits_to_f32(W1).astype(np.float64), b1.astype(np.float64),
                          bf16_bits_to_f32(w2).astype(np.float64), float(b2))
        hs = [bf16_bits_to_f32(h).astype(np.float64) for h in w.hidden_step(j)]
        return (kind, hs, cache["W"])
    t = int(w.t0[row]) + j
    G = w.group
    q = w.to_f64(w.q_step_layer(j, layer)[row][g * G:(g + 1) * G])
    if kind == "local":
        K, V = _kv_rows(w, layer, row, g, O.local_access_set(t, w.sink, w.window))
    else:
        K, V = _kv_rows(w, layer, row, g, range(1, t + 1))
    return (kind, q, K, V, t)


def _run_task(w, prep):
    import oracle as O
    if prep[0] == "recall":
        _, hs, (W1, b1, w2, b2) = prep
        score = O.recall_score(*hs, W1, b1, w2, b2)
        O.gate(score.astype(np.float32), 0.0)
    elif prep[0] == "local":
        _, q, K, V, t = prep
        O.local_attention(q, K, V, t, w.sink, w.window)
    else:
        _, q, K, V, t = prep
        O.full_attention(q, K, V, t)


def _oracle_worker(spec, n_steps, tasks, start_barrier, out_q):
    """One worker process: generate the inputs of its tasks, wait at the
    barrier, time each oracle call."""
    import types
    w, _ = make_workload(types.SimpleNamespace(**spec), n_steps)
    cache = {}
    prepared = [(task[0], _prepare_task(w, task, cache)) for task in tasks]
    start_barrier.wait()
    res = []
    for kind, prep in prepared:
        t0 = time.perf_counter()
        _run_task(w, prep)
        res.append((kind, time.perf_counter() - t0))
    out_q.put(res)


def oracle_sample(args, w, flags, timed_records):
    """The bounded oracle sample on this host's cores; the cpu_baseline dict.
    flags: [records][B]; timed_records: the record index of every timed step."""
    import multiprocessing as mp
    steps = cpu_sample_steps(sorted(set(timed_records)), flags.max(axis=1),
                             max(1, getattr(args, "cpu_steps", 4)))
    tasks = []
    n_rows_l = min(w.batch, 2)
    for j in steps:
        for b in range(n_rows_l):
            for g in range(w.hkv):
                tasks.append(("local", j, 0, b, g))
        fl = [b for b in range(w.batch) if flags[j][b]]
        for b in fl[:1]:
            for g in range(w.hkv):
                tasks.append(("full", j, 0, b, g))
        if w.recall:
            tasks.append(("recall", j, 0, 0, 0))
    cores = len(os.sched_getaffinity(0))
    C = getattr(args, "cpu_workers", 0) or cores
    C = max(1, min(C, len(tasks)))
    # heavy tasks first, dealt round robin
    order = sorted(tasks, key=lambda t: {"full": 0, "recall": 1, "local": 2}[t[0]])
    per_worker = [order[i::C] for i in range(C)]
    ctx = mp.get_context("spawn")
    blas = ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")
    old = {k: os.environ.get(k) for k in blas}
    for k in blas:
        os.environ[k] = "1"            # inherited by the spawned workers
    try:
        bar = ctx.Barrier(C + 1)
        q = ctx.Queue()
        procs = [ctx.Process(target=_oracle_worker, args=(_wl_spec(args), w.steps, ts, bar, q))
                 for ts in per_worker]
        for p in procs:
            p.start()
        bar.wait(timeout=1800)
        t0 = time.perf_counter()
        results = [q.get(timeout=1800) for _ in procs]
        wall = time.perf_counter() - t0
        for p in procs:
            p.join(timeout=60)
    finally:
        for k, v in old.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v
    by = {}
    for res in results:
        for kind, sec in res:
            by.setdefault(kind, []).append(sec)
    mean = {k: float(np.mean(v)) for k, v in by.items()}
    task_s = float(sum(sum(v) for v in by.values()))
    speedup = task_s / wall if wall > 0 else 1.0
    # tasks of an average timed step
    nf = float(np.mean([flags[j].sum() for j in timed_records]))
    per_step = {"local": float(w.batch * w.layers * w.hkv), "full": nf * w.layers * w.hkv,
                "recall": 1.0 if w.recall else 0.0}
    full_mean = mean.get("full")
    if full_mean is None:      # no flagged step sampled: a Local task scaled by length
        tmean = float(np.mean(w.t0))
        full_mean = mean.get("local", 0.0) * tmean / min(tmean, w.sink + w.window)
    cpu_s = (per_step["local"] * mean.get("local", 0.0) + per_step["full"] * full_mean +
             per_step["recall"] * mean.get("recall", 0.0))
    step_s = cpu_s / speedup
    counts = {k: len(v) for k, v in by.items()}
    text = (f"{w.name}: decode steps {list(map(int, steps))}; float64 oracle tasks {counts} "
            f"(Local: rows 0..{n_rows_l - 1}, layer 0, every KV head; Full: the first flagged "
            f"row, layer 0, every KV head; recall head + gate: the batch) on {C} worker "
            f"processes of one thread; {task_s:.2f} s of oracle calls in {wall:.2f} s wall "
            f"(inputs generated before the clock); a step = sum over its tasks of the mean "
            f"task seconds / the measured parallel speedup")
    return {"value": w.batch / step_s, "unit": UNIT, "cores": C, "kind": "oracle",
            "sample": text, "extrapolated": True, "sample_wall_s": wall,
            "sample_task_s": task_s, "parallel_speedup": speedup,
            "task_s": mean, "tasks_per_step": per_step, "sample_tasks": counts,
            "seconds_per_step": step_s}


def cpu_sample_steps(candidates, flags, n: int):
    """About n steps: a quarter flagged (at least one), the rest unflagged."""
    fl = [i for i in candidates if flags[i]]
    un = [i for i in candidates if not flags[i]]
    nf = min(len(fl), max(1, n // 4)) if fl else 0
    return sorted(fl[:nf] + un[:max(1, n - nf)])


def workload_flags(w):
    """[steps][B] uint8 flags drawn by the workload (None for the recall
    workload, whose flags come from the recall head)."""
    f = w.flags()
    return None if f is None else f.astype(np.uint8)


def oracle_recall_flags(w, steps):
    """Flags of the recall workload from the oracle's own scores (reference arm)."""
    import oracle as O
    from synth import bf16_bits_to_f32
    W1, b1, w2, b2 = w.recall_weights()
    W1 = bf16_bits_to_f32(W1).astype(np.float64)
    w2 = bf16_bits_to_f32(w2).astype(np.float64)
    flags = np.zeros((w.steps, w.batch), np.uint8)
    for j in sorted(set(steps)):
        hs = [bf16_bits_to_f32(h).astype(np.float64) for h in w.hidden_step(j)]
        s = O.recall_score(*hs, W1, b1.astype(np.float64), w2, float(b2))
        flags[j] = O.gate(s.astype(np.float32), 0.0)[0]
    return flags


# ----------------------------------------------------------------------------
# reference arm: the oracle, as it stands, on the host cores
# ----------------------------------------------------------------------------

def run_reference(args, rank, ws):
    if rank != 0:
        return
    W, K = args.warmup, args.steps
    w, external = make_workload(args, W + K)
    timed = list(range(W, W + K))
    flags = workload_flags(w)
    if flags is None:
        flags = oracle_recall_flags(w, timed)
    cpu = oracle_sample(args, w, flags, timed)
    value = cpu["value"]
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": getattr(args, "gpus", 1), "steps": K, "warmup": W,
        "ms_per_step": 1000.0 * cpu["seconds_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_block(w, args, ws),
        "cpu_baseline": cpu,
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_block(w, args, ws, copies: int = 1):
    mode = getattr(args, "mode", "oda")
    wl = getattr(args, "workload", "ctx128k")
    t0 = [int(x) for x in w.t0]
    ctx_desc = f"t={t0[0]}+step" if len(set(t0)) == 1 else f"t in [{min(t0)}, {max(t0)}]+step"
    desc = (f"{w.name}: batch {w.batch}, {w.layers} layers, {w.hq}/{w.hkv} heads, d={w.d}, "
            f"{w.dtype}, {ctx_desc}, s={w.sink}, w={w.window}, ")
    if mode == "full-only":
        desc += "dense decode: append + Full attention every layer, every step"
        rate = 1.0
    elif wl == "recall":
        desc += "recall head 6144->4096->1 scores decide the gate (theta=0)"
        rate = None
    else:
        rate = w.flag_rate
        per = "step" if w.flag_per == "step" else "row"
        desc += (f"Full calls Bernoulli({w.flag_rate:g}) per {per}, "
                 f"recall head 6144->4096->1 every step")
    local_mb = (w.layers * sum(min(t, w.sink + w.window) for t in t0)
                * KV_BYTES_PER_TOKEN_LAYER / 1e6)
    cache_gb = w.layers * sum(t0) * KV_BYTES_PER_TOKEN_LAYER / 1e9
    if copies > 1:
        l2 = (f"the steps rotate through {copies} independently allocated copies of the KV "
              f"state and recall weights (Local reads {local_mb:.0f} MB per step)")
    else:
        l2 = ("no flush needed: per-step reads (ring %d MB, Full %d GB) exceed the 126 MB L2"
              % (round(local_mb), round(cache_gb)))
    return {"workload": desc, "mode": mode, "name": w.name,
            "batch_per_gpu": int(w.batch), "global_batch": int(w.batch * ws),
            "context": t0[0] if len(set(t0)) == 1 else [min(t0), max(t0)],
            "layers": int(w.layers), "hq": w.hq, "hkv": w.hkv,
            "head_dim": w.d, "sink": w.sink, "window": w.window,
            "full_call_rate": rate,
            "parallelism": f"replicas x{ws}", "launch": getattr(args, "launch", "graph"),
            "copies": copies, "l2": l2}


# ----------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------

def run_recall_loss(args, rank, ws, local):
    """The recall head's training objective (oda_recall_loss) over
    --positions seeded synthetic positions: 12 bytes read per position."""
    import torch
    from gated_local_full_b200 import oda
    torch.cuda.set_device(local)
    n, K, W = args.positions, args.steps, args.warmup
    gen = torch.Generator(device="cuda").manual_seed(7 + rank)
    q = torch.randn(n, device="cuda", generator=gen) * 2.0
    lf = torch.randn(n, device="cuda", generator=gen) * 1.5 - 2.0
    ll = lf - (torch.randn(n, device="cuda", generator=gen) + 0.1)
    cfg = oda.make_config(layers=1, max_batch=1, hq=2, hkv=1, head_dim=64, sink=4, window=16,
                          dtype="f32", max_blocks_per_seq=4, num_blocks=4)
    ctx = oda.OdaContext(cfg)
    loss = torch.zeros(1, device="cuda")
    nf = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()
    for _ in range(W):
        ctx.recall_loss(q, lf, ll, 0.0, loss, nf)
    torch.cuda.synchronize()
    barrier(ws)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(K):
        ctx.recall_loss(q, lf, ll, 0.0, loss, nf)
    b.record(stream)
    torch.cuda.synchronize()
    t = max_over_ranks(a.elapsed_time(b) / 1000.0, ws)
    err = ctx.get_device_error()
    ctx.close()
    if rank == 0:
        hbm, kind = peaks()
        gbs = 12.0 * n * K * ws / t / 1e9
        print(json.dumps({
            "metric": "recall-head training objective GB/s (12 B per position)", "value": gbs,
            "unit": "GB/s", "n_gpus": ws, "steps": K, "warmup": W,
            "ms_per_step": 1000.0 * t / K, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32 (f64 sum)", "data": "synthetic (seeded)",
            "config": {"workload": f"oda_recall_loss over {n} positions", "positions": n,
                       "l2": "inputs of %d MB exceed the 126 MB L2" % (12 * n // 10**6)},
            "roofline": {"bound": "hbm", "achieved": gbs / ws, "peak": hbm, "unit": "GB/s",
                         "frac": gbs / ws / hbm, "frac_of_nominal": gbs / ws / NOMINAL_HBM_GBS,
                         "traffic": None, "peak_kind": kind},
            "device_error": err}), flush=True)


def device_flags(ctx, st, recs, r, n_rec, w, torch):
    """Flags of every record from the recall head's own scores, computed on the
    device by the same kernels as in the step (untimed)."""
    scores = torch.empty(w.batch, dtype=torch.float32, device="cuda")
    fl = torch.empty(w.batch, dtype=torch.uint8, device="cuda")
    idx = torch.empty(w.batch, dtype=torch.int32, device="cuda")
    cnt = torch.empty(1, dtype=torch.int32, device="cuda")
    out = np.zeros((n_rec, w.batch), np.uint8)
    for j in range(n_rec):
        ctx.recall_score(st.record_view(recs, j, "h_prev"), st.record_view(recs, j, "emb"),
                         st.record_view(recs, j, "h_local"), r["H"], r["W1"], r["b1"], r["w2"],
                         r["b2"], r["hidden"], scores, w.batch)
        ctx.gate(scores, 0.0, w.batch, fl, idx, cnt)
        out[j] = fl.cpu().numpy()
    return out


def run_oda(args, rank, ws, local):
    import torch

    from gated_local_full_b200 import oda
    from gated_local_full_b200.runtime import DecodeStep
    from synth.device import DeviceWorkload

    torch.cuda.set_device(local)
    K, W = args.steps, args.warmup
    S = W + K
    dense = args.mode == "full-only"
    R = args.copies or (1 if args.workload == "ctx128k" else 3)
    n_rec = (S + R - 1) // R                     # step i runs copy i % R on record i // R
    w, external = make_workload(args, n_rec)
    bt, nb = w.paging()
    cfg = oda.make_config(layers=w.layers, max_batch=w.batch, hq=w.hq, hkv=w.hkv, head_dim=w.d,
                          sink=w.sink, window=w.window, dtype=w.dtype,
                          max_blocks_per_seq=bt.shape[1], num_blocks=nb)
    ctx = oda.OdaContext(cfg)
    copies = []
    for c in range(R):
        dw = DeviceWorkload(w, ctx.layout, w.batch)
        pre = torch.from_numpy((w.t0 - 1).astype(np.int32)).cuda()
        ctx.ring_init(0, w.layers, pre, dw.block_table, dw.cache, dw.ring, w.batch)
        st = DecodeStep(ctx, w.batch, dw.cache, dw.ring, dw.block_table, recall=dw.recall,
                        external_scores=external, graph=(args.launch == "graph"))
        copies.append((dw, st))
    dw0, st0 = copies[0]
    recs = st0.new_records(n_rec)
    r = dw0.recall
    for j in range(n_rec):
        st0.pack(recs, j, q=dw0.q[j], k_new=dw0.k_new[j], v_new=dw0.v_new[j],
                 seq_lens=dw0.seq_lens[j], gate_scores=dw0.scores[j] if external else None,
                 h_prev=r["h_prev"][j], emb=r["emb"][j], h_local=r["h_local"][j])
    for dw, _ in copies:
        del dw.q, dw.k_new, dw.v_new
    torch.cuda.synchronize()
    assert ctx.get_device_error() == 0
    stream = torch.cuda.current_stream()
    flags = workload_flags(w) if external else device_flags(ctx, st0, recs, r, n_rec, w, torch)

    def step_of(i):
        return copies[i % R], i // R

    if dense:
        # dense decode on the same kernels: commit the token, then Full
        # attention for every row in every layer, captured once as a graph
        cnt_all = torch.full((1,), w.batch, dtype=torch.int32, device="cuda")
        idx_all = torch.arange(w.batch, dtype=torch.int32, device="cuda")
        dgraphs = []
        for dw, st in copies:
            def dense_step(dw=dw, st=st):
                ctx.append_kv(0, w.layers, st.k_new, st.v_new, st.seq_lens, dw.block_table,
                              dw.cache, dw.ring, w.batch)
                for l in range(w.layers):
                    ctx.full_attn_gated(l, st.q[l], st.seq_lens, dw.block_table, dw.cache,
                                        idx_all, cnt_all, st.out[l], None, w.batch,
                                        inputs_ready=l > 0)
            side = torch.cuda.Stream()
            side.wait_stream(stream)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=side):
                dense_step()
            stream.wait_stream(side)
            dgraphs.append(g)

        def run_step(i):
            (dw, st), j = step_of(i)
            st.feed_record(recs, j)
            dgraphs[i % R].replay()
    else:
        def run_step(i):
            (dw, st), j = step_of(i)
            st.feed_record(recs, j)
            st.run()

    sampler = ClockSampler(gpu_id(local))
    for i in range(W):
        run_step(i)
    torch.cuda.synchronize()
    barrier(ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    h0 = time.time()
    e0.record(stream)
    for i in range(W, S):
        run_step(i)
    e1.record(stream)
    torch.cuda.synchronize()
    h1 = time.time()
    barrier(ws)
    elapsed = e0.elapsed_time(e1) / 1000.0
    clocks = sampler.summary(h0, h1)
    sampler.stop()              # nvidia-smi no longer competes with the legs below
    err = ctx.get_device_error()
    t_max = max_over_ranks(elapsed, ws)
    timed = list(range(W, S))
    recs_timed = [i // R for i in timed]
    n_flag_rows = int(sum(flags[j].sum() for j in recs_timed))
    n_flag_steps = int(sum(1 for j in recs_timed if flags[j].any()))
    if dense:
        kv_bytes = sum(w.layers * sum(int(w.t0[b]) + j + 2 for b in range(w.batch))
                       * KV_BYTES_PER_TOKEN_LAYER for j in recs_timed)
        launches = K * (w.layers + 1)
    else:
        kv_bytes = sum(batch_step_bytes(w, j, flags[j]) for j in recs_timed)
        # the recall head's prefix kernel (its first layer over h_{t-1} and
        # E(x_t), in steps of enough layers; every workload here has a head
        # shape the step splits), append, Local x L, the rest of the recall
        # head (its last CTA gates), then Full x L: behind the IF node only
        # steps with a flagged row launch them; plain launches issue the Full
        # launches every step
        pre = 1 if w.layers >= oda.RECALL_SPLIT_MIN_LAYERS else 0
        if args.launch == "graph":
            launches = K * (w.layers + 2 + pre) + n_flag_steps * w.layers
        else:
            launches = K * (2 * w.layers + 2 + pre)

    # ---- per-kernel launch times, as in a step: the L layers' launches back
    # to back (flag set from the second on), for up to 16 timed steps, each on
    # its own copy, captured in one CUDA graph and replayed between two CUDA
    # events on this stream
    outb = torch.empty_like(st0.out[0])
    ids = {}
    for j in sorted(set(recs_timed)):
        rows = [b for b in range(w.batch) if flags[j][b]]
        if rows:
            idx = torch.full((w.batch,), -1, dtype=torch.int32)
            idx[:len(rows)] = torch.tensor(rows, dtype=torch.int32)
            ids[j] = (idx.cuda(), torch.tensor([len(rows)], dtype=torch.int32, device="cuda"))
    fl_steps = [i for i in timed if (i // R) in ids][:16]
    loc_steps = timed[:16]

    def run_full():
        for i in fl_steps:
            (dw, st), j = step_of(i)
            q = st.record_view(recs, j, "q")
            sl = st.record_view(recs, j, "seq_lens")
            idx, cnt = ids[j]
            for l in range(w.layers):
                ctx.full_attn_gated(l, q[l], sl, dw.block_table, dw.cache, idx, cnt, outb, None,
                                    w.batch, inputs_ready=l > 0)

    def run_local():
        for i in loc_steps:
            (dw, st), j = step_of(i)
            q = st.record_view(recs, j, "q")
            sl = st.record_view(recs, j, "seq_lens")
            for l in range(w.layers):
                ctx.local_attn(l, q[l], sl, dw.ring, outb, None, w.batch, inputs_ready=l > 0)

    hbm, hbm_kind = peaks()
    kernels = {}
    local_s = replay_seconds(torch, run_local, stream)
    n_local = len(loc_steps) * w.layers
    local_bytes = sum(sum(min(int(w.t0[b]) + i // R, w.sink + w.window) for b in range(w.batch))
                      for i in loc_steps) * w.layers * KV_BYTES_PER_TOKEN_LAYER
    kernels["local"] = {"kernel": "attn_kernel<bf16,128,2,RING=true> (Local attention)",
                        "mean_launch_us": local_s / n_local * 1e6,
                        "bytes_per_launch": local_bytes / n_local,
                        "achieved_gbs": local_bytes / local_s / 1e9,
                        "launches_timed": n_local}
    if fl_steps:
        full_s = replay_seconds(torch, run_full, stream)
        n_full = len(fl_steps) * w.layers
        full_bytes = sum(sum(int(w.t0[b]) + i // R for b in range(w.batch) if flags[i // R][b])
                         for i in fl_steps) * w.layers * KV_BYTES_PER_TOKEN_LAYER
        kernels["full"] = {"kernel": "attn_kernel<bf16,128,2,RING=false> (Full attention)",
                           "mean_launch_us": full_s / n_full * 1e6,
                           "bytes_per_launch": full_bytes / n_full,
                           "achieved_gbs": full_bytes / full_s / 1e9,
                           "launches_timed": n_full}
    if r is not None:
        # the recall head alone (oda_recall_score over the step's batch, the
        # whole 6144-column W1 in one call), back to back, each call on one of
        # at least four weight copies (4 x 50 MB > the 126 MB L2), so that every
        # call streams its W1 from HBM
        w1s = [dw.recall["W1"] for dw, _ in copies]
        while len(w1s) < 4:
            w1s.append(w1s[0].clone())
        sc_out = torch.empty(w.batch, dtype=torch.float32, device="cuda")
        n_rc = 16

        def run_recall():
            for i in range(n_rc):
                ctx.recall_score(r["h_prev"][0], r["emb"][0], r["h_local"][0], r["H"],
                                 w1s[i % len(w1s)], r["b1"], r["w2"], r["b2"], r["hidden"],
                                 sc_out, w.batch)

        rc_s = replay_seconds(torch, run_recall, stream)
        # W1, the three states, b1 and w2 (float32), the scores
        rc_bytes = n_rc * (w1s[0].numel() * 2 + 3 * w.batch * r["H"] * 2
                           + 2 * r["hidden"] * 4 + w.batch * 4)
        kernels["recall"] = {"kernel": "recall_cluster_kernel (tcgen05 first layer, GELU, w2, "
                                       "fixed-order sum; one call per step's batch)",
                             "mean_launch_us": rc_s / n_rc * 1e6,
                             "bytes_per_launch": rc_bytes / n_rc,
                             "achieved_gbs": rc_bytes / rc_s / 1e9,
                             "launches_timed": n_rc}
        del w1s
    for k in kernels.values():
        k["frac_of_peak"] = k["achieved_gbs"] / hbm
        k["frac_of_nominal"] = k["achieved_gbs"] / NOMINAL_HBM_GBS
    # the dominant kernel: the larger share of an average step's time
    share_local = kernels["local"]["mean_launch_us"] * w.layers
    share_full = (kernels["full"]["mean_launch_us"] * w.layers * n_flag_steps / K
                  if "full" in kernels else 0.0)
    dom = "full" if share_full >= share_local else "local"
    traffic = None
    if dom == "full" and args.workload == "ctx128k":
        traffic, _ = recorded_traffic()
    dk = kernels[dom]
    roofline = {"bound": "hbm", "achieved": dk["achieved_gbs"], "peak": hbm, "unit": "GB/s",
                "frac": dk["achieved_gbs"] / hbm,
                "frac_of_nominal": dk["achieved_gbs"] / NOMINAL_HBM_GBS,
                "traffic": traffic, "kernel": dk["kernel"], "peak_kind": hbm_kind,
                "launches_timed": dk["launches_timed"],
                "timing": "CUDA events on the launching stream around a graph replay of L "
                          "back-to-back launches per step",
                "mean_launch_us": dk["mean_launch_us"]}

    # ---- end to end: host records in, result out, every step
    e2e = None
    if not args.no_e2e:
        # the same K steps as the device-timed run (same Full calls), fed from
        # pinned host memory one step at a time
        hrec = st0.new_records(n_rec, pin=True)
        hrec.copy_(recs.cpu())
        res = torch.empty((w.batch, w.hq, w.d), dtype=torch.bfloat16).pin_memory()
        cnt = torch.empty(1, dtype=torch.int32).pin_memory()
        hres = st0.new_result()
        one_call = st0.graph is not None and not dense
        # replays steps W.. on caches that already hold later positions: the
        # same work per step; outputs are not checked here
        torch.cuda.synchronize()
        barrier(ws)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for i in timed:
            (dw, st), j = step_of(i)
            if one_call:
                # record in, step graph, last layer's output and count out, wait
                st.run_io(hrec[j], hres)
            else:
                st.feed_record(hrec, j)
                if dense:
                    dgraphs[i % R].replay()
                else:
                    st.run()
                res.copy_(st.out[w.layers - 1], non_blocking=True)
                cnt.copy_(st.count, non_blocking=True)
                stream.synchronize()
        b.record(stream)
        torch.cuda.synchronize()
        e2e_t = max_over_ranks(a.elapsed_time(b) / 1000.0, ws)
        e2e = {"value": job_throughput(K * w.batch, ws, e2e_t), "unit": UNIT,
               "h2d_bytes_per_step": int(st0.record_bytes),
               "d2h_bytes_per_step": int(res.numel() * res.element_size() + 4),
               "steps": K, "read_back": "the last layer's output and the flagged-row count"}

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline and not dense:
        cpu = oracle_sample(args, w, flags, recs_timed)

    if rank == 0:
        value = job_throughput(K * w.batch, ws, t_max)
        kv_gbs = kv_bytes / elapsed / 1e9
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": K,
            "warmup": W, "ms_per_step": 1000.0 * t_max / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded counter-based generator; no datasets or weights)",
            "config": config_block(w, args, ws, R),
            "kv_gbs": kv_gbs, "kv_frac_of_hbm": kv_gbs / hbm,
            "kv_frac_of_nominal": kv_gbs / NOMINAL_HBM_GBS,
            "kv_bytes_per_step": kv_bytes / K,
            "full_call_rate_realised": 1.0 if dense else n_flag_rows / (K * w.batch),
            "full_steps_realised": n_flag_steps,
            "recall_weight_bytes_per_step": int(w.recall_hidden * 3 * w.hidden * 2),
            "roofline": roofline, "kernels": kernels,
            "local_attn_mean_launch_us": kernels["local"]["mean_launch_us"],
            "cpu_baseline": cpu, "e2e": e2e, "clocks": clocks, "gpu_launches": launches,
            "device_error": err,
        }
        print(json.dumps(line), flush=True)
    for _, st in copies:
        st.close()
    ctx.close()
    return line if rank == 0 else None


def main():
    args = parse()
    rank, ws, local = dist_init()
    try:
        if args.impl == "reference":
            run_reference(args, rank, ws)
        elif args.mode == "recall-loss":
            run_recall_loss(args, rank, ws, local)
        else:
            run_oda(args, rank, ws, local)
    finally:
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()

#!/usr/bin/env python
"""Benchmark of the gated local/full decode-attention step on B200.

Workload (default): batch 1, 28 layers of GQA attention (16 query / 8 KV
heads, head_dim 128, bf16), context t = 131072 at the first step and growing
by one per step, s = 4 sinks + w = 2048 window for Local, Full recomputation
on a Bernoulli(0.125) draw per step, plus the 6144 -> 4096 -> 1 recall head
on synthetic states every step. One "step" = one decode step of the whole
path (append, Local x 28, recall head, gate, Full x 28 when flagged) replayed
from a captured CUDA graph; inputs are resident in HBM and fed with one
device copy per step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl oda|reference]

Prints one JSON line (rank 0). Under torchrun every rank runs an independent
replica (the path has no cross-request exchange) and the time is the max
over ranks.
"""

from __future__ import annotations

import argparse
import hashlib
import re
import json
import os
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


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1024)
    ap.add_argument("--warmup", type=int, default=8)
    ap.add_argument("--impl", choices=["oda", "reference"], default="oda")
    ap.add_argument("--layers", type=int, default=28)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--cpu-steps", type=int, default=8)
    ap.add_argument("--launch", choices=["graph", "plain"], default="graph",
                    help="graph: captured step with the IF node; plain: the same kernels "
                         "launched one by one (visible to ncu)")
    ap.add_argument("--context", type=int, default=131072,
                    help="context length t at the first step (the headline is 131072)")
    ap.add_argument("--rate", type=float, default=0.125,
                    help="Full-call rate: Bernoulli per step (the headline is 0.125)")
    ap.add_argument("--mode", choices=["oda", "full-only", "recall-loss"], default="oda",
                    help="full-only: every step appends and runs Full attention in every "
                         "layer, no Local, recall head or gate (dense decode, for the "
                         "speedup and the short-context crossover); recall-loss: the recall "
                         "head's training objective over --positions positions")
    ap.add_argument("--positions", type=int, default=1 << 24,
                    help="positions per recall-loss call (--mode recall-loss)")
    return ap.parse_args()


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
# algorithmic bytes (KV actually read + KV written)
# ----------------------------------------------------------------------------

def step_kv_bytes(t: int, flagged: bool, layers: int, s=4, w=2048) -> int:
    local = min(t, s + w)
    full = t if flagged else 0
    return layers * (local + full + 2) * KV_BYTES_PER_TOKEN_LAYER


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
# ----------------------------------------------------------------------------

class OracleSample:
    """Oracle inputs for the sample: Local on layer 0 (all 8 KV heads), Full on
    layer 0 KV head 0, the recall head for batch row 0. Generating them is not
    timed; the oracle calls are."""

    def __init__(self, w, t_max: int):
        import oracle as O  # noqa: F401  (test infrastructure; baseline leg only)
        from synth.gen import table_values
        self.w = w
        d, tab = w.d, w.kv_table()
        lo = max(1, int(w.t0[0]) - w.window)
        self.Kl, self.Vl = [], []
        for g in range(w.hkv):
            K = np.zeros((1, t_max, d))
            V = np.zeros((1, t_max, d))
            for kv, dst in ((0, K), (1, V)):
                key = w.kv_key(0, 0, g, kv)
                dst[0, :w.sink] = w.to_f64(table_values(key, 0, w.sink * d, tab).reshape(-1, d))
                dst[0, lo - 1:t_max] = w.to_f64(
                    table_values(key, (lo - 1) * d, (t_max - lo + 1) * d, tab).reshape(-1, d))
            self.Kl.append(K)
            self.Vl.append(V)
        self.Kf = np.zeros((1, t_max, d))
        self.Vf = np.zeros((1, t_max, d))
        self.Kf[0] = w.to_f64(table_values(w.kv_key(0, 0, 0, 0), 0, t_max * d, tab).reshape(-1, d))
        self.Vf[0] = w.to_f64(table_values(w.kv_key(0, 0, 0, 1), 0, t_max * d, tab).reshape(-1, d))
        W1, b1, w2, b2 = w.recall_weights()
        from synth import bf16_bits_to_f32
        self.W1 = bf16_bits_to_f32(W1).astype(np.float64)
        self.b1 = b1.astype(np.float64)
        self.w2 = bf16_bits_to_f32(w2).astype(np.float64)
        self.b2 = float(b2)

    def step_seconds(self, step: int, flagged: bool) -> float:
        """Extrapolated seconds for one full decode step (28 layers)."""
        import oracle as O
        from synth import bf16_bits_to_f32
        w = self.w
        t = int(w.t0[0]) + step
        q = w.to_f64(w.q_step_layer(step, 0)[0])             # [hq][d] of row 0, layer 0
        hs = [bf16_bits_to_f32(h).astype(np.float64) for h in w.hidden_step(step)]
        G = w.group
        t0 = time.perf_counter()
        for g in range(w.hkv):
            O.local_attention(q[g * G:(g + 1) * G], self.Kl[g], self.Vl[g], t, w.sink, w.window)
        t_local = time.perf_counter() - t0
        t0 = time.perf_counter()
        score = O.recall_score(*hs, self.W1, self.b1, self.w2, self.b2)
        O.gate(score.astype(np.float32), 0.0)
        t_recall = time.perf_counter() - t0
        t_full = 0.0
        if flagged:
            t0 = time.perf_counter()
            O.full_attention(q[0:G], self.Kf, self.Vf, t)
            t_full = time.perf_counter() - t0
        return w.layers * t_local + t_recall + w.layers * w.hkv * t_full


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return 1


def cpu_sample_steps(candidates, flags, n: int):
    """About n steps: a quarter flagged (at least one), the rest unflagged."""
    fl = [i for i in candidates if flags[i]]
    un = [i for i in candidates if not flags[i]]
    nf = min(len(fl), max(1, n // 4)) if fl else 0
    return sorted(fl[:nf] + un[:max(1, n - nf)])


def weighted_step_seconds(secs: dict, flags, rate: float) -> float:
    """Mean seconds per step at the realised Full-call rate."""
    un = [v for i, v in secs.items() if not flags[i]]
    fl = [v for i, v in secs.items() if flags[i]]
    t_un = float(np.mean(un)) if un else 0.0
    t_fl = float(np.mean(fl)) if fl else t_un
    return (1.0 - rate) * t_un + rate * t_fl


def sample_text(steps, flags, rate):
    return (f"decode steps {list(map(int, steps))} ({int(sum(flags))} flagged) of the 128K "
            f"workload, batch row 0: Local on layer 0 for all 8 KV heads (x28 layers), Full on "
            f"layer 0 KV head 0 (x28 layers x 8 heads), recall head and gate once per step; "
            f"float64 oracle; unflagged and flagged step means weighted by the realised "
            f"Full-call rate {rate:.4f}")


# ----------------------------------------------------------------------------
# reference arm: the oracle, as it stands, on the host cores
# ----------------------------------------------------------------------------

def run_reference(args, rank, ws):
    if rank != 0:
        return
    import synth
    w = synth.ctx128k(steps=args.warmup + args.steps, layers=args.layers, context=args.context,
                      rate=args.rate)
    w.recall = True
    flags = w.flags()[:, 0]
    t_max = int(w.t0[0]) + w.steps
    sample = OracleSample(w, t_max)
    for i in range(min(args.warmup, 1)):                 # warm caches and BLAS threads
        sample.step_seconds(i, bool(flags[i]))
    steps = list(range(args.warmup, args.warmup + args.steps))
    rate = float(flags[steps].mean())
    # every timed step is represented by a bounded sample of at most 16 of
    # them (flagged and unflagged in proportion, at least one flagged when
    # any is), so the run ends within minutes whatever K is
    timed_steps = cpu_sample_steps(steps, flags, min(len(steps), 16))
    secs = {i: sample.step_seconds(i, bool(flags[i])) for i in timed_steps}
    per_step = weighted_step_seconds(secs, flags, rate)
    value = w.batch / per_step
    cores = blas_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_block(w, args, ws),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample_text(timed_steps, flags[timed_steps], rate)},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_block(w, args, ws):
    mode = getattr(args, "mode", "oda")
    desc = (f"{w.name}: batch 1, {w.layers} layers, 16/8 heads, d=128, bf16, "
            f"t={int(w.t0[0])}+step, s=4, w=2048, ")
    desc += ("Full calls Bernoulli(%g) per step, recall head 6144->4096->1" % w.flag_rate
             if mode == "oda" else "dense decode: append + Full attention every layer, every step")
    return {"workload": desc, "mode": mode,
            "batch_per_gpu": int(w.batch), "global_batch": int(w.batch * ws),
            "context": int(w.t0[0]), "layers": int(w.layers), "hq": w.hq, "hkv": w.hkv,
            "head_dim": w.d, "sink": w.sink, "window": w.window,
            "full_call_rate": w.flag_rate if mode == "oda" else 1.0,
            "parallelism": f"replicas x{ws}", "launch": getattr(args, "launch", "graph"),
            "l2": "no flush needed: per-step reads (ring %d MB, Full %d GB) exceed the 126 MB L2"
                  % (round(w.layers * min(int(w.t0[0]), w.sink + w.window) * KV_BYTES_PER_TOKEN_LAYER / 1e6),
                     round(w.layers * int(w.t0[0]) * KV_BYTES_PER_TOKEN_LAYER / 1e9))}


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
                         "frac": gbs / ws / hbm, "traffic": None, "peak_kind": kind},
            "device_error": err}), flush=True)


def run_oda(args, rank, ws, local):
    import torch

    import synth
    from gated_local_full_b200 import oda
    from gated_local_full_b200.runtime import DecodeStep
    from synth.device import DeviceWorkload

    torch.cuda.set_device(local)
    K, W = args.steps, args.warmup
    w = synth.ctx128k(steps=W + K, layers=args.layers, context=args.context, rate=args.rate)
    w.recall = True                                   # recall head runs every step
    flags = w.flags()[:, 0]
    bt, nb = w.paging()
    cfg = oda.make_config(layers=w.layers, max_batch=w.batch, hq=w.hq, hkv=w.hkv, head_dim=w.d,
                          sink=w.sink, window=w.window, dtype=w.dtype,
                          max_blocks_per_seq=bt.shape[1], num_blocks=nb)
    ctx = oda.OdaContext(cfg)
    dw = DeviceWorkload(w, ctx.layout, w.batch)
    pre = torch.from_numpy((w.t0 - 1).astype(np.int32)).cuda()
    ctx.ring_init(0, w.layers, pre, dw.block_table, dw.cache, dw.ring, w.batch)
    st = DecodeStep(ctx, w.batch, dw.cache, dw.ring, dw.block_table, recall=dw.recall,
                    external_scores=True, graph=(args.launch == "graph"))
    S = W + K
    recs = st.new_records(S)
    r = dw.recall
    for i in range(S):
        st.pack(recs, i, q=dw.q[i], k_new=dw.k_new[i], v_new=dw.v_new[i],
                seq_lens=dw.seq_lens[i], gate_scores=dw.scores[i], h_prev=r["h_prev"][i],
                emb=r["emb"][i], h_local=r["h_local"][i])
    del dw.q, dw.k_new, dw.v_new
    torch.cuda.synchronize()
    assert ctx.get_device_error() == 0
    stream = torch.cuda.current_stream()

    dense = args.mode == "full-only"
    if dense:
        # dense decode on the same kernels: commit the token, then Full
        # attention for every row in every layer, captured once as a graph
        cnt_all = torch.full((1,), w.batch, dtype=torch.int32, device="cuda")
        idx_all = torch.arange(w.batch, dtype=torch.int32, device="cuda")

        def dense_step():
            ctx.append_kv(0, w.layers, st.k_new, st.v_new, st.seq_lens, dw.block_table, dw.cache,
                          dw.ring, w.batch)
            for l in range(w.layers):
                ctx.full_attn_gated(l, st.q[l], st.seq_lens, dw.block_table, dw.cache, idx_all,
                                    cnt_all, st.out[l], None, w.batch, inputs_ready=l > 0)

        side = torch.cuda.Stream()
        side.wait_stream(stream)
        dgraph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(dgraph, stream=side):
            dense_step()
        stream.wait_stream(side)
        run_step = dgraph.replay
    else:
        run_step = st.run

    sampler = ClockSampler(gpu_id(local))
    for i in range(W):
        st.feed_record(recs, i)
        run_step()
    torch.cuda.synchronize()
    barrier(ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    h0 = time.time()
    e0.record(stream)
    for i in range(W, W + K):
        st.feed_record(recs, i)
        run_step()
    e1.record(stream)
    torch.cuda.synchronize()
    h1 = time.time()
    barrier(ws)
    elapsed = e0.elapsed_time(e1) / 1000.0
    clocks = sampler.summary(h0, h1)
    sampler.stop()              # nvidia-smi no longer competes with the legs below
    err = ctx.get_device_error()
    t_max = max_over_ranks(elapsed, ws)
    timed = list(range(W, W + K))
    n_flag = int(flags[timed].sum())
    if dense:
        kv_bytes = sum(w.layers * (int(w.t0[0]) + i + 2) * KV_BYTES_PER_TOKEN_LAYER
                       for i in timed)
        launches = K * (w.layers + 1)
    else:
        kv_bytes = sum(step_kv_bytes(int(w.t0[0]) + i, bool(flags[i]), w.layers) for i in timed)
        # append, Local x L, recall, gate, then Full x L: behind the IF node
        # only flagged steps launch them; plain launches issue them every step
        launches = K * (w.layers + 4) + (n_flag if args.launch == "graph" else K) * w.layers

    # ---- dominant kernel: Full attention. As in a flagged step, the L layers'
    # launches run back to back: the runs of up to 16 flagged steps are
    # captured in one CUDA graph (no host launch cost between kernels), which
    # is replayed between two CUDA events on this stream; the average launch
    # duration is the replay's time over its launches.
    cnt1 = torch.ones(1, dtype=torch.int32, device="cuda")
    idx0 = torch.zeros(w.batch, dtype=torch.int32, device="cuda")
    outb = torch.empty_like(st.out[0])
    fl_steps = [i for i in timed if flags[i]][:16] or [timed[0]]

    def run_full():
        for i in fl_steps:
            q = st.record_view(recs, i, "q")
            sl = st.record_view(recs, i, "seq_lens")
            for l in range(w.layers):
                ctx.full_attn_gated(l, q[l], sl, dw.block_table, dw.cache, idx0, cnt1, outb,
                                    None, w.batch, inputs_ready=l > 0)

    def run_local():
        for i in timed[:16]:
            q = st.record_view(recs, i, "q")
            sl = st.record_view(recs, i, "seq_lens")
            for l in range(w.layers):
                ctx.local_attn(l, q[l], sl, dw.ring, outb, None, w.batch, inputs_ready=l > 0)

    full_s, n_full = replay_seconds(torch, run_full, stream), len(fl_steps) * w.layers
    local_s, n_local = replay_seconds(torch, run_local, stream), min(K, 16) * w.layers
    full_bytes = sum((int(w.t0[0]) + i) * KV_BYTES_PER_TOKEN_LAYER for i in fl_steps) * w.layers
    full_gbs = float(full_bytes / full_s / 1e9)
    local_us = float(local_s / n_local * 1e6)
    hbm, hbm_kind = peaks()
    traffic, _ = recorded_traffic()

    # ---- end to end: host records in, result out, every step
    e2e = None
    if not args.no_e2e:
        # the same K steps as the device-timed run (same Full calls), fed from
        # pinned host memory one step at a time
        n_e2e = K
        hrec = st.new_records(n_e2e, pin=True)
        hrec.copy_(recs[W:W + n_e2e].cpu())
        res = torch.empty((w.batch, w.hq, w.d), dtype=torch.bfloat16).pin_memory()
        cnt = torch.empty(1, dtype=torch.int32).pin_memory()
        hres = st.new_result()
        one_call = st.graph is not None and not dense
        # replays steps W.. on a cache that already holds later positions: the
        # same work per step; outputs are not checked here
        torch.cuda.synchronize()
        barrier(ws)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for j in range(n_e2e):
            if one_call:
                # record in, step graph, last layer's output and count out, wait
                st.run_io(hrec[j], hres)
            else:
                st.feed_record(hrec, j)
                run_step()
                res.copy_(st.out[w.layers - 1], non_blocking=True)
                cnt.copy_(st.count, non_blocking=True)
                stream.synchronize()
        b.record(stream)
        torch.cuda.synchronize()
        e2e_t = max_over_ranks(a.elapsed_time(b) / 1000.0, ws)
        e2e = {"value": job_throughput(n_e2e * w.batch, ws, e2e_t), "unit": UNIT,
               "h2d_bytes_per_step": int(st.record_bytes),
               "d2h_bytes_per_step": int(res.numel() * res.element_size() + 4),
               "steps": n_e2e}

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline and not dense:
        steps = cpu_sample_steps(timed, flags, args.cpu_steps)
        sample = OracleSample(w, int(w.t0[0]) + S)
        secs = {i: sample.step_seconds(i, bool(flags[i])) for i in steps}
        per_step = weighted_step_seconds(secs, flags, n_flag / K)
        cpu = {"value": w.batch / per_step, "unit": UNIT, "cores": blas_threads(),
               "kind": "oracle", "sample": sample_text(steps, flags[steps], n_flag / K)}

    if rank == 0:
        value = job_throughput(K * w.batch, ws, t_max)
        kv_gbs = kv_bytes / elapsed / 1e9
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": K,
            "warmup": W, "ms_per_step": 1000.0 * t_max / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded counter-based generator; no datasets or weights)",
            "config": config_block(w, args, ws),
            "kv_gbs": kv_gbs, "kv_frac_of_hbm": kv_gbs / hbm,
            "kv_bytes_per_step": kv_bytes / K,
            "full_call_rate_realised": 1.0 if dense else n_flag / K,
            "recall_weight_bytes_per_step": int(w.recall_hidden * 3 * w.hidden * 2),
            "roofline": {"bound": "hbm", "achieved": full_gbs, "peak": hbm, "unit": "GB/s",
                         "frac": full_gbs / hbm, "traffic": traffic,
                         "kernel": "attn_kernel<bf16,128,2,RING=false> (Full attention)",
                         "peak_kind": hbm_kind,
                         "launches_timed": n_full,
                         "timing": "CUDA events on the launching stream around a graph "
                                   "replay of L back-to-back launches per flagged step",
                         "mean_launch_us": float(full_s / n_full * 1e6)},
            "local_attn_mean_launch_us": local_us,
            "cpu_baseline": cpu, "e2e": e2e, "clocks": clocks, "gpu_launches": launches,
            "device_error": err,
        }
        print(json.dumps(line), flush=True)
    st.close()
    ctx.close()


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

"""The multi-GPU plumbing of bench.py (replicas only) on CPU with gloo,
world size 2: rendezvous, barrier, max-over-ranks timing, whole-job
throughput, and the reference arm running on rank 0 only."""

import os
import subprocess
import sys
import textwrap

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = textwrap.dedent("""
    import io, contextlib, json, os, sys
    sys.path.insert(0, {root!r})
    import bench
    rank, ws, local = bench.dist_init("gloo")
    assert ws == 2 and rank == int(os.environ["RANK"])
    bench.barrier(ws)
    mine = 1.5 if rank == 0 else 4.0          # per-rank seconds
    t = bench.max_over_ranks(mine, ws)
    assert t == 4.0, t
    v = bench.job_throughput(1024, ws, t)
    assert abs(v - 1024 * 2 / 4.0) < 1e-9
    # the reference arm: rank 0 alone runs and prints, rank 1 returns at once
    class A: steps = 2; warmup = 1; gpus = 2; layers = 2
    buf = io.StringIO()
    if rank == 1:
        with contextlib.redirect_stdout(buf):
            bench.run_reference(A, rank, ws)
        assert buf.getvalue() == ""
    bench.barrier(ws)
    import torch.distributed as dist
    dist.destroy_process_group()
    print("rank", rank, "ok")
""")


def test_two_rank_gloo_plumbing(tmp_path):
    script = tmp_path / "child.py"
    script.write_text(CHILD.format(root=ROOT))
    env = dict(os.environ, MASTER_ADDR="127.0.0.1", MASTER_PORT="29533", WORLD_SIZE="2",
               CUDA_VISIBLE_DEVICES="")
    procs = []
    for r in range(2):
        e = dict(env, RANK=str(r), LOCAL_RANK=str(r))
        procs.append(subprocess.Popen([sys.executable, str(script)], env=e,
                                      stdout=subprocess.PIPE, stderr=subprocess.STDOUT,
                                      text=True))
    outs = [p.communicate(timeout=240)[0] for p in procs]
    for r, (p, o) in enumerate(zip(procs, outs)):
        assert p.returncode == 0, o
        assert f"rank {r} ok" in o

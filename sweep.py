#!/usr/bin/env python
"""Context-length x Full-call-rate sweep of the decode step: the ODA step
against dense decode on the same kernels (append, then Full attention in
every layer), for the batch-1, 28-layer request of the 128K workload at
other lengths.

    python sweep.py [--contexts 4096,16384,131072,524288] [--rates 0.125,0.41]
                    [--steps 64] [--warmup 4]

Prints each run's bench.py JSON line, then one summary line: per context, the
dense and ODA milliseconds per step, the measured speedup at each rate, and
the speedup the algorithmic-bytes model gives at the realised rate (it tends
to 1/rate as the context grows: Local and the recall head cost the same at
every length, Full grows with it). One GPU; the runs go one after another.
"""

from __future__ import annotations

import argparse
import json
import os
import sys

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--contexts", default="4096,16384,131072,524288")
    ap.add_argument("--rates", default="0.125,0.41")
    ap.add_argument("--steps", type=int, default=64)
    ap.add_argument("--warmup", type=int, default=4)
    a = ap.parse_args()
    import torch
    summary = []
    for ctx in [int(x) for x in a.contexts.split(",")]:
        common = ["--steps", str(a.steps), "--warmup", str(a.warmup), "--context", str(ctx),
                  "--no-cpu-baseline", "--no-e2e"]
        dense = bench.run_oda(bench.parse(common + ["--mode", "full-only"]), 0, 1, 0)
        torch.cuda.empty_cache()
        row = {"context": ctx, "dense_ms": dense["ms_per_step"], "rates": []}
        for rate in [float(x) for x in a.rates.split(",")]:
            oda = bench.run_oda(bench.parse(common + ["--rate", str(rate)]), 0, 1, 0)
            torch.cuda.empty_cache()
            rho = oda["full_call_rate_realised"]
            row["rates"].append({
                "rate": rate, "rate_realised": rho, "oda_ms": oda["ms_per_step"],
                "speedup": dense["ms_per_step"] / oda["ms_per_step"],
                "model_speedup": bench.model_speedup(ctx + a.warmup + a.steps // 2, rho),
                "inverse_rate": 1.0 / rho if rho > 0 else None})
        summary.append(row)
    print(json.dumps({"sweep": summary}), flush=True)


if __name__ == "__main__":
    main()

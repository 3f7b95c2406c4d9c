"""Build liboda.so (and the synthetic-input fill library) in-tree for sm_100a.

    python -m gated_local_full_b200.build [--verbose]

Each .cu file is compiled to an object in parallel, then linked into a shared
library beside this file. Nothing is JIT-compiled at import time.
"""

from __future__ import annotations

import argparse
import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMMON = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr",
          "-Wno-deprecated-declarations"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _compile(src: str, obj: str, extra, verbose: bool) -> str:
    cmd = [nvcc(), *ARCH, *COMMON, *extra, "-c", src, "-o", obj]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stderr}")
    return r.stderr


def _build_lib(name: str, src_dir: str, out_dir: str, verbose: bool, extra=()) -> str:
    build_dir = os.path.join(out_dir, "_build")
    os.makedirs(build_dir, exist_ok=True)
    srcs = sorted(os.path.join(src_dir, f) for f in os.listdir(src_dir) if f.endswith(".cu"))
    objs = [os.path.join(build_dir, os.path.basename(s)[:-3] + ".o") for s in srcs]
    with cf.ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        logs = list(ex.map(lambda so: _compile(so[0], so[1], list(extra), verbose), zip(srcs, objs)))
    if verbose:
        for s, log in zip(srcs, logs):
            print(f"==== {os.path.basename(s)}\n{log}", file=sys.stderr)
    lib = os.path.join(out_dir, name)
    tmp = lib + ".tmp"
    cmd = [nvcc(), *ARCH, "-shared", "-o", tmp, *objs, "-lcudart_static", "-lrt", "-ldl",
           "-lpthread"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed for {name}:\n{r.stderr}")
    os.replace(tmp, lib)
    return lib


def build(verbose: bool = False) -> list:
    """Compile liboda.so and libsynth.so; returns their paths."""
    inc = ["-I", os.path.join(ROOT, "include")]
    oda = _build_lib("liboda.so", os.path.join(PKG, "csrc"), PKG, verbose, inc)
    syn_dir = os.path.join(ROOT, "synth")
    syn = _build_lib("libsynth.so", os.path.join(syn_dir, "csrc"), syn_dir, verbose)
    return [oda, syn]


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose", action="store_true")
    a = ap.parse_args()
    for p in build(a.verbose):
        print(p)

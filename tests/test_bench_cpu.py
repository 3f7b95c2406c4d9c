"""bench.py host logic on the CPU: workload options, the kernel-source digest
that gates recorded ncu traffic, and the reference arm's JSON line."""

import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _args(*argv):
    import bench
    old = sys.argv
    try:
        sys.argv = ["bench.py", *argv]
        return bench.parse()
    finally:
        sys.argv = old


def test_default_config_names_the_headline_workload():
    import bench
    import synth
    a = _args()
    assert (a.context, a.rate, a.mode, a.steps, a.warmup, a.gpus) == (131072, 0.125, "oda", 1024, 8, 1)
    w = synth.ctx128k(steps=4, layers=a.layers, context=a.context, rate=a.rate)
    c = bench.config_block(w, a, 1)
    assert c["workload"].startswith("ctx128k_b1_l28: batch 1, 28 layers")
    assert c["full_call_rate"] == 0.125 and c["context"] == 131072 and c["mode"] == "oda"
    assert "ring 235 MB, Full 15 GB" in c["l2"]


def test_other_context_rate_and_dense_mode():
    import bench
    import synth
    a = _args("--context", "4096", "--rate", "0.41")
    w = synth.ctx128k(steps=4, layers=a.layers, context=a.context, rate=a.rate)
    c = bench.config_block(w, a, 2)
    assert w.name == "ctx4096_rho0.41_b1_l28"
    assert c["context"] == 4096 and c["full_call_rate"] == 0.41 and c["global_batch"] == 2
    d = _args("--mode", "full-only")
    c = bench.config_block(synth.ctx128k(steps=4), d, 1)
    assert c["mode"] == "full-only" and c["full_call_rate"] == 1.0
    assert "dense decode" in c["workload"]


def test_digest_ignores_comments_but_not_code():
    import bench
    code = "int f(int x) {\n  return x + 1;  // one more\n}\n"
    assert bench._code_only(code) == bench._code_only(
        "// header\nint f(int x) {\n\n  return x + 1;\n  /* block\n comment */\n}\n")
    assert bench._code_only(code) != bench._code_only(code.replace("x + 1", "x + 2"))


@pytest.mark.timeout(300)
def test_reference_arm_prints_one_oracle_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "6", "--warmup", "1", "--layers", "2"],
                       capture_output=True, text=True, cwd=ROOT, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


@pytest.mark.parametrize("wl,extra,name,B", [
    ("ctx16k", (), "ctx16k_b8", 8),
    ("mixed", ("--rate", "0.41"), "mixed_b32_rho0.41", 32),
    ("recall", ("--context", "4096"), "recall_b16_ctx4096", 16),
])
def test_other_workloads_and_their_bytes(wl, extra, name, B):
    """The 16K, mixed-batch and recall-head workloads: shapes, whose scores
    gate, the L2 rotation note, and the per-step algorithmic bytes (Local
    min(t, s+w) positions, Full t positions for a flagged row, two appended
    positions, 4096 bytes per position and layer)."""
    import bench
    a = _args("--workload", wl, *extra)
    w, external = bench.make_workload(a, 3)
    assert w.name == name and w.batch == B and w.layers == 1 and w.recall
    assert external == (wl != "recall")
    c = bench.config_block(w, a, 1, 3)
    assert c["copies"] == 3 and "3 independently allocated copies" in c["l2"]
    flags = bench.workload_flags(w)
    if external:
        assert flags.shape == (3, B)
        j = 2
        want = sum((min(int(w.t0[b]) + j, 2052) + (int(w.t0[b]) + j) * int(flags[j][b]) + 2)
                   * 4096 for b in range(B))
        assert bench.batch_step_bytes(w, j, flags[j]) == want
    else:
        assert flags is None
    assert a.mode == "oda" and a.copies == 0


def test_full_only_needs_the_headline_request():
    with pytest.raises(SystemExit):
        _args("--workload", "mixed", "--mode", "full-only")


def test_bytes_model_speedup_tends_to_inverse_rate():
    """The pages' asymptote (speedup -> 1/rho as the context grows): under
    the algorithmic-bytes model the ODA-over-dense ratio rises with t and
    its gap to 1/rho shrinks like (s + w) / (rho t)."""
    import bench
    for rho in (0.125, 0.41):
        prev = 0.0
        for t in (4096, 16384, 131072, 524288, 1 << 22):
            sp = bench.model_speedup(t, rho)
            assert prev < sp < 1.0 / rho
            gap = (1.0 / rho - sp) / (1.0 / rho)
            assert gap <= (2052 + 2) / (rho * t) + 1e-12
            prev = sp
    assert abs(bench.model_speedup(524288, 0.125) - 8.0) / 8.0 < 0.04

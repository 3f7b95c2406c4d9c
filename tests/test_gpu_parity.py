"""GPU parity of the decode path against the float64 oracle, through the C ABI.

Bars: gate flags / compacted indices / count bit-exact; attention within
max-abs 2e-3 + relative 1e-2 (bf16 storage, fp32 accumulation) or 1e-5 (fp32).
"""

import numpy as np
import pytest

import oracle as O
import synth
from tests import _harness as hx

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch():
    import torch as _t
    if not _t.cuda.is_available():
        pytest.skip("needs a GPU")
    return _t


def _bufs(torch, w, dt=None):
    import synth.device as sd
    dt = dt or sd.storage_dtype(w)
    B = w.batch
    return dict(
        out=torch.empty((B, w.hq, w.d), dtype=dt, device="cuda"),
        lse=torch.empty((B, w.hq), dtype=torch.float32, device="cuda"),
        flags=torch.empty(B, dtype=torch.uint8, device="cuda"),
        idx=torch.empty(B, dtype=torch.int32, device="cuda"),
        count=torch.empty(1, dtype=torch.int32, device="cuda"),
    )


def _run_step(ctx, dw, b, step, layer=0, scores=None, theta=0.0):
    """append (this layer) -> local -> gate -> full; returns (local, lse_local)."""
    w = dw.w
    seq = dw.seq_lens[step]
    ctx.append_kv(layer, layer + 1, dw.k_new[step, layer], dw.v_new[step, layer], seq,
                  dw.block_table, dw.cache, dw.ring, w.batch)
    ctx.local_attn(layer, dw.q[step, layer], seq, dw.ring, b["out"], b["lse"], w.batch)
    local, lse_local = b["out"].clone(), b["lse"].clone()
    sc = dw.scores[step] if scores is None else scores
    ctx.gate(sc, theta, w.batch, b["flags"], b["idx"], b["count"])
    ctx.full_attn_gated(layer, dw.q[step, layer], seq, dw.block_table, dw.cache, b["idx"],
                        b["count"], b["out"], b["lse"], w.batch)
    return local, lse_local


def _check_step(torch, w, dw, b, step, local, lse_local, q_host=None, layer=0):
    atol, rtol = hx.tol(w)
    sc = dw.scores[step].cpu().numpy()
    flags, idx, count = O.gate(sc, 0.0)
    assert b["flags"].cpu().numpy().tolist() == flags.tolist()
    assert b["idx"].cpu().numpy().tolist() == idx.tolist()
    assert int(b["count"].item()) == count
    loc = hx.to_f64(local, w)
    out = hx.to_f64(b["out"], w)
    lse_l = lse_local.cpu().numpy().astype(np.float64)
    lse_o = b["lse"].cpu().numpy().astype(np.float64)
    qh = q_host if q_host is not None else w.q_step(step)
    for r in range(w.batch):
        ref = hx.oracle_row(w, step, layer, r, q_host=qh)
        hx.assert_close(loc[r], ref["local"], atol, rtol, f"local step {step} row {r}")
        hx.assert_close(lse_l[r], ref["lse_local"], 1e-4, 1e-5, f"lse local step {step} row {r}")
        want = ref["full"] if flags[r] else ref["local"]
        hx.assert_close(out[r], want, atol, rtol, f"final step {step} row {r}")
        want_lse = ref["lse_full"] if flags[r] else ref["lse_local"]
        hx.assert_close(lse_o[r], want_lse, 1e-4, 1e-5, f"final lse step {step} row {r}")


def test_device_fill_matches_generator(torch):
    w = synth.custom("fill", dtype="bf16", t0=(70, 33), steps=3)
    ctx, dw = hx.setup(w)
    for (l, r, g, kv, p) in ((0, 0, 0, 0, 1), (0, 1, 1, 1, 32), (0, 0, 1, 0, 69)):
        got = dw.read_cache_row(l, r, g, kv, p).view(torch.int16).cpu().numpy().view(np.uint16)
        ref = w.kv_history(l, r, g, kv, p)[p - 1]
        assert np.array_equal(got, ref)
    q = dw.q.view(torch.int16).cpu().numpy().view(np.uint16)
    for s in range(3):
        assert np.array_equal(q[s], w.q_step(s))
        kn, vn = w.kv_new_step(s)
        assert np.array_equal(dw.k_new[s].view(torch.int16).cpu().numpy().view(np.uint16), kn)
        assert np.array_equal(dw.v_new[s].view(torch.int16).cpu().numpy().view(np.uint16), vn)


def test_tiny_fp32_32_steps(torch):
    """fp32, B=2, 2/1 heads, d=64, t0 = 40 and 64, s=4, w=16, needles with
    raw dot +8, fixed scores (+1, -1): every one of the 32 steps matches."""
    w = synth.tiny_fp32()
    ctx, dw = hx.setup(w)
    b = _bufs(torch, w)
    for step in range(w.steps):
        local, lse_local = _run_step(ctx, dw, b, step)
        torch.cuda.synchronize()
        _check_step(torch, w, dw, b, step, local, lse_local)
    assert ctx.get_device_error() == 0
    # the needle makes Local and Full differ on the flagged row
    ref = hx.oracle_row(w, w.steps - 1, 0, 0)
    assert np.abs(ref["local"] - ref["full"]).max() > 1e-2


def test_ctx16k_single_step(torch):
    """bf16, B=8, 16/8 heads, d=128, t=16384, Bernoulli(0.41) flags, needles."""
    w = synth.ctx16k()
    ctx, dw = hx.setup(w)
    b = _bufs(torch, w)
    local, lse_local = _run_step(ctx, dw, b, 0)
    torch.cuda.synchronize()
    _check_step(torch, w, dw, b, 0, local, lse_local)
    assert ctx.get_device_error() == 0


EDGE = [
    dict(name="short_t", t0=(1, 5, 19, 20, 21, 2), sink=4, window=16, d=64, hq=4, hkv=2,
         steps=3),
    dict(name="ragged", t0=(100, 37, 16, 17, 2069, 33), sink=4, window=64, steps=2),
    dict(name="no_sinks", t0=(90, 3, 40), sink=0, window=24, steps=2),
    dict(name="tiny_window", t0=(50, 6, 7), sink=3, window=5, steps=4),
    dict(name="group1", t0=(130, 17), hq=4, hkv=4, steps=2),
    dict(name="group4", t0=(130, 17), hq=8, hkv=2, steps=2),
    dict(name="f32_d128", dtype="f32", t0=(70, 129), steps=2),
    dict(name="bf16_d64", t0=(300, 45), d=64, steps=2),
    dict(name="ring_wraps", t0=(20, 41), sink=4, window=16, steps=40),
    dict(name="long_window", t0=(5000, 4100, 777), sink=4, window=2048, steps=2),
]


@pytest.mark.parametrize("spec", EDGE, ids=[e["name"] for e in EDGE])
def test_edge_cases(torch, spec):
    spec = dict(spec)
    B = len(spec["t0"])
    scores = np.where(np.arange(B) % 2 == 0, 1.0, -1.0).astype(np.float32)
    w = synth.custom(spec.pop("name"), fixed_scores=scores, batch=B, **spec)
    ctx, dw = hx.setup(w)
    b = _bufs(torch, w)
    for step in range(w.steps):
        local, lse_local = _run_step(ctx, dw, b, step)
        torch.cuda.synchronize()
        _check_step(torch, w, dw, b, step, local, lse_local)
        for r in range(B):
            t = int(w.t0[r]) + step
            if t <= w.sink + w.window:   # Local == Full inside the window
                ref = hx.oracle_row(w, step, 0, r)
                assert np.array_equal(ref["local"], ref["full"])
    assert ctx.get_device_error() == 0


@pytest.mark.parametrize("cap", ["0", "2", "16"])
def test_local_cluster_merge_and_global_merge(torch, monkeypatch, cap):
    """Local through each merge of the split KV: the global partials merge
    (cluster size cap 0) and the distributed-shared-memory cluster merge
    (2 and 16 CTAs per segment). Rows span t <= s, t < s + w and t > s + w,
    with ragged last tiles and ranks that get no tile at all."""
    monkeypatch.setenv("ODA_LOCAL_CLUSTER", cap)
    w = synth.custom("cluster", dtype="bf16", hq=8, hkv=4, window=200,
                     t0=(3, 90, 205, 700), steps=2, fixed_scores=(0.0, 0.0, 0.0, 0.0))
    ctx, dw = hx.setup(w)
    b = _bufs(torch, w)
    for step in range(w.steps):
        local, lse_local = _run_step(ctx, dw, b, step)
        torch.cuda.synchronize()
        assert ctx.get_device_error() == 0
        _check_step(torch, w, dw, b, step, local, lse_local)


def test_all_rows_flagged_and_none(torch):
    w = synth.custom("flags", t0=(300, 200, 100), steps=1)
    ctx, dw = hx.setup(w)
    b = _bufs(torch, w)
    for sc in (np.ones(3, np.float32), -np.ones(3, np.float32)):
        s = torch.from_numpy(sc).cuda()
        if sc[0] > 0:
            local, lse_local = _run_step(ctx, dw, b, 0, scores=s)
        else:
            seq = dw.seq_lens[0]
            ctx.local_attn(0, dw.q[0, 0], seq, dw.ring, b["out"], b["lse"], 3)
            local = b["out"].clone()
            ctx.gate(s, 0.0, 3, b["flags"], b["idx"], b["count"])
            ctx.full_attn_gated(0, dw.q[0, 0], seq, dw.block_table, dw.cache, b["idx"],
                                b["count"], b["out"], b["lse"], 3)
            torch.cuda.synchronize()
            assert int(b["count"].item()) == 0
            assert torch.equal(local, b["out"])       # nothing recomputed
            continue
        torch.cuda.synchronize()
        out = hx.to_f64(b["out"], w)
        for r in range(3):
            ref = hx.oracle_row(w, 0, 0, r)
            hx.assert_close(out[r], ref["full"], *hx.tol(w), what=f"row {r}")


GATE_CASES = [1, 31, 32, 33, 100, 1000, 1024]


@pytest.mark.parametrize("B", GATE_CASES)
def test_gate_bit_exact(torch, B):
    from gated_local_full_b200 import oda
    w = synth.custom("gate", t0=(64,), batch=1)
    ctx, _ = hx.setup(w)
    rng = np.random.default_rng(B)
    s = rng.normal(size=B).astype(np.float32)
    specials = np.array([0.0, -0.0, np.nan, np.inf, -np.inf, 1e-45, -1e-45, 0.5], np.float32)
    s[:min(B, specials.size)] = specials[:min(B, specials.size)]
    for theta in (0.0, 0.5, -1.0):
        sc = torch.from_numpy(s).cuda()
        flags = torch.full((B,), 7, dtype=torch.uint8, device="cuda")
        idx = torch.full((B,), 12345, dtype=torch.int32, device="cuda")
        count = torch.full((1,), -9, dtype=torch.int32, device="cuda")
        ctx.gate(sc, theta, B, flags, idx, count)
        torch.cuda.synchronize()
        f, i, c = O.gate(s, theta)
        assert flags.cpu().numpy().tolist() == f.tolist()
        assert idx.cpu().numpy().tolist() == i.tolist()
        assert int(count.item()) == c
    with pytest.raises(oda.OdaError):
        ctx.gate(sc, 0.0, 1025, flags, idx, count)


def test_gate_empty_batch(torch):
    w = synth.custom("gate0", t0=(64,), batch=1)
    ctx, _ = hx.setup(w)
    count = torch.full((1,), -9, dtype=torch.int32, device="cuda")
    ctx.gate(None, 0.0, 0, None, None, count)
    torch.cuda.synchronize()
    assert int(count.item()) == 0


def test_bad_block_table_entry_is_reported(torch):
    from gated_local_full_b200 import oda
    w = synth.custom("bounds", t0=(200, 90), fixed_scores=(1.0, 1.0), batch=2)
    ctx, dw = hx.setup(w)
    b = _bufs(torch, w)
    bt = dw.block_table.clone()
    bt[0, 3] = 10 ** 6                       # out of range physical block
    seq = dw.seq_lens[0]
    ctx.append_kv(0, 1, dw.k_new[0, 0], dw.v_new[0, 0], seq, dw.block_table, dw.cache,
                  dw.ring, 2)
    ctx.gate(dw.scores[0], 0.0, 2, b["flags"], b["idx"], b["count"])
    ctx.full_attn_gated(0, dw.q[0, 0], seq, bt, dw.cache, b["idx"], b["count"], b["out"],
                        b["lse"], 2)
    assert ctx.get_device_error() == oda.ERR_BOUNDS
    assert ctx.get_device_error() == 0        # cleared on read
    # still usable: a correct call matches the oracle
    ctx.full_attn_gated(0, dw.q[0, 0], seq, dw.block_table, dw.cache, b["idx"], b["count"],
                        b["out"], b["lse"], 2)
    torch.cuda.synchronize()
    assert ctx.get_device_error() == 0
    ref = hx.oracle_row(w, 0, 0, 1)
    hx.assert_close(hx.to_f64(b["out"], w)[1], ref["full"], *hx.tol(w), what="after error")


def test_bounded_wait_times_out(torch):
    from gated_local_full_b200 import oda
    w = synth.custom("timeout", t0=(64,), batch=1)
    ctx, _ = hx.setup(w)
    ctx.selftest_wait_timeout(50_000_000)         # 50 ms; nothing ever arrives
    assert ctx.get_device_error() == oda.ERR_TIMEOUT
    with pytest.raises(oda.OdaError):
        ctx.selftest_wait_timeout(0)
    # the context and the device keep working
    test_gate_empty_batch(torch)


def test_argument_errors(torch):
    from gated_local_full_b200 import oda
    w = synth.custom("args", t0=(64, 10), batch=2)
    ctx, dw = hx.setup(w)
    b = _bufs(torch, w)
    seq = dw.seq_lens[0]
    cases = [
        (lambda: ctx.local_attn(1, dw.q[0, 0], seq, dw.ring, b["out"], None, 2), oda.ERR_ARG),
        (lambda: ctx.local_attn(0, None, seq, dw.ring, b["out"], None, 2), oda.ERR_ARG),
        (lambda: ctx.local_attn(0, dw.q[0, 0], seq, dw.ring, b["out"], None, 3), oda.ERR_SHAPE),
        (lambda: ctx.local_attn(0, dw.q[0, 0], seq, dw.ring, b["out"], None, -1), oda.ERR_ARG),
        (lambda: ctx.append_kv(0, 2, dw.k_new[0], dw.v_new[0], seq, dw.block_table, dw.cache,
                               dw.ring, 2), oda.ERR_ARG),
        (lambda: ctx.full_attn_gated(0, dw.q[0, 0], seq, dw.block_table, dw.cache, None,
                                     b["count"], b["out"], None, 2), oda.ERR_ARG),
        (lambda: ctx.recall_score(None, None, None, 64, None, None, None, 0.0, 128, None, 1),
         oda.ERR_ARG),
    ]
    for fn, code in cases:
        with pytest.raises(oda.OdaError) as e:
            fn()
        assert e.value.status == code
    # B == 0 is a valid no-op
    ctx.local_attn(0, dw.q[0, 0], seq, dw.ring, b["out"], None, 0)
    assert ctx.get_device_error() == 0


@pytest.mark.parametrize("shape", ["cluster_b2", "partials_b40"])
def test_inputs_ready_back_to_back(torch, shape):
    """Local and Full launches of consecutive layers with ODA_ATTN_INPUTS_READY
    on every launch but the first (the step's order): the later launches stage
    their first K/V tiles before their dependency wait. Every row, every head
    and every layer is compared with the oracle; batch 2 takes the cluster
    merge, batch 40 the partials merge with the append kernel's plan-free
    in-kernel partition."""
    L = 4
    if shape == "cluster_b2":
        t0 = (9000, 2100)
    else:
        rng = np.random.default_rng(17)
        t0 = tuple(int(x) for x in rng.integers(1, 6000, size=40))
    B = len(t0)
    scores = np.where(np.arange(B) % 3 == 0, 1.0, -1.0).astype(np.float32)
    w = synth.custom("ready_" + shape, layers=L, hq=16, hkv=8, d=128, window=2048,
                     t0=t0, fixed_scores=scores, steps=1)
    ctx, dw = hx.setup(w)
    seq = dw.seq_lens[0]
    ctx.append_kv(0, L, dw.k_new[0], dw.v_new[0], seq, dw.block_table, dw.cache, dw.ring, B)
    dt = dw.q.dtype
    loc = torch.zeros((L, B, w.hq, w.d), dtype=dt, device="cuda")
    lse_l = torch.zeros((L, B, w.hq), dtype=torch.float32, device="cuda")
    for l in range(L):
        ctx.local_attn(l, dw.q[0, l], seq, dw.ring, loc[l], lse_l[l], B, inputs_ready=l > 0)
    flags = torch.empty(B, dtype=torch.uint8, device="cuda")
    idx = torch.empty(B, dtype=torch.int32, device="cuda")
    count = torch.empty(1, dtype=torch.int32, device="cuda")
    ctx.gate(dw.scores[0], 0.0, B, flags, idx, count)
    out = loc.clone()
    lse_o = lse_l.clone()
    for l in range(L):
        ctx.full_attn_gated(l, dw.q[0, l], seq, dw.block_table, dw.cache, idx, count, out[l],
                            lse_o[l], B, inputs_ready=l > 0)
    torch.cuda.synchronize()
    assert ctx.get_device_error() == 0
    f_ref, _, _ = O.gate(scores, 0.0)
    loc64, out64 = hx.to_f64(loc, w), hx.to_f64(out, w)
    lsl, lso = lse_l.cpu().numpy().astype(np.float64), lse_o.cpu().numpy().astype(np.float64)
    atol, rtol = hx.tol(w)
    for l in range(L):
        for r in range(B):
            ref = hx.oracle_row(w, 0, l, r)
            hx.assert_close(loc64[l, r], ref["local"], atol, rtol, f"local l{l} r{r}")
            hx.assert_close(lsl[l, r], ref["lse_local"], 1e-4, 1e-5, f"lse local l{l} r{r}")
            want, wl = (ref["full"], ref["lse_full"]) if f_ref[r] else (ref["local"],
                                                                          ref["lse_local"])
            hx.assert_close(out64[l, r], want, atol, rtol, f"final l{l} r{r}")
            hx.assert_close(lso[l, r], wl, 1e-4, 1e-5, f"final lse l{l} r{r}")
    # a flag bit the library does not define is refused
    from gated_local_full_b200 import oda
    st = oda.lib().oda_local_attn(ctx.handle, 0, oda.ptr(dw.q[0, 0]), oda.ptr(seq),
                                  oda.ptr(dw.ring), oda.ptr(loc[0]), None, B, 2,
                                  oda._stream(None))
    assert st == oda.ERR_ARG


def test_smem_limit_never_lowered(torch):
    """A context sized for 32 rows keeps working after a second context and an
    allocation-free call sized for 4 rows: a kernel's shared-memory limit is
    one value per process, and the library only ever raises it."""
    from gated_local_full_b200 import oda
    w = synth.custom("smemlim", hq=16, hkv=8, d=128, window=256, t0=(3000, 500, 1200, 77),
                     fixed_scores=(1.0, 1.0, -1.0, 1.0), batch=4)
    ctx, dw = hx.setup(w, max_batch=32)
    small_cfg = oda.make_config(layers=1, max_batch=4, hq=16, hkv=8, head_dim=128, sink=4,
                                window=256, dtype="bf16", max_blocks_per_seq=dw.max_blocks,
                                num_blocks=dw.num_blocks)
    small = oda.OdaContext(small_cfg)
    b = _bufs(torch, w)
    seq = dw.seq_lens[0]
    ctx.append_kv(0, 1, dw.k_new[0, 0], dw.v_new[0, 0], seq, dw.block_table, dw.cache,
                  dw.ring, 4)
    ctx.gate(dw.scores[0], 0.0, 4, b["flags"], b["idx"], b["count"])
    scratch = torch.zeros((4, w.hq, w.d), dtype=torch.bfloat16, device="cuda")
    oda.full_attn_gated_static(small_cfg, 0, dw.q[0, 0], seq, dw.block_table, dw.cache,
                               b["idx"], b["count"], scratch, None, 4)
    # the 32-row context after both smaller users
    ctx.local_attn(0, dw.q[0, 0], seq, dw.ring, b["out"], b["lse"], 4)
    local = b["out"].clone()
    ctx.full_attn_gated(0, dw.q[0, 0], seq, dw.block_table, dw.cache, b["idx"], b["count"],
                        b["out"], b["lse"], 4)
    torch.cuda.synchronize()
    assert ctx.get_device_error() == 0 and small.get_device_error() == 0
    loc, out, st = hx.to_f64(local, w), hx.to_f64(b["out"], w), hx.to_f64(scratch, w)
    for r in range(4):
        ref = hx.oracle_row(w, 0, 0, r)
        hx.assert_close(loc[r], ref["local"], *hx.tol(w), what=f"local row {r}")
        want = ref["full"] if r != 2 else ref["local"]
        hx.assert_close(out[r], want, *hx.tol(w), what=f"final row {r}")
        if r != 2:
            hx.assert_close(st[r], ref["full"], *hx.tol(w), what=f"static row {r}")
    small.close()


def test_range_attention(torch):
    """oda_range_attn (the "<focus>" mode) over [lo, hi) regions of the paged
    history: the whole history (= Full), regions that start and end inside a
    block, a single position, a region inside one tile, one from a block
    boundary to the current token, and one of almost 9000 positions; every
    listed row and KV head against the oracle. Then a call that lists a
    subset: unlisted rows keep their output, and regions outside 1..t+1 are
    reported and leave their row untouched."""
    from gated_local_full_b200 import oda
    t0 = (5000, 3000, 700, 2100, 160, 9000)
    B = len(t0)
    regions = [(1, 5001), (1000, 2000), (350, 351), (35, 42), (17, 161), (2, 8999)]
    w = synth.custom("range", hq=16, hkv=8, d=128, window=256, t0=t0, batch=B,
                     fixed_scores=np.ones(B, np.float32))
    ctx, dw = hx.setup(w)
    seq = dw.seq_lens[0]
    ctx.append_kv(0, 1, dw.k_new[0, 0], dw.v_new[0, 0], seq, dw.block_table, dw.cache, dw.ring,
                  B)
    lo = torch.tensor([r[0] for r in regions], dtype=torch.int32, device="cuda")
    hi = torch.tensor([r[1] for r in regions], dtype=torch.int32, device="cuda")
    idx = torch.arange(B, dtype=torch.int32, device="cuda")
    count = torch.full((1,), B, dtype=torch.int32, device="cuda")
    out = torch.zeros((B, w.hq, w.d), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((B, w.hq), dtype=torch.float32, device="cuda")
    ctx.range_attn(0, dw.q[0, 0], seq, lo, hi, dw.block_table, dw.cache, idx, count, out, lse, B)
    torch.cuda.synchronize()
    assert ctx.get_device_error() == 0
    q = w.q_step(0)[0]
    tasks = [(q[b], 0, b, g, regions[b][0], regions[b][1]) for b in range(B)
             for g in range(w.hkv)]
    got, got_lse = hx.to_f64(out, w), lse.cpu().numpy().astype(np.float64)
    for (qb, _, b, g, l_, h_), (o_, lse_) in zip(tasks, hx.oracle_range_heads(w, tasks)):
        hs = slice(g * w.group, (g + 1) * w.group)
        hx.assert_close(got[b, hs], o_, *hx.tol(w), what=f"row {b} head {g} [{l_}, {h_})")
        hx.assert_close(got_lse[b, hs], lse_, 1e-4, 1e-5, what=f"lse row {b} head {g}")
    # the whole history is Full attention
    ref = hx.oracle_row(w, 0, 0, 0)
    hx.assert_close(got[0], ref["full"], *hx.tol(w), what="region = whole history")
    # a subset of rows, two of them with bad regions
    before = out.clone()
    lo2 = lo.clone()
    hi2 = hi.clone()
    lo2[1] = 0                               # lo < 1
    hi2[3] = t0[3] + 2                       # hi > t + 1
    idx2 = torch.tensor([1, 3, 4, -1, -1, -1], dtype=torch.int32, device="cuda")
    count2 = torch.full((1,), 3, dtype=torch.int32, device="cuda")
    hi2[4] = 100
    ctx.range_attn(0, dw.q[0, 0], seq, lo2, hi2, dw.block_table, dw.cache, idx2, count2, out,
                   None, B)
    torch.cuda.synchronize()
    assert ctx.get_device_error() == oda.ERR_BOUNDS
    for b in (0, 1, 2, 3, 5):
        assert torch.equal(out[b], before[b]), f"row {b} changed"
    (o4, _), = hx.oracle_range_heads(w, [(q[4], 0, 4, 0, 17, 100)])
    hx.assert_close(hx.to_f64(out, w)[4, 0:2], o4, *hx.tol(w), what="row 4 [17, 100)")
    with pytest.raises(oda.OdaError):
        ctx.range_attn(0, dw.q[0, 0], seq, None, hi, dw.block_table, dw.cache, idx, count, out,
                       None, B)

"""GPU parity at the workloads' full sizes, in the launch configuration the
benchmark uses (the captured step graph), on outputs the oracle computes one
(row, layer, KV head) at a time."""

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


def _check_heads(w, out_step, q_step, step, pairs, flags_row):
    """out_step: [L][B][hq][d] float64; pairs: (layer, row, kv_head). The
    oracle evaluations run in a process pool (see hx.oracle_heads)."""
    tasks = [(q_step[l, b], l, b, g, int(w.t0[b]) + step, bool(flags_row[b])) for (l, b, g) in pairs]
    for (l, b, g), (o, _) in zip(pairs, hx.oracle_heads(w, tasks)):
        hx.assert_close(out_step[l, b, g * w.group:(g + 1) * w.group], o, *hx.tol(w),
                        what=f"step {step} layer {l} row {b} head {g}")


def test_ctx128k_graph_sampled(torch):
    """batch 1, 28 layers, t = 131072 + step, Full calls drawn per step, with
    the recall head in the step (its last CTA gates the injected scores):
    steps 0..7 run through the captured step graph. Every flagged step is
    checked on all 8 KV heads of layers 0 and 27; an unflagged step the
    same; and 16 random (step, layer, head) triples besides."""
    from gated_local_full_b200.runtime import DecodeStep
    w = synth.ctx128k(steps=8)
    w.recall = True
    flags = w.flags()[:, 0]
    assert flags[1] == 0 and flags[2] == 1 and flags[6] == 1
    ctx, dw = hx.setup(w)
    r = dw.recall
    st = DecodeStep(ctx, 1, dw.cache, dw.ring, dw.block_table, recall=r, external_scores=True,
                    with_lse=True)
    keep = {}
    for step in range(w.steps):
        st.feed(dw.q[step], dw.k_new[step], dw.v_new[step], dw.seq_lens[step],
                gate_scores=dw.scores[step], h_prev=r["h_prev"][step], emb=r["emb"][step],
                h_local=r["h_local"][step])
        st.run()
        keep[step] = (st.out.to(torch.float64).cpu().numpy(), int(st.count.item()),
                      st.flags.cpu().numpy().copy())
    torch.cuda.synchronize()
    assert ctx.get_device_error() == 0
    rng = np.random.default_rng(5)
    extra = {}
    for _ in range(16):
        s_, l_, g_ = int(rng.integers(0, w.steps)), int(rng.integers(1, 27)), int(rng.integers(0, 8))
        extra.setdefault(s_, []).append((l_, 0, g_))
    checked = [i for i in range(w.steps) if flags[i]] + [1]
    for step in range(w.steps):
        out, count, fl = keep[step]
        assert count == int(flags[step]) and fl[0] == flags[step]
        pairs = ([(l, 0, g) for l in (0, 27) for g in range(8)] if step in checked else [])
        pairs += extra.get(step, [])
        if pairs:
            _check_heads(w, out, w.q_step(step), step, pairs, fl)
    st.close()


@pytest.mark.parametrize("rate", synth.MIXED_RATES)
def test_mixed_batch(torch, rate):
    """batch 32, contexts uniform in [4096, 65536], Full calls Bernoulli(rate)
    per row, append inside the step (graph)."""
    from gated_local_full_b200.runtime import DecodeStep
    w = synth.mixed_batch(rate)
    ctx, dw = hx.setup(w)
    st = DecodeStep(ctx, w.batch, dw.cache, dw.ring, dw.block_table, external_scores=True)
    st.feed(dw.q[0], dw.k_new[0], dw.v_new[0], dw.seq_lens[0], gate_scores=dw.scores[0])
    st.run()
    torch.cuda.synchronize()
    assert ctx.get_device_error() == 0
    flags = w.flags()[0]
    f, i, c = O.gate(w.scores()[0], 0.0)
    assert st.flags.cpu().numpy().tolist() == f.tolist() == flags.tolist()
    assert st.idx.cpu().numpy().tolist() == i.tolist() and int(st.count.item()) == c
    out = st.out.to(torch.float64).cpu().numpy()
    q = w.q_step(0)
    # every row and every KV head: Full for the flagged rows, Local for the rest
    pairs = [(0, b, g) for b in range(w.batch) for g in range(w.hkv)]
    _check_heads(w, out, q, 0, pairs, flags)
    st.close()


def test_graph_equals_plain_launches_and_skips_full(torch):
    """The captured step (IF node) and the plain launch sequence give
    bit-identical outputs; with no flagged row the graph leaves Local."""
    from gated_local_full_b200.runtime import DecodeStep
    w = synth.custom("graph", layers=3, batch=4, hq=8, hkv=4, t0=(3000, 100, 2500, 50),
                     fixed_scores=(1.0, -1.0, 1.0, -1.0), steps=2)
    res = {}
    for mode in ("graph", "plain"):
        ctx, dw = hx.setup(w)
        st = DecodeStep(ctx, 4, dw.cache, dw.ring, dw.block_table, external_scores=True,
                        with_lse=True, graph=(mode == "graph"))
        outs = []
        for step in range(2):
            st.feed(dw.q[step], dw.k_new[step], dw.v_new[step], dw.seq_lens[step],
                    gate_scores=dw.scores[step])
            st.run()
            outs.append((st.out.clone(), st.lse.clone()))
        torch.cuda.synchronize()
        assert ctx.get_device_error() == 0
        res[mode] = outs
        if mode == "graph":
            # no flagged row: every row must keep its Local output
            st.feed(dw.q[1], dw.k_new[1], dw.v_new[1], dw.seq_lens[1],
                    gate_scores=-torch.ones(4, device="cuda"))
            st.run()
            torch.cuda.synchronize()
            assert int(st.count.item()) == 0
            out = st.out.to(torch.float64).cpu().numpy()
            q = w.q_step(1)
            for l in range(3):
                for b in range(4):
                    ref = hx.oracle_row(w, 1, l, b)
                    hx.assert_close(out[l, b], ref["local"], *hx.tol(w), what=f"l{l} b{b}")
        st.close()
    for (a, la), (b, lb) in zip(res["graph"], res["plain"]):
        assert torch.equal(a, b) and torch.equal(la, lb)
    out = res["graph"][1][0].to(torch.float64).cpu().numpy()
    for l in range(3):
        for b in range(4):
            ref = hx.oracle_row(w, 1, l, b)
            want = ref["full"] if b % 2 == 0 else ref["local"]
            hx.assert_close(out[l, b], want, *hx.tol(w), what=f"graph l{l} b{b}")


def test_run_io_matches_launch_and_copies(torch):
    """oda_step_graph_run_io (host record in, step, result out, one call)
    gives the same last-layer output and count as feeding the record,
    launching the graph and copying back separately; and the result matches
    the oracle (Full for the flagged rows, Local for the others)."""
    from gated_local_full_b200.runtime import DecodeStep
    w = synth.custom("runio", layers=2, batch=3, hq=8, hkv=4, t0=(700, 90, 1500),
                     fixed_scores=(1.0, -1.0, 1.0), steps=2)
    ctx, dw = hx.setup(w)
    st = DecodeStep(ctx, 3, dw.cache, dw.ring, dw.block_table, external_scores=True)
    recs = st.new_records(w.steps)
    for i in range(w.steps):
        st.pack(recs, i, q=dw.q[i], k_new=dw.k_new[i], v_new=dw.v_new[i],
                seq_lens=dw.seq_lens[i], gate_scores=dw.scores[i])
    hrec = st.new_records(w.steps, pin=True)
    hrec.copy_(recs.cpu())
    # step 0 the separate way, step 1 in one call
    st.feed_record(recs, 0)
    st.run()
    hres = st.new_result()
    st.run_io(hrec[1], hres)
    out1, cnt1 = st.split_result(hres)
    assert int(cnt1.item()) == 2
    got = torch.empty_like(st.out[w.layers - 1])
    got.copy_(st.out[w.layers - 1])
    torch.cuda.synchronize()
    assert ctx.get_device_error() == 0
    assert torch.equal(out1, got.cpu())
    out = out1.to(torch.float64).numpy()
    for b in range(3):
        ref = hx.oracle_row(w, 1, w.layers - 1, b)
        want = ref["full"] if b != 1 else ref["local"]
        hx.assert_close(out[b], want, *hx.tol(w), what=f"run_io row {b}")
    st.close()


def test_full_512k_single_launch(torch):
    """One Full launch at t = 524288 on a one-layer, 2 GB cache (the pages'
    512K operating point; 32768 tiles per KV head, so the split, the dynamic
    tail pool and the 37-partial merges are four times longer than at 128K):
    every KV head against the oracle, and lse too."""
    w = synth.ctx128k(steps=1, layers=1, context=524288)
    ctx, dw = hx.setup(w)
    seq = dw.seq_lens[0]
    ctx.append_kv(0, 1, dw.k_new[0], dw.v_new[0], seq, dw.block_table, dw.cache, dw.ring, 1)
    idx = torch.zeros(1, dtype=torch.int32, device="cuda")
    count = torch.ones(1, dtype=torch.int32, device="cuda")
    out = torch.zeros((1, w.hq, w.d), dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros((1, w.hq), dtype=torch.float32, device="cuda")
    ctx.full_attn_gated(0, dw.q[0, 0], seq, dw.block_table, dw.cache, idx, count, out, lse, 1)
    torch.cuda.synchronize()
    assert ctx.get_device_error() == 0
    q = w.q_step(0)[0]
    t = int(w.t0[0])
    tasks = [(q[0], 0, 0, g, t, True) for g in range(w.hkv)]
    got, got_lse = hx.to_f64(out, w)[0], lse.cpu().numpy().astype(np.float64)[0]
    for g, (o, l) in enumerate(hx.oracle_heads(w, tasks)):
        hs = slice(g * w.group, (g + 1) * w.group)
        hx.assert_close(got[hs], o, *hx.tol(w), what=f"512K head {g}")
        hx.assert_close(got_lse[hs], l, 1e-4, 1e-5, what=f"512K lse head {g}")

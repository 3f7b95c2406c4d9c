"""GPU parity of the tensor-core recall head and the gate it drives.

Score tolerance: |gpu - ref| <= 1e-3 + 1e-3 |ref|. bf16 products are exact in
the fp32 accumulator; what remains is fp32 accumulation over K = 3H terms and
over the hidden units, a few units of 1e-6 relative to the score scale (~1),
far inside the bound. Flags are compared bit-exactly when both sides gate the
same float32 scores, and against the oracle's own scores on every row whose
score is not within the score tolerance of theta.
"""

import numpy as np
import pytest

import oracle as O
import synth
from tests import _harness as hx

pytestmark = pytest.mark.gpu

SCORE_ATOL, SCORE_RTOL = 1e-3, 1e-3


@pytest.fixture(scope="module")
def torch():
    import torch as _t
    if not _t.cuda.is_available():
        pytest.skip("needs a GPU")
    return _t


def _recall_oracle(w, step=0, W1=None, b1=None):
    W1_, b1_, w2, b2 = w.recall_weights()
    W1 = W1_ if W1 is None else W1
    b1 = b1_ if b1 is None else b1
    hs = [synth.bf16_bits_to_f32(h).astype(np.float64) for h in w.hidden_step(step)]
    Wf = synth.bf16_bits_to_f32(W1).astype(np.float64)
    w2f = synth.bf16_bits_to_f32(w2).astype(np.float64)
    return O.recall_score(*hs, Wf, np.asarray(b1, np.float64), w2f, float(b2))


SHAPES = [(16, 2048, 4096), (1, 2048, 4096), (17, 64, 128), (5, 192, 384), (256, 128, 256),
          (33, 2048, 4096), (2, 64, 128), (3, 192, 384), (4, 2048, 4096), (1, 1024, 8192),
          (2, 4096, 1024)]


@pytest.mark.parametrize("B,H,hidden", SHAPES, ids=[f"B{b}_H{h}_hid{n}" for b, h, n in SHAPES])
def test_recall_scores(torch, B, H, hidden):
    w = synth.custom("recall", batch=B, t0=[20] * B, recall=True, hidden=H, recall_hidden=hidden)
    ctx, dw = hx.setup(w)
    r = dw.recall
    scores = torch.full((B,), float("nan"), dtype=torch.float32, device="cuda")
    ctx.recall_score(r["h_prev"][0], r["emb"][0], r["h_local"][0], H, r["W1"], r["b1"], r["w2"],
                     r["b2"], hidden, scores, B)
    torch.cuda.synchronize()
    assert ctx.get_device_error() == 0
    got = scores.cpu().numpy().astype(np.float64)
    ref = _recall_oracle(w)
    hx.assert_close(got, ref, SCORE_ATOL, SCORE_RTOL, "recall score")
    # deterministic: a second call gives the same bits
    again = torch.empty_like(scores)
    ctx.recall_score(r["h_prev"][0], r["emb"][0], r["h_local"][0], H, r["W1"], r["b1"], r["w2"],
                     r["b2"], hidden, again, B)
    torch.cuda.synchronize()
    assert torch.equal(scores, again)


def test_recall_zero_weights_special_case(torch):
    """W1 = 0 reduces the head to w2 . GELU(b1) + b2 for every row."""
    B, H, hidden = 4, 128, 256
    w = synth.custom("recall0", batch=B, t0=[20] * B, recall=True, hidden=H, recall_hidden=hidden)
    ctx, dw = hx.setup(w)
    r = dw.recall
    rng = np.random.default_rng(0)
    b1 = rng.normal(size=hidden).astype(np.float32)
    W1z = torch.zeros_like(r["W1"])
    scores = torch.empty(B, dtype=torch.float32, device="cuda")
    ctx.recall_score(r["h_prev"][0], r["emb"][0], r["h_local"][0], H, W1z,
                     torch.from_numpy(b1).cuda(), r["w2"], 0.75, hidden, scores, B)
    torch.cuda.synchronize()
    w2 = r["w2"].cpu().numpy().astype(np.float64)
    expect = w2 @ O.gelu_erf(b1.astype(np.float64)) + 0.75
    hx.assert_close(scores.cpu().numpy().astype(np.float64), np.full(B, expect), 1e-5, 1e-5,
                    "W1=0 score")


def test_recall_rejects_unsupported_shapes(torch):
    from gated_local_full_b200 import oda
    w = synth.custom("recallbad", batch=2, t0=[20, 20], recall=True, hidden=128,
                     recall_hidden=256)
    ctx, dw = hx.setup(w)
    r = dw.recall
    s = torch.empty(2, dtype=torch.float32, device="cuda")
    for H, hidden, B in ((100, 256, 2), (128, 200, 2), (128, 256, 257)):
        with pytest.raises(oda.OdaError) as e:
            ctx.recall_score(r["h_prev"][0], r["emb"][0], r["h_local"][0], H, r["W1"], r["b1"],
                             r["w2"], 0.0, hidden, s, B)
        assert e.value.status == oda.ERR_SHAPE


@pytest.mark.parametrize("ctxlen", [4096, 131072])
def test_gated_step_with_recall_head(torch, ctxlen):
    """B=16, hidden 2048, 6144 -> 4096 -> 1 GELU head, theta = 0: the scores
    decide the gate; flagged rows get Full, the rest keep Local."""
    from gated_local_full_b200.runtime import DecodeStep
    w = synth.recall_step(ctxlen)
    ctx, dw = hx.setup(w)
    r = dw.recall
    st = DecodeStep(ctx, w.batch, dw.cache, dw.ring, dw.block_table, recall=r, with_lse=True)
    st.feed(dw.q[0], dw.k_new[0], dw.v_new[0], dw.seq_lens[0], h_prev=r["h_prev"][0],
            emb=r["emb"][0], h_local=r["h_local"][0])
    st.run()
    torch.cuda.synchronize()
    assert ctx.get_device_error() == 0
    got_s = st.scores.cpu().numpy()
    ref_s = _recall_oracle(w)
    hx.assert_close(got_s.astype(np.float64), ref_s, SCORE_ATOL, SCORE_RTOL, "scores")
    flags = st.flags.cpu().numpy()
    f_gpu, i_gpu, c_gpu = O.gate(got_s, 0.0)
    assert flags.tolist() == f_gpu.tolist()
    assert st.idx.cpu().numpy().tolist() == i_gpu.tolist() and int(st.count.item()) == c_gpu
    f_ref, _, _ = O.gate(ref_s.astype(np.float32), 0.0)
    clear = np.abs(ref_s) > SCORE_ATOL + SCORE_RTOL * np.abs(ref_s)
    assert np.array_equal(flags[clear], f_ref[clear])
    assert 0 < c_gpu < w.batch
    # attention: sampled rows and heads (all rows' Local at ctx 4096)
    out = hx.to_f64(st.out[0], w)
    q = w.q_step(0)[0]
    # every row; two KV heads each at 131072, all eight at 4096
    rng = np.random.default_rng(ctxlen)
    pairs = [(b, g) for b in range(w.batch) for g in
             (range(w.hkv) if ctxlen <= 4096 else rng.choice(w.hkv, 2, replace=False))]
    tasks = [(q[b], 0, b, int(g), ctxlen, bool(flags[b])) for (b, g) in pairs]
    for (b, g), (o, _) in zip(pairs, hx.oracle_heads(w, tasks)):
        hx.assert_close(out[b, g * w.group:(g + 1) * w.group], o, *hx.tol(w),
                        what=f"row {b} head {g}")
    st.close()


@pytest.mark.parametrize("B", [1, 2, 16, 64])
def test_step_recall_split_plain_and_graph(torch, B):
    """The step splits the head's first layer: h_{t-1} and E(x_t) in a kernel
    that starts with the step (beside the Local launches in the graph, first
    on one stream otherwise), h^L_t after the last Local launch. A rank of the
    head that finds the prefix incomplete computes its share of the prefix's
    range itself, so the sum order (not the result) can differ between runs:
    both stay within the head's tolerance of the oracle and agree to float32
    rounding. On one stream the prefix is always complete, so repeated plain
    steps agree bit for bit."""
    from gated_local_full_b200.runtime import DecodeStep
    from gated_local_full_b200 import oda
    # a step of enough layers for the split (hidden 2048, 6144 -> 4096; batch
    # widths 16 and 64)
    w = synth.custom("recall_split", layers=oda.RECALL_SPLIT_MIN_LAYERS, batch=B, t0=[300],
                     hq=16, hkv=8, window=128, recall=True, hidden=2048, recall_hidden=4096)
    ctx, dw = hx.setup(w)
    r = dw.recall
    got = []
    for graph in (False, True, False, True):
        st = DecodeStep(ctx, w.batch, dw.cache, dw.ring, dw.block_table, recall=r, graph=graph)
        st.feed(dw.q[0], dw.k_new[0], dw.v_new[0], dw.seq_lens[0], h_prev=r["h_prev"][0],
                emb=r["emb"][0], h_local=r["h_local"][0])
        st.run()
        torch.cuda.synchronize()
        assert ctx.get_device_error() == 0
        got.append(st.scores.cpu().numpy().astype(np.float64))
        st.close()
    assert np.array_equal(got[0], got[2])
    ref = _recall_oracle(w)
    for g in got:
        hx.assert_close(g, ref, SCORE_ATOL, SCORE_RTOL, "scores")
        np.testing.assert_allclose(g, got[0], rtol=1e-5, atol=1e-5)
    # the standalone head: every rank computes its quarter of the prefix's range
    s = torch.empty(w.batch, dtype=torch.float32, device="cuda")
    ctx.recall_score(r["h_prev"][0], r["emb"][0], r["h_local"][0], r["H"], r["W1"], r["b1"],
                     r["w2"], r["b2"], r["hidden"], s, w.batch)
    torch.cuda.synchronize()
    alone = s.cpu().numpy().astype(np.float64)
    hx.assert_close(alone, ref, SCORE_ATOL, SCORE_RTOL, "standalone scores")
    np.testing.assert_allclose(alone, got[0], rtol=1e-5, atol=1e-5)


"""GPU parity of the budgeted selection (oda_select_budget) against the
float64 oracle: the selected set bit-exact (k largest scores, ties to the
earlier position, NaN lowest, +0 and -0 equal) and the net gain per
reference position within 1e-12 relative (a float64 sum of float32 gains)."""

import numpy as np
import pytest

import oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def torch():
    import torch as _t
    if not _t.cuda.is_available():
        pytest.skip("needs a GPU")
    return _t


@pytest.fixture(scope="module")
def ctx(torch):
    from gated_local_full_b200 import oda
    cfg = oda.make_config(layers=1, max_batch=1, hq=2, hkv=1, head_dim=64, sink=4, window=16,
                          dtype="f32", max_blocks_per_seq=4, num_blocks=4)
    c = oda.OdaContext(cfg)
    yield c
    c.close()


def _select(torch, ctx, scores, gain, k):
    s = torch.from_numpy(scores).cuda()
    g = torch.from_numpy(gain).cuda()
    sel = torch.full((scores.size,), 7, dtype=torch.uint8, device="cuda")
    net = torch.zeros(1, dtype=torch.float64, device="cuda")
    ctx.select_budget(s, g, k, sel, net)
    torch.cuda.synchronize()
    assert ctx.get_device_error() == 0
    return sel.cpu().numpy(), float(net.item())


def _inputs(n, seed):
    rng = np.random.default_rng(seed)
    gain = rng.normal(0.0, 1.0, n).astype(np.float32)
    q = (gain + rng.normal(0.0, 1.0, n)).astype(np.float32)    # a noisy predictor of the gain
    q[::97] = np.float32(0.5)                                   # runs of equal scores
    q[5::101] = np.float32(-0.0)
    q[7::103] = np.float32(0.0)
    q[11::211] = np.nan
    q[13::307] = np.inf
    q[17::409] = -np.inf
    q[19::503] = np.float32(1e-40)                              # denormal
    return q, gain


@pytest.mark.parametrize("n", [1, 5, 1000, 200003])
def test_select_matches_oracle(torch, ctx, n):
    q, gain = _inputs(n, n)
    for k in sorted({0, 1, O.budget_count(n, 0.4), O.budget_count(n, 0.125), n}):
        if k > n:
            continue
        got, net = _select(torch, ctx, q, gain, k)
        ref = O.select_top(q, k)
        assert np.array_equal(got, ref), f"n={n} k={k}: {int((got != ref).sum())} differ"
        want = O.net_gain_per_position(gain, ref)
        assert abs(net - want) <= 1e-12 * max(1.0, abs(want)), (net, want)


def test_select_ties_and_specials(torch, ctx):
    """All-equal scores take the first k; a run of equal scores straddling the
    k-th place is cut in position order; -0 and +0 are one value; NaN is
    taken only after every number, -inf included."""
    eq = np.full(300, 2.0, np.float32)
    got, _ = _select(torch, ctx, eq, np.ones(300, np.float32), 123)
    assert got.tolist() == [1] * 123 + [0] * 177
    s = np.array([np.nan, -0.0, 3.0, 0.0, -np.inf, 0.0, np.nan, -0.0, 1e-45], np.float32)
    g = np.arange(9, dtype=np.float32)
    for k in range(10):
        got, net = _select(torch, ctx, s, g, k)
        ref = O.select_top(s, k)
        assert np.array_equal(got, ref), (k, got.tolist(), ref.tolist())
        assert net == O.net_gain_per_position(g, ref)


def test_select_large_by_properties_and_oracle_policy(torch, ctx):
    """4M + 5 positions at a 40 % budget: exactly k selected, no unselected
    score above a selected one, equal scores cut in position order, the net
    gain equal to numpy's float64 sum; and the offline Oracle (selecting by
    the gain itself) captures at least the noisy predictor's net gain, which
    beats random selection."""
    n = (1 << 22) + 5
    q, gain = _inputs(n, 3)
    q[np.isnan(q)] = 0.25                      # order checks below on numbers only
    k = O.budget_count(n, 0.4)
    got, net = _select(torch, ctx, q, gain, k)
    sel = got.astype(bool)
    assert int(sel.sum()) == k
    lo_sel, hi_unsel = q[sel].min(), q[~sel].max()
    assert lo_sel >= hi_unsel
    if lo_sel == hi_unsel:
        at = np.nonzero(q == lo_sel)[0]
        picked = sel[at]
        assert np.all(picked[:int(picked.sum())]) and not np.any(picked[int(picked.sum()):])
    want = float(gain.astype(np.float64)[sel].sum() / n)
    assert abs(net - want) <= 1e-12 * max(1.0, abs(want))
    _, net_oracle = _select(torch, ctx, gain, gain, k)
    rand = O.random_expected_net_gain(gain, k)
    assert net_oracle >= net > rand

"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: brute-force
enumeration, closed forms, special cases that reduce to a known value,
invariants, and the FLOP ratios the pages print. A plausible slip in the
oracle (a dropped term, an off-by-one in a set bound, a wrong GQA index, a
transposed operand, a non-strict comparison) fails at least one of them.
"""

import json
import math
import os

import numpy as np
import pytest

import oracle as o

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------------
# access sets (ODA summary, Methodology / Local-First Decoding)
# --------------------------------------------------------------------------

def test_access_sets_brute_force():
    """Membership by the words of the definition: position j is Local iff it
    is one of the first s positions or one of the w most recent ones."""
    for t in range(1, 41):
        for s in range(0, 6):
            for w in range(1, 21):
                expect = {j for j in range(1, t + 1) if j <= s or t - j < w}
                assert o.local_access_set(t, s, w) == expect, (t, s, w)
                assert o.full_access_set(t) == set(range(1, t + 1))


def test_access_set_sizes_and_inclusion():
    for t in range(1, 200, 7):
        for s, w in ((4, 16), (0, 8), (4, 2048), (3, 1)):
            SL, SF = o.local_access_set(t, s, w), o.full_access_set(t)
            assert len(SL) == min(t, s + w)
            assert SL <= SF
            assert (SL == SF) == (t <= s + w)
            assert t in SL                      # the current token is always local
            assert set(range(1, min(s, t) + 1)) <= SL


def test_pages_operating_point_sizes():
    # s = 4, w = 2048 at 128K: 2052 local keys, 131072 full keys
    assert len(o.local_access_set(131072, 4, 2048)) == 2052
    assert len(o.full_access_set(131072)) == 131072


# --------------------------------------------------------------------------
# attention
# --------------------------------------------------------------------------

def _rng(seed=0):
    return np.random.default_rng(seed)


def test_single_key_returns_its_value():
    r = _rng(1)
    q = r.normal(size=(2, 8)); K = r.normal(size=(1, 1, 8)); V = r.normal(size=(1, 1, 8))
    out, lse = o.attend(q, K, V, {1})
    assert np.array_equal(out, np.repeat(V[0], 2, axis=0))
    assert np.allclose(lse, (q @ K[0, 0]) / math.sqrt(8), rtol=0, atol=1e-15)


def test_identical_keys_average_values():
    r = _rng(2)
    n, d = 9, 16
    q = r.normal(size=(1, d)); k = r.normal(size=d)
    K = np.repeat(k[None, None, :], n, axis=1); V = r.normal(size=(1, n, d))
    out, lse = o.attend(q, K, V, range(1, n + 1))
    assert np.allclose(out[0], V[0].mean(axis=0), atol=1e-14)
    assert math.isclose(lse[0], q[0] @ k / math.sqrt(d) + math.log(n), abs_tol=1e-13)


def test_two_keys_logistic_weights():
    """Two keys: the weight on key 1 is the logistic function of the logit gap."""
    d = 4
    q = np.array([[2.0, 0.0, 0.0, 0.0]])
    K = np.array([[[1.5, 0, 0, 0], [-0.5, 0, 0, 0]]])
    V = np.array([[[1.0, 0, 0, 0], [0, 1.0, 0, 0]]])
    gap = (2.0 * 1.5 - 2.0 * -0.5) / math.sqrt(d)          # = 2.0
    p1 = 1.0 / (1.0 + math.exp(-gap))
    out, _ = o.attend(q, K, V, {1, 2})
    assert np.allclose(out[0], [p1, 1 - p1, 0, 0], atol=1e-15)


def test_dominant_needle():
    r = _rng(3)
    n, d = 300, 32
    q = r.normal(size=(1, d)); q /= np.linalg.norm(q)
    K = r.normal(size=(1, n, d)) * 0.01
    K[0, 123] = q[0] * 60.0 * math.sqrt(d)                  # logit ~ +60 above the rest
    V = r.normal(size=(1, n, d))
    out, _ = o.attend(q, K, V, range(1, n + 1))
    assert np.allclose(out[0], V[0, 123], atol=1e-12)


def test_permutation_invariance_and_subset():
    r = _rng(4)
    n, d = 50, 8
    q = r.normal(size=(2, d)); K = r.normal(size=(1, n, d)); V = r.normal(size=(1, n, d))
    perm = r.permutation(n)
    Kp, Vp = K[:, perm], V[:, perm]
    S = {5, 9, 17, 40}
    Sp = {int(np.where(perm == j - 1)[0][0]) + 1 for j in S}
    a, la = o.attend(q, K, V, S)
    b, lb = o.attend(q, Kp, Vp, Sp)
    assert np.allclose(a, b, atol=1e-14) and np.allclose(la, lb, atol=1e-14)


def test_gqa_group_mapping():
    """Query head h reads KV head h // (Hq/Hkv): contiguous groups."""
    d, n = 8, 6
    r = _rng(5)
    q = r.normal(size=(4, d))
    K = np.zeros((2, n, d)); K[0] = r.normal(size=(n, d))   # group 1 has equal (zero) keys
    V = r.normal(size=(2, n, d))
    out, _ = o.attend(q, K, V, range(1, n + 1))
    for h in (2, 3):
        assert np.allclose(out[h], V[1].mean(axis=0), atol=1e-14)
    for h in (0, 1):
        assert not np.allclose(out[h], V[0].mean(axis=0), atol=1e-3)


def test_scale_is_inverse_sqrt_d():
    d = 64
    q = np.zeros((1, d)); q[0, 0] = 1.0
    K = np.zeros((1, 2, d)); K[0, 0, 0] = 8.0               # raw dot 8 -> logit 1
    V = np.zeros((1, 2, d)); V[0, 0, 0] = 1.0
    out, lse = o.attend(q, K, V, {1, 2})
    assert math.isclose(out[0, 0], math.e / (math.e + 1.0), rel_tol=1e-15)
    assert math.isclose(lse[0], math.log(math.e + 1.0), rel_tol=1e-15)


def test_local_equals_full_inside_window():
    r = _rng(6)
    s, w, d = 4, 16, 8
    for t in (1, 5, 19, 20):
        q = r.normal(size=(2, d)); K = r.normal(size=(1, t, d)); V = r.normal(size=(1, t, d))
        a, la = o.local_attention(q, K, V, t, s, w)
        b, lb = o.full_attention(q, K, V, t)
        assert np.array_equal(a, b) and np.array_equal(la, lb)
    t = 21
    q = r.normal(size=(2, d)); K = r.normal(size=(1, t, d)); V = r.normal(size=(1, t, d))
    a, _ = o.local_attention(q, K, V, t, s, w)
    b, _ = o.full_attention(q, K, V, t)
    assert not np.allclose(a, b)


def test_empty_set_rejected():
    with pytest.raises(ValueError):
        o.attend(np.zeros((1, 4)), np.zeros((1, 1, 4)), np.zeros((1, 1, 4)), set())


# --------------------------------------------------------------------------
# gate (ODA summary, Methodology / Local-First Decoding: Full iff q_t > theta)
# --------------------------------------------------------------------------

def test_gate_edge_values_bit_exact():
    tiny = np.float32(1e-45)                                  # smallest positive denormal
    scores = np.array([0.0, -0.0, np.nan, np.inf, -np.inf, tiny, -tiny, 1.0, -1.0],
                      dtype=np.float32)
    flags, idx, count = o.gate(scores, 0.0)
    assert flags.tolist() == [0, 0, 0, 1, 0, 1, 0, 1, 0]
    assert count == 3
    assert idx.tolist() == [3, 5, 7, -1, -1, -1, -1, -1, -1]
    assert idx.dtype == np.int32 and flags.dtype == np.uint8


def test_gate_strict_at_theta_and_float32_compare():
    th = 0.5
    s = np.array([0.5, np.nextafter(np.float32(0.5), np.float32(1)), 0.49999997], np.float32)
    flags, idx, count = o.gate(s, th)
    assert flags.tolist() == [0, 1, 0] and count == 1 and idx.tolist() == [1, -1, -1]
    # 0.1 is compared in float32: f32(0.1) is not greater than f32(0.1)
    flags, _, _ = o.gate(np.array([0.1], np.float32), 0.1)
    assert flags.tolist() == [0]


def test_gate_all_and_none():
    assert o.gate(np.ones(5, np.float32))[2] == 5
    f, idx, c = o.gate(-np.ones(5, np.float32))
    assert c == 0 and idx.tolist() == [-1] * 5 and f.sum() == 0
    f, idx, c = o.gate(np.zeros(0, np.float32))
    assert c == 0 and idx.size == 0


# --------------------------------------------------------------------------
# training-side math (ODA summary, Learning to Predict Recall Benefit)
# --------------------------------------------------------------------------

def test_signed_log_closed_forms():
    assert o.signed_log(0.0) == 0.0
    assert math.isclose(float(o.signed_log(math.e - 1.0)), 1.0, rel_tol=1e-15)
    assert math.isclose(float(o.signed_log(-(math.e ** 2 - 1.0))), -2.0, rel_tol=1e-15)
    u = np.linspace(-50, 50, 2001)
    T = o.signed_log(u)
    assert np.allclose(T, -o.signed_log(-u), atol=0)                 # odd
    assert np.all(np.diff(T) > 0)                                      # strictly increasing
    inv = np.sign(T) * np.expm1(np.abs(T))
    assert np.allclose(inv, u, rtol=1e-13, atol=1e-13)                 # invertible
    assert np.array_equal(np.sign(T), np.sign(u))                      # gate sign unchanged


def test_huber_transition_one():
    assert o.huber1(0.5) == 0.125
    assert o.huber1(1.0) == 0.5
    assert o.huber1(2.0) == 1.5
    assert o.huber1(-3.0) == 2.5
    eps = 1e-7                                                          # C1 at |r| = 1
    left = (o.huber1(1.0) - o.huber1(1.0 - eps)) / eps
    right = (o.huber1(1.0 + eps) - o.huber1(1.0)) / eps
    assert abs(left - 1.0) < 1e-6 and abs(right - 1.0) < 1e-6
    assert o.recall_regression_loss([0.0, 3.0], [0.5, 0.0]) == (0.125 + 2.5) / 2


def test_gain_and_penalized_loss():
    lpF, lpL = np.log(0.6), np.log(0.2)
    g = o.access_gain(lpF, lpL)
    assert math.isclose(float(g), math.log(3.0), rel_tol=1e-15)
    lossL, lossF = -lpL, -lpF
    lam = 0.3
    assert o.penalized_step_loss(lossL, g, 0, lam) == lossL
    assert math.isclose(float(o.penalized_step_loss(lossL, g, 1, lam)), lossF + lam, rel_tol=1e-14)
    gains = np.linspace(-2, 2, 41)
    for gg in gains:
        losses = [float(o.penalized_step_loss(1.0, gg, a, lam)) for a in (0, 1)]
        a_star = int(o.best_action(gg, lam))
        assert losses[a_star] == min(losses)
        assert (float(o.regression_target(gg, lam)) > 0) == bool(a_star)


# --------------------------------------------------------------------------
# recall head
# --------------------------------------------------------------------------

def test_gelu_erf_values():
    g = o.gelu_erf(np.array([0.0, 1.0, -1.0, 2.0]))
    assert g[0] == 0.0
    assert math.isclose(g[1], 0.8413447460685429, rel_tol=1e-15)     # Phi(1)
    assert math.isclose(g[2], -0.15865525393145707, rel_tol=1e-14)    # -Phi(-1)
    assert math.isclose(g[3], 2 * 0.9772498680518208, rel_tol=1e-15)  # 2 Phi(2)
    x = np.linspace(-4, 4, 81)
    assert np.allclose(o.gelu_erf(x) - o.gelu_erf(-x), x, atol=1e-14)


def test_recall_score_special_cases():
    r = _rng(7)
    B, H, hid = 3, 5, 7
    hp, em, hl = (r.normal(size=(B, H)) for _ in range(3))
    b1 = r.normal(size=hid); w2 = r.normal(size=hid); b2 = 0.25
    s = o.recall_score(hp, em, hl, np.zeros((hid, 3 * H)), b1, w2, b2)
    assert np.allclose(s, w2 @ o.gelu_erf(b1) + b2, atol=1e-14)
    # one hidden unit reading input H+3 must see E(x_t)[3] (concat order h, E, hL)
    W1 = np.zeros((1, 3 * H)); W1[0, H + 3] = 1.0
    s = o.recall_score(hp, em, hl, W1, np.zeros(1), np.ones(1), 0.0)
    assert np.allclose(s, o.gelu_erf(em[:, 3]), atol=1e-15)
    W1 = np.zeros((1, 3 * H)); W1[0, 2 * H] = 1.0
    s = o.recall_score(hp, em, hl, W1, np.zeros(1), np.ones(1), 0.0)
    assert np.allclose(s, o.gelu_erf(hl[:, 0]), atol=1e-15)


# --------------------------------------------------------------------------
# decode step composition and the savings model
# --------------------------------------------------------------------------

def test_decode_step_selects_full_for_flagged_rows():
    r = _rng(8)
    B, hq, hkv, d, s, w = 3, 4, 2, 8, 2, 4
    t = [30, 3, 12]
    q = r.normal(size=(B, hq, d))
    K = [r.normal(size=(hkv, tt, d)) for tt in t]
    V = [r.normal(size=(hkv, tt, d)) for tt in t]
    res = o.decode_step(q, K, V, t, s, w, scores=[0.3, 2.0, -1.0])
    assert res["count"] == 2 and res["idx"].tolist() == [0, 1, -1]
    for b in range(B):
        full, _ = o.full_attention(q[b], K[b], V[b], t[b])
        local, _ = o.local_attention(q[b], K[b], V[b], t[b], s, w)
        expect = full if res["flags"][b] else local
        assert np.array_equal(res["out"][b], expect)
    assert np.array_equal(res["out"][1], res["local"][1])   # t=3 <= s+w: Local == Full


def test_delta_F_matches_counted_flops():
    """Run the oracle for many steps at fixed n, count what it executed, and
    compare with the closed form at the realised call rate (exact integers)."""
    r = _rng(9)
    hq, hkv, d, s, w, n = 4, 2, 16, 4, 16, 100
    H, hid = 6, 5
    steps = 40
    flags = (r.random(steps) < 0.3).astype(int)
    q = r.normal(size=(1, hq, d)); K = [r.normal(size=(hkv, n, d))]; V = [r.normal(size=(hkv, n, d))]
    W1 = r.normal(size=(hid, 3 * H)); b1 = np.zeros(hid); w2 = r.normal(size=hid)
    fc = o.FlopCounter()
    for i in range(steps):
        hs = [r.normal(size=(1, H)) for _ in range(3)]
        o.recall_score(*hs, W1, b1, w2, 0.0, flops=fc)
        o.decode_step(q, K, V, [n], s, w, scores=[1.0 if flags[i] else -1.0], flops=fc)
    F_full = o.attention_flops(n, d, hq)
    F_local = o.attention_flops(min(n, s + w), d, hq)
    F_recall = o.recall_flops(3 * H, hid)
    rho = __import__("fractions").Fraction(int(flags.sum()), steps)
    saved_per_step = __import__("fractions").Fraction(steps * F_full - fc.total(), steps)
    assert saved_per_step == o.delta_F(F_full, F_local, F_recall, rho)
    assert fc.by["local"] == steps * F_local
    assert fc.by["full"] == int(flags.sum()) * F_full


def test_flop_fractions_printed_on_the_pages():
    g = json.load(open(os.path.join(GOLDEN, "flop_fractions.json")))
    for p in g["points"]:
        n = p["n_input"] + p["n_output"]
        frac = o.oda_flop_fraction(n, p["rho"], s=g["s"], w=g["w"],
                                   recall_params=g["recall_params"], **g["assumed_backbone"])
        tol = g["tolerance_abs"][str(p["fraction"])]
        assert abs(frac - p["fraction"]) <= tol, (p, frac)


def test_speedup_tends_to_inverse_rate():
    """A fixed call rate rho leaves Full's O(n) term, so the FLOP ratio tends to
    rho as n grows (learnaivisually explainer: the speedup approaches 1/rho)."""
    shape = dict(layers=28, hidden=2048, hq=16, hkv=8, d=128, intermediate=6144, vocab=151936)
    prev = None
    for n in (2 ** 17, 2 ** 20, 2 ** 24, 2 ** 28):
        f = o.oda_flop_fraction(n, 0.125, s=4, w=2048, recall_params=28325889, **shape)
        assert f > 0.125
        if prev is not None:
            assert f < prev
        prev = f
    assert abs(prev - 0.125) < 1e-3


# --------------------------------------------------------------------------
# range-restricted ("focus") attention (Declarative Attention pages, the
# "<focus>" mode: attention narrowed to one region, reading only its KV)
# --------------------------------------------------------------------------

def test_range_access_set_brute_force():
    """Position p is in the region [lo, hi) iff lo <= p and p < hi, and the
    set never reaches outside it."""
    for lo in range(1, 12):
        for hi in range(lo, 14):
            want = {p for p in range(1, 20) if lo <= p < hi}
            assert o.range_access_set(lo, hi) == want
            assert len(o.range_access_set(lo, hi)) == hi - lo


def test_range_special_cases():
    """Three regions with a known answer: the whole history is Full, the w
    most recent positions are Local without sinks, and one position gives
    its value with lse = its logit."""
    rng = np.random.default_rng(11)
    d, t, w = 16, 37, 9
    q = rng.normal(size=(4, d))
    K = rng.normal(size=(2, t, d))
    V = rng.normal(size=(2, t, d))
    full, lse_f = o.full_attention(q, K, V, t)
    r, lse_r = o.range_attention(q, K, V, 1, t + 1)
    assert np.array_equal(full, r) and np.array_equal(lse_f, lse_r)
    loc, lse_l = o.local_attention(q, K, V, t, 0, w)
    r, lse_r = o.range_attention(q, K, V, t - w + 1, t + 1)
    assert np.array_equal(loc, r) and np.array_equal(lse_l, lse_r)
    p = 13
    r, lse_r = o.range_attention(q, K, V, p, p + 1)
    for h in range(4):
        g = h // 2
        assert np.allclose(r[h], V[g, p - 1], atol=1e-15)
        assert abs(lse_r[h] - K[g, p - 1] @ q[h] / math.sqrt(d)) < 1e-12


def test_range_two_positions_closed_form():
    """A region of two positions: the logistic weights of their logit gap,
    and no weight at all on positions outside it (here a huge-logit key at
    position 1 that a wrong lower bound would let dominate)."""
    d = 4
    q = np.array([[1.0, 0.0, 0.0, 0.0]])
    K = np.zeros((1, 5, d))
    K[0, 0, 0] = 100.0            # position 1, outside [3, 5)
    K[0, 2, 0] = 2.0              # position 3
    K[0, 3, 0] = -2.0             # position 4
    K[0, 4, 0] = 100.0            # position 5, outside [3, 5)
    V = np.zeros((1, 5, d))
    V[0, 2, 1] = 1.0
    V[0, 3, 2] = 1.0
    V[0, 0, 3] = V[0, 4, 3] = 1.0
    gap = (2.0 - -2.0) / math.sqrt(d)
    p3 = 1.0 / (1.0 + math.exp(-gap))
    out, _ = o.range_attention(q, K, V, 3, 5)
    assert np.allclose(out[0], [0.0, p3, 1.0 - p3, 0.0], atol=1e-15)


def test_range_empty_rejected():
    with pytest.raises(ValueError):
        o.range_attention(np.zeros((1, 4)), np.zeros((1, 5, 4)), np.zeros((1, 5, 4)), 3, 3)


# --------------------------------------------------------------------------
# selection at a call budget (ODA summary, State-Dependent Access
# Effectiveness; Conclusion: the offline Oracle)
# --------------------------------------------------------------------------

def test_budget_count_closed_forms():
    assert o.budget_count(10, 0.4) == 4
    assert o.budget_count(7, 0.4) == 2             # floor(2.8)
    assert o.budget_count(5, 1) == 5 and o.budget_count(5, 0) == 0
    assert o.budget_count(1000, "0.125") == 125


def test_oracle_selection_is_best_and_random_is_the_subset_mean():
    """Brute force over every k-subset of small gain vectors: selecting by the
    true gain reaches the largest net gain of any k-subset, and the random
    expectation is the mean net gain over all k-subsets."""
    import itertools
    rng = np.random.default_rng(21)
    for n in range(1, 8):
        g = rng.normal(size=n).astype(np.float32)
        for k in range(0, n + 1):
            best = max(sum(float(g[i]) for i in c) for c in itertools.combinations(range(n), k))
            sel = o.select_top(g, k)
            assert sel.sum() == k
            assert abs(o.net_gain_per_position(g, sel) - best / n) < 1e-12
            subsets = list(itertools.combinations(range(n), k))
            mean = np.mean([sum(float(g[i]) for i in c) / n for c in subsets])
            assert abs(o.random_expected_net_gain(g, k) - mean) < 1e-12


def test_selection_worked_example_and_ties():
    g = np.array([3.0, -1.0, 2.0, 0.5, -2.0], np.float32)
    sel = o.select_top(g, 2)
    assert sel.tolist() == [1, 0, 1, 0, 0]
    assert o.net_gain_per_position(g, sel) == 1.0
    assert abs(o.random_expected_net_gain(g, 2) - 0.2) < 1e-15     # 2/5 * 2.5/5
    # equal scores (+0 and -0 included) go to the earlier position
    assert o.select_top(np.array([1.0, 1.0, 1.0, 1.0], np.float32), 2).tolist() == [1, 1, 0, 0]
    assert o.select_top(np.array([-0.0, 0.0, -1.0], np.float32), 1).tolist() == [1, 0, 0]
    assert o.select_top(np.array([0.0, -0.0, -1.0], np.float32), 1).tolist() == [1, 0, 0]
    # NaN below every number, -inf included; NaNs among themselves by position
    s = np.array([np.nan, -np.inf, np.nan, 5.0], np.float32)
    assert o.select_top(s, 2).tolist() == [0, 1, 0, 1]
    assert o.select_top(s, 3).tolist() == [1, 1, 0, 1]
    # the comparison is float32: values equal after rounding tie
    assert o.select_top(np.array([1.0 + 1e-9, 1.0], np.float64), 1).tolist() == [1, 0]
    with pytest.raises(ValueError):
        o.select_top(g, 6)

"""The seeded input generator: published test vectors, rounding, determinism."""

import numpy as np

import synth
from synth import gen


def test_splitmix64_published_sequence():
    # SplitMix64 seeded with 0 outputs E220A8397B1DCDAF, 6E789E6AA1B965F4,
    # 06C45D188009454F: output k is mix64(k * gamma).
    expect = [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]
    for k, e in enumerate(expect):
        assert synth.mix64_int((k * gen.GAMMA) & gen.MASK64) == e
    arr = synth.mix64(np.array([(k * gen.GAMMA) & gen.MASK64 for k in range(3)], np.uint64))
    assert [int(x) for x in arr] == expect


def test_bf16_round_to_nearest_even():
    one = np.float32(1.0)
    ulp = np.float32(2.0 ** -7)
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 0.0, -0.0, np.inf, np.nan],
                 np.float32)
    b = synth.f32_to_bf16_bits(x)
    assert b[0] == 0x3F80
    assert b[1] == 0x3F80          # tie -> even
    assert b[2] == 0x3F82          # tie -> even (up)
    assert b[3] == 0xC020
    assert b[4] == 0x0000 and b[5] == 0x8000 and b[6] == 0x7F80
    assert np.isnan(synth.bf16_bits_to_f32(b[7:8]))[0]
    back = synth.bf16_bits_to_f32(b[:4])
    assert back[0] == one and back[2] == one + 2 * ulp


def test_tables_are_quantiles():
    t = synth.normal_table(1.0, "f32")
    assert t.shape == (65536,) and np.all(np.diff(t) > 0)
    assert abs(float(t.mean())) < 1e-6 and abs(float(t.std()) - 1.0) < 2e-3
    tb = synth.bf16_bits_to_f32(synth.normal_table(0.5, "bf16"))
    assert abs(float(tb.std()) - 0.5) < 2e-3
    u = synth.uniform_table(0.25, "f32")
    assert u.min() > -0.25 and u.max() < 0.25 and np.all(np.diff(u) > 0)


def test_values_independent_of_shapes():
    tab = synth.normal_table(1.0, "f32")
    key = synth.stream_key(5, synth.KIND_KV, 0, 1, 2, 0)
    a = synth.table_values(key, 0, 1000, tab)
    b = synth.table_values(key, 300, 200, tab)
    assert np.array_equal(a[300:500], b)
    f = synth.fill_streams([key, key + 1], [0, 7], 3, 10, tab)
    assert np.array_equal(f[:, 0, :].reshape(-1), a[:30])
    assert np.array_equal(f[1, 1], synth.table_values(key + 1, 17, 10, tab))


def test_workload_recipes():
    w = synth.tiny_fp32()
    assert w.group == 2 and len(w.needles) == 2
    for n in w.needles:
        assert w.sink < n.position <= int(w.t0[n.row]) - w.window
        q = w.q_step(5)[n.layer, n.row, n.q_head]
        assert abs(w.to_f64(q) @ w.to_f64(n.key) - 8.0) < 1e-4
    tb, nb = w.paging()
    used = tb[tb >= 0]
    assert sorted(used.tolist()) == list(range(nb))
    c3 = synth.ctx128k()
    f = c3.flags()
    assert f.shape == (1024, 1) and 0.10 < f.mean() < 0.15
    m = synth.mixed_batch(0.41)
    assert m.t0.min() >= 4096 and m.t0.max() <= 65536
    k_new, v_new = w.kv_new_step(3)
    hist = w.kv_history(0, 1, 0, 0, int(w.t0[1]) + 3)
    assert np.array_equal(k_new[0, 1, 0], hist[-1])

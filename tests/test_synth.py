"""Host-side checks of the seeded input generators (no GPU)."""
import math

import numpy as np

import synth


def test_counter_stream_slices_are_consistent():
    a = synth.normal(5, 3, 0, 1000)
    b = synth.normal(5, 3, 400, 100)
    np.testing.assert_array_equal(a[400:500], b)
    assert not np.array_equal(synth.normal(5, 4, 0, 10), a[:10])
    assert not np.array_equal(synth.normal(6, 3, 0, 10), a[:10])


def test_splitmix64_reference_value():
    # splitmix64 seeded with 0: first output of the published generator is
    # mix(0 + gamma) = 0xE220A8397B1DCDAF
    z = np.array([0x9E3779B97F4A7C15], dtype=np.uint64)
    assert int(synth._mix64(z)[0]) == 0xE220A8397B1DCDAF


def test_normal_moments():
    x = synth.normal(1, 0, 0, 200000)
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1) < 0.01
    u = synth.uniform(1, 0, 0, 100000)
    assert u.min() > 0 and u.max() < 1 and abs(u.mean() - 0.5) < 0.005


def test_bf16_rounding_is_round_to_nearest_even():
    # bf16 keeps 7 explicit mantissa bits: 1+2^-7 is exact; 1+2^-8 is a tie
    # between 1 and 1+2^-7 -> even (1.0); 1+3*2^-8 is a tie between 1+2^-7
    # (odd) and 1+2^-6 (even) -> 1+2^-6; 1+2^-9 rounds down
    vals = np.array([1.0 + 2 ** -7, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9, -2.5, 3.0e38], np.float32)
    r = synth.bf16_bits_to_f32(synth.round_to_bf16_bits(vals))
    np.testing.assert_array_equal(r[:5], np.array([1.0 + 2 ** -7, 1.0, 1.0 + 2 ** -6, 1.0, -2.5], np.float32))
    assert math.isfinite(r[5])


def test_workload_rows_regenerate_independently():
    w = synth.workload(1)
    rows = [0, 5, w.channels - 1]
    v_part = synth.v_rows(w, rows)
    v_one = synth.v_rows(w, [5])
    np.testing.assert_array_equal(v_part[1], v_one[0])
    # bf16 workload: values are exactly representable in bf16
    bits = synth.round_to_bf16_bits(v_part)
    np.testing.assert_array_equal(synth.bf16_bits_to_f32(bits), v_part)


def test_onehot_and_sigmoid_inputs():
    w4 = synth.custom(2, "bf16", 2, 8, 64, v_kind="onehot4")
    v = synth.v_rows(w4)
    # per time step, channels take the values of one row of the 4 x D table
    table = synth.normal(w4.seed, synth.TID_EMBED, 0, 4 * 8).reshape(4, 8)
    tb = synth.bf16_bits_to_f32(synth.round_to_bf16_bits(table.astype(np.float32)))
    for b in range(2):
        for t in range(64):
            col = v[b * 8:(b + 1) * 8, t]
            assert any(np.array_equal(col, tb[s]) for s in range(4))
    w3 = synth.custom(2, "bf16", 1, 4, 128, x_kind="sigmoid_normal")
    x = synth.x_rows(w3, 1)
    assert (x > 0).all() and (x < 1).all()


def test_weights_ranges_and_roofline_bytes():
    w = synth.workload(2)
    wt = synth.filter_weights(w)
    assert wt["W1"].shape == (64, 17) and wt["W3"].shape == (3 * 1024, 64)
    assert np.abs(wt["W1"]).max() <= 1 / math.sqrt(17)
    assert np.abs(wt["W2"]).max() <= 1 / math.sqrt(64)
    assert w.roofline_bytes() == 369_123_328
    assert synth.workload(1).roofline_bytes() == 75_509_760
    assert synth.workload(4).roofline_bytes() == 6_442_455_040


def test_sample_rows():
    w = synth.workload(2)
    s = synth.sample_rows(w, 10)
    assert len(s) == 10 and s[0] == 0 and s[-1] == w.channels - 1
    assert s == synth.sample_rows(w, 10)


def test_nd_workloads_and_kernels():
    for w in synth.ND_WORKLOADS:
        assert w.grid == int(np.prod(w.dims))
        assert w.padded == int(np.prod([2 * d if w.boundary == "zero" else d for d in w.dims]))
        assert w.padded <= 16384                      # one on-chip grid per (channel, pair)
        assert w.roofline_bytes() == ((w.N + 2) * w.B * w.D * w.grid * w.elem_bytes
                                      + w.N * w.D * w.padded * 8)
    w = synth.nd_custom(2, "f32", 2, 3, (4, 8), "circular", seed=9)
    K1, K2 = synth.nd_kernels(w), synth.nd_kernels(w)
    assert K1.shape == (2, 3, 32) and K1.dtype == np.float32
    np.testing.assert_array_equal(K1, K2)             # seeded, reproducible
    # the window peaks at offset 0 and, on a circular grid, is symmetric in the periodic distance
    Kz = synth.nd_kernels(synth.nd_custom(1, "f32", 1, 1, (16,), "circular", seed=1))[0, 0]
    g = synth.normal(1, 500, 0, 16)
    win = Kz / g
    np.testing.assert_allclose(win[1:], win[1:][::-1], rtol=1e-5)
    assert np.argmax(win) == 0
    np.testing.assert_allclose(np.linalg.norm(win), 1.0, rtol=1e-5)
    v, xs = synth.nd_inputs(w)
    assert v.shape == (6, 32) and len(xs) == 2

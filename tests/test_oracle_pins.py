"""Pins of the float64 oracle to things other than itself.

Each check ties a part of the oracle to an independent fact: a brute-force
definition evaluated a different way, a library routine computing the same
quantity by another algorithm, a closed form, or an invariant of the method
(causality, linearity, shift-equivariance, commutativity). They are chosen
so that a dropped term, a wrong sign or index, or a transposed operand in the
oracle fails at least one of them. No GPU is used.
"""
import math

import numpy as np
import pytest

import oracle


rng = np.random.default_rng(12345)


# ---------------------------------------------------------------- FFT ------

@pytest.mark.parametrize("n", [1, 2, 4, 8, 16, 32, 64])
def test_fft_matches_bruteforce_dft(n):
    x = rng.standard_normal(n) + 1j * rng.standard_normal(n)
    # O(n^2) definition, one term at a time
    ref = np.zeros(n, dtype=complex)
    for k in range(n):
        for j in range(n):
            ref[k] += x[j] * complex(math.cos(-2 * math.pi * j * k / n), math.sin(-2 * math.pi * j * k / n))
    np.testing.assert_allclose(oracle.fft(x, -1), ref, rtol=0, atol=1e-12 * n)
    ref_inv = np.conj(oracle.fft(np.conj(x), -1))
    np.testing.assert_allclose(oracle.fft(x, +1), ref_inv, rtol=0, atol=1e-12 * n)


@pytest.mark.parametrize("n", [1024, 1 << 16])
def test_fft_matches_numpy(n):
    x = rng.standard_normal(n) + 1j * rng.standard_normal(n)
    X = oracle.fft(x)
    ref = np.fft.fft(x)
    assert np.linalg.norm(X - ref) / np.linalg.norm(ref) < 1e-13
    # inverse round trip and Parseval
    back = oracle.fft(X, +1) / n
    assert np.abs(back - x).max() < 1e-12
    assert abs(np.vdot(X, X).real / n - np.vdot(x, x).real) / np.vdot(x, x).real < 1e-12


# ------------------------------------------------------------- causal conv ---

@pytest.mark.parametrize("L", [1, 2, 3, 5, 7, 64, 1000])
def test_direct_conv_matches_numpy_convolve(L):
    h, z = rng.standard_normal(L), rng.standard_normal(L)
    ref = np.convolve(h, z)[:L]
    np.testing.assert_allclose(oracle.causal_conv(h, z, "direct"), ref, rtol=0, atol=1e-11 * L)


@pytest.mark.parametrize("L", [1, 2, 4, 8, 16, 32, 64, 1024, 8192])
def test_fft_conv_matches_direct_conv(L):
    h, z = rng.standard_normal(L), rng.standard_normal(L)
    a = oracle.causal_conv(h, z, "direct")
    b = oracle.causal_conv(h, z, "fft")
    assert np.abs(a - b).max() <= 1e-11 * math.sqrt(L) * max(1.0, np.abs(a).max())


def test_auto_branch_switches_at_8192():
    # above the direct limit the oracle uses the FFT branch; check it against a
    # direct evaluation of the definition at one size past the switch
    L = 16384
    h = rng.standard_normal(L) * np.exp(-np.arange(L) / 3000.0)
    z = rng.standard_normal(L)
    auto = oracle.causal_conv(h, z)
    direct = oracle.causal_conv(h, z, "direct")
    assert np.abs(auto - direct).max() / np.abs(direct).max() < 1e-12


def test_delta_filter_returns_input():
    L = 257
    z = rng.standard_normal(L)
    h = np.zeros(L); h[0] = 1.0
    np.testing.assert_array_equal(oracle.causal_conv(h, z, "direct"), z)
    L = 4096
    z = rng.standard_normal(L)
    h = np.zeros(L); h[0] = 1.0
    np.testing.assert_allclose(oracle.causal_conv(h, z, "fft"), z, atol=1e-12)


def test_delta_input_returns_filter():
    for L, m in [(300, "direct"), (2048, "fft")]:
        h = rng.standard_normal(L)
        z = np.zeros(L); z[0] = 1.0
        np.testing.assert_allclose(oracle.causal_conv(h, z, m), h, atol=1e-12)


@pytest.mark.parametrize("L,method", [(64, "direct"), (5000, "direct"), (16384, "fft")])
def test_exponential_filter_matches_recurrence(L, method):
    # h_t = R lambda^t (lag t, 0-based) <=> y_t = lambda y_{t-1} + R z_t, y_{-1} = 0
    R, lam = 0.7, 0.9993
    h = R * lam ** np.arange(L)
    z = rng.standard_normal(L)
    y = np.empty(L)
    prev = 0.0
    for t in range(L):
        prev = lam * prev + R * z[t]
        y[t] = prev
    got = oracle.causal_conv(h, z, method)
    assert np.abs(got - y).max() <= 1e-9 * max(1.0, np.abs(y).max())


def test_conv_is_causal_and_bilinear():
    L = 512
    h, z1, z2 = rng.standard_normal(L), rng.standard_normal(L), rng.standard_normal(L)
    a, b = 1.75, -0.375
    f = lambda hh, zz: oracle.causal_conv(hh, zz, "direct")
    np.testing.assert_allclose(f(h, a * z1 + b * z2), a * f(h, z1) + b * f(h, z2), atol=1e-10)
    np.testing.assert_allclose(f(a * h + b * z2, z1), a * f(h, z1) + b * f(z2, z1), atol=1e-10)
    t0 = 200
    zp = z1.copy(); zp[t0] += 10.0
    np.testing.assert_array_equal(f(h, zp)[:t0], f(h, z1)[:t0])
    assert np.abs(f(h, zp)[t0:] - f(h, z1)[t0:]).max() > 1.0


# --------------------------------------------------------- recurrence -------

def _rand_hyena(C, L, N, decay=0.01):
    v = rng.standard_normal((C, L))
    xs = [rng.standard_normal((C, L)) for _ in range(N)]
    hs = [rng.standard_normal((C, L)) * np.exp(-decay * np.arange(L)) for _ in range(N)]
    return v, xs, hs


def test_recurrence_delta_filters_give_product_of_gates():
    C, L, N = 3, 128, 3
    v, xs, _ = _rand_hyena(C, L, N)
    delta = np.zeros((C, L)); delta[:, 0] = 1.0
    y = oracle.hyena_forward(v, xs, [delta] * N)
    np.testing.assert_allclose(y, v * xs[0] * xs[1] * xs[2], rtol=1e-14, atol=0)


def test_recurrence_order_and_gate_placement():
    # z2 = x1 * (h1 conv v); z3 = x2 * (h2 conv z2) -- written out with numpy
    # convolve so that a gate applied before the convolution, or the filters
    # used in the other order, fails
    C, L, N = 2, 200, 2
    v, xs, hs = _rand_hyena(C, L, N)
    y = oracle.hyena_forward(v, xs, hs)
    for r in range(C):
        z2 = xs[0][r] * np.convolve(hs[0][r], v[r])[:L]
        z3 = xs[1][r] * np.convolve(hs[1][r], z2)[:L]
        np.testing.assert_allclose(y[r], z3, rtol=1e-10, atol=1e-10 * np.abs(z3).max())


def test_recurrence_delta_input_unit_gates_gives_filter_product():
    L = 256
    v = np.zeros((1, L)); v[0, 0] = 1.0
    ones = np.ones((1, L))
    h1 = rng.standard_normal((1, L)); h2 = rng.standard_normal((1, L))
    y1 = oracle.hyena_forward(v, [ones], [h1])
    np.testing.assert_allclose(y1, h1, atol=1e-13)
    y2 = oracle.hyena_forward(v, [ones, ones], [h1, h2])
    np.testing.assert_allclose(y2[0], np.convolve(h1[0], h2[0])[:L], atol=1e-11)


def test_recurrence_commutes_and_shifts_with_unit_gates():
    C, L = 2, 1024
    v, _, hs = _rand_hyena(C, L, 2, decay=0.003)
    ones = [np.ones((C, L))] * 2
    y = oracle.hyena_forward(v, ones, hs)
    y_sw = oracle.hyena_forward(v, ones, hs[::-1])
    assert np.abs(y - y_sw).max() <= 1e-11 * np.abs(y).max()
    s = 37
    vs = np.zeros_like(v); vs[:, s:] = v[:, :-s]
    ys = oracle.hyena_forward(vs, ones, hs)
    assert np.abs(ys[:, s:] - y[:, :-s]).max() <= 1e-11 * np.abs(y).max()
    assert np.abs(ys[:, :s]).max() == 0.0


def test_recurrence_linear_in_v():
    C, L, N = 2, 300, 3
    v1, xs, hs = _rand_hyena(C, L, N)
    v2 = rng.standard_normal((C, L))
    a, b = -2.5, 0.625
    y = oracle.hyena_forward(a * v1 + b * v2, xs, hs)
    ref = a * oracle.hyena_forward(v1, xs, hs) + b * oracle.hyena_forward(v2, xs, hs)
    assert np.abs(y - ref).max() <= 1e-10 * np.abs(ref).max()


def test_recurrence_filter_row_mapping():
    # channel r uses filter row filter_row[r]
    C, L = 4, 64
    v, xs, _ = _rand_hyena(C, L, 1)
    hs = [rng.standard_normal((2, L))]
    fr = np.array([1, 0, 1, 1])
    y = oracle.hyena_forward(v, xs, hs, filter_row=fr)
    for r in range(C):
        ref = xs[0][r] * np.convolve(hs[0][fr[r]], v[r])[:L]
        np.testing.assert_allclose(y[r], ref, atol=1e-12)


def test_recurrence_fft_branch_matches_direct_branch_large_L():
    # L = 16384 takes the FFT branch inside the recurrence; compare with the
    # direct causal sum chained by hand
    L = 16384
    v, xs, hs = _rand_hyena(1, L, 2, decay=0.0005)
    y = oracle.hyena_forward(v, xs, hs)
    z = v[0]
    for n in range(2):
        z = xs[n][0] * oracle.causal_conv(hs[n][0], z, "direct")
    assert np.abs(y[0] - z).max() <= 1e-11 * np.abs(z).max()


# ---------------------------------------------------------- spectrum --------

@pytest.mark.parametrize("L", [16, 64, 8192, 16384])
def test_spectrum_closed_forms(L):
    k = np.arange(L + 1)
    w = np.exp(-1j * np.pi * k / L)            # exp(-2 pi i k / 2L)
    d0 = np.zeros(L); d0[0] = 1.0
    np.testing.assert_allclose(oracle.filter_spectrum(d0), np.ones(L + 1), atol=1e-12)
    d1 = np.zeros(L); d1[1] = 1.0
    np.testing.assert_allclose(oracle.filter_spectrum(d1), w, atol=1e-12)
    R, lam = 1.3, 0.97
    h = R * lam ** np.arange(L)
    geo = R * (1 - (lam * w) ** L) / (1 - lam * w)
    np.testing.assert_allclose(oracle.filter_spectrum(h), geo, rtol=1e-11, atol=1e-11)


@pytest.mark.parametrize("L", [32, 1024, 16384])
def test_spectrum_matches_numpy_rfft(L):
    h = rng.standard_normal(L)
    ref = np.fft.rfft(np.concatenate([h, np.zeros(L)]))
    got = oracle.filter_spectrum(h)
    assert np.linalg.norm(got - ref) / np.linalg.norm(ref) < 1e-12


# ------------------------------------------------------ implicit filter -----

def test_embedding_closed_forms():
    L = 1024
    e0 = oracle.embedding(0, L)
    np.testing.assert_array_equal(e0, np.concatenate([[0.0], np.zeros(8), np.ones(8)]))
    e = oracle.embedding(L // 4, L)
    k = np.arange(1, 9)
    np.testing.assert_allclose(e, np.concatenate([[0.25], np.sin(np.pi * k / 2), np.cos(np.pi * k / 2)]),
                               atol=1e-15)
    e = oracle.embedding(3, 8, n_bands=2)
    np.testing.assert_allclose(e, [3 / 8, math.sin(2 * math.pi * 3 / 8), math.sin(2 * math.pi * 6 / 8),
                                   math.cos(2 * math.pi * 3 / 8), math.cos(2 * math.pi * 6 / 8)], atol=1e-15)


def test_alpha_spacing():
    assert oracle.alpha(0, 5, 0.5, 20.0) == 0.5
    assert oracle.alpha(4, 5, 0.5, 20.0) == 20.0
    assert abs(oracle.alpha(2, 5, 0.5, 20.0) - 10.25) < 1e-15
    assert oracle.alpha(0, 1, 0.1, 10.0) == 0.1


def _zero_weights(N, D, H=64, E=17):
    return {"W1": np.zeros((H, E), np.float32), "b1": np.zeros(H, np.float32),
            "W2": np.zeros((H, H), np.float32), "b2": np.zeros(H, np.float32),
            "W3": np.zeros((N * D, H), np.float32), "b3": np.zeros(N * D, np.float32)}


def test_filter_constant_hidden_state_closed_form():
    # W1 = W2 = 0, b2 = pi/2  =>  s2 = 1  =>  h_n[c][t] = (sum_j W3[o][j] + b3[o]) exp(-alpha_c t/L)
    N, D, L, lo, hi = 2, 5, 64, 0.5, 20.0
    w = _zero_weights(N, D)
    w["b2"][:] = np.float32(math.pi / 2)
    w["W3"] = rng.uniform(-1, 1, (N * D, 64)).astype(np.float32)
    w["b3"] = rng.uniform(-1, 1, N * D).astype(np.float32)
    h = oracle.implicit_filter(w, N, D, L, lo, hi)
    s2 = math.sin(float(np.float32(math.pi / 2)))
    t = np.arange(L)
    for n in range(N):
        for c in range(D):
            o = n * D + c
            amp = w["W3"][o].astype(np.float64).sum() * s2 + float(w["b3"][o])
            alpha = lo + (hi - lo) * c / (D - 1)
            np.testing.assert_allclose(h[o], amp * np.exp(-alpha * t / L), rtol=1e-13, atol=1e-15)


def test_filter_selected_embedding_closed_form():
    # hidden unit j reads embedding dim i_j with weight a_j; layer 2 unit m
    # copies hidden unit j_m; output o reads layer-2 unit m_o.
    # => h = sin(sin(a_j e_i(t) + b1_j) + b2_m) * W3 + b3, times the window
    N, D, L, lo, hi, H = 3, 2, 128, 0.25, 4.0, 64
    w = _zero_weights(N, D)
    picks = [(0, 1.3, 0.1), (1, 0.7, -0.2), (8, 1.1, 0.0), (9, 0.9, 0.3), (16, 1.7, 0.05), (5, -0.8, 0.4)]
    for j, (i, a, b) in enumerate(picks):
        w["W1"][j, i] = a
        w["b1"][j] = b
    b2 = np.float32(0.15)
    for m in range(6):
        w["W2"][10 + m, 5 - m] = 1.0     # layer-2 unit 10+m copies hidden unit 5-m
        w["b2"][10 + m] = b2
    scale = np.float32(1.5)
    for o in range(N * D):
        w["W3"][o, 10 + o] = scale
        w["b3"][o] = np.float32(0.01 * o)
    h = oracle.implicit_filter(w, N, D, L, lo, hi)
    t = np.arange(L)
    emb = np.stack([oracle.embedding(tt, L) for tt in t])          # pinned above
    k = np.arange(1, 9)
    np.testing.assert_allclose(emb[:, 0], t / L, atol=1e-15)
    np.testing.assert_allclose(emb[:, 1:9], np.sin(2 * np.pi * np.outer(t, k) / L), atol=1e-12)
    np.testing.assert_allclose(emb[:, 9:], np.cos(2 * np.pi * np.outer(t, k) / L), atol=1e-12)
    for o in range(N * D):
        n, c = divmod(o, D)
        j = 5 - o
        i, a, b = picks[j]
        a32, b32 = float(np.float32(a)), float(np.float32(b))
        s1 = np.sin(a32 * emb[:, i] + b32)
        s2 = np.sin(s1 + float(b2))
        alpha = lo + (hi - lo) * c / (D - 1)
        ref = (float(scale) * s2 + float(np.float32(0.01 * o))) * np.exp(-alpha * t / L)
        np.testing.assert_allclose(h[o], ref, rtol=1e-12, atol=1e-14)


def test_filter_row_selection_matches_full():
    import synth
    w = synth.custom(2, "f32", 1, 6, 256)
    wt = synth.filter_weights(w)
    full = oracle.implicit_filter(wt, 2, 6, 256, 0.5, 20.0)
    rows = [(1, 5), (0, 0), (1, 2)]
    part = oracle.implicit_filter(wt, 2, 6, 256, 0.5, 20.0, rows=rows)
    for i, (n, c) in enumerate(rows):
        np.testing.assert_array_equal(part[i], full[n * 6 + c])
    # window at t = 0 is 1 and the window is monotone: |h| / |FFN| decays
    assert np.isfinite(full).all()

"""Property-based pins of the oracle (hypothesis, CPU): random small shapes
and values checked against brute-force sums written independently of the
oracle's code paths, and against identities of the operator (causal
convolution, order-N recurrence, ND convolution) that hold for every input.
"""
import itertools

import numpy as np
import pytest
from hypothesis import given, settings, strategies as st

import oracle

SETTINGS = settings(max_examples=40, deadline=None)


def brute_causal(h, z):
    L = len(z)
    return np.array([sum(h[t - s] * z[s] for s in range(t + 1)) for t in range(L)])


@st.composite
def rows(draw, max_len=48):
    L = draw(st.integers(1, max_len))
    seed = draw(st.integers(0, 2**31 - 1))
    rng = np.random.default_rng(seed)
    return rng.standard_normal(L), rng.standard_normal(L)


@SETTINGS
@given(rows())
def test_causal_conv_is_the_causal_sum(hz):
    h, z = hz
    np.testing.assert_allclose(oracle.causal_conv(h, z), brute_causal(h, z), rtol=1e-10, atol=1e-10)


@SETTINGS
@given(rows(), st.integers(0, 47))
def test_causal_conv_commutes_with_delay(hz, d):
    # delaying the input by d delays the output by d (zeros enter at the front)
    h, z = hz
    L = len(z)
    d = min(d, L)
    zd = np.concatenate([np.zeros(d), z[:L - d]])
    y, yd = oracle.causal_conv(h, z), oracle.causal_conv(h, zd)
    np.testing.assert_allclose(yd[d:], y[:L - d], rtol=1e-10, atol=1e-10)
    np.testing.assert_allclose(yd[:d], 0.0, atol=1e-12)


@SETTINGS
@given(st.integers(1, 4), st.integers(1, 3), st.integers(2, 40), st.integers(0, 2**31 - 1))
def test_recurrence_is_the_written_recurrence(N, C, L, seed):
    rng = np.random.default_rng(seed)
    v = rng.standard_normal((C, L))
    xs = [rng.standard_normal((C, L)) for _ in range(N)]
    hs = [rng.standard_normal((C, L)) for _ in range(N)]
    got = oracle.hyena_forward(v, xs, hs)
    for c in range(C):
        z = v[c]
        for n in range(N):
            z = xs[n][c] * brute_causal(hs[n][c], z)
        np.testing.assert_allclose(got[c], z, rtol=1e-9, atol=1e-9)


@SETTINGS
@given(st.lists(st.sampled_from([1, 2, 3, 4, 6]), min_size=1, max_size=3),
       st.sampled_from(["zero", "circular"]), st.integers(0, 2**31 - 1))
def test_nd_conv_is_the_nd_sum(dims, boundary, seed):
    dims = tuple(dims)
    rng = np.random.default_rng(seed)
    K, z = rng.standard_normal(dims), rng.standard_normal(dims)
    want = np.zeros(dims)
    for p in itertools.product(*(range(d) for d in dims)):
        acc = 0.0
        for q in itertools.product(*(range(d) for d in dims)):
            off = tuple(a - b for a, b in zip(p, q))
            if boundary == "circular":
                off = tuple(o % d for o, d in zip(off, dims))
            elif min(off) < 0:
                continue
            acc += K[off] * z[q]
        want[p] = acc
    np.testing.assert_allclose(oracle.nd_conv(K, z, boundary), want, rtol=1e-9, atol=1e-9)


@SETTINGS
@given(st.sampled_from([(8,), (4, 8), (2, 4, 4)]), st.integers(0, 2**31 - 1))
def test_circular_nd_conv_is_shift_equivariant(dims, seed):
    rng = np.random.default_rng(seed)
    K, z = rng.standard_normal(dims), rng.standard_normal(dims)
    shift = tuple(int(s) for s in rng.integers(0, dims))
    axes = tuple(range(len(dims)))
    a = oracle.nd_conv(K, np.roll(z, shift, axis=axes), "circular")
    b = np.roll(oracle.nd_conv(K, z, "circular"), shift, axis=axes)
    np.testing.assert_allclose(a, b, rtol=1e-9, atol=1e-9)


@SETTINGS
@given(st.integers(1, 8), st.integers(1, 12), st.integers(8, 64), st.integers(0, 2**31 - 1))
def test_striped_operator_is_the_written_fir_composition(lf, lg, L, seed):
    rng = np.random.default_rng(seed)
    xq, xk, xv = (rng.standard_normal((1, L)) for _ in range(3))
    hT, hH, hK = (rng.standard_normal((1, lf)) for _ in range(3))
    hG = rng.standard_normal((1, lg))

    def fir(h, x):
        return np.array([sum(h[j] * x[t - j] for j in range(len(h)) if t - j >= 0) for t in range(L)])

    want = fir(hT[0], xq[0]) * fir(hG[0], fir(hH[0], xk[0]) * fir(hK[0], xv[0]))
    got = oracle.striped_forward(xq, xk, xv, hT, hH, hK, hG)[0]
    np.testing.assert_allclose(got, want, rtol=1e-9, atol=1e-9)

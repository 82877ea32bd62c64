"""Pins of the HyenaND oracle (ND convolution, circular or zero-padded
boundary; page "Native Multi-Dimensional Subquadratic Operators via Input
Dependent Long Convolutions", section 手法) to results fixed independently of
its FFT evaluation: brute-force sums on tiny grids, delta and shifted-delta
kernels, separable kernels against the 1D causal sum of the C oracle, the
1D case against the 1D order-N oracle, and the no-wrap equivalence of the
two boundaries."""
import itertools

import numpy as np
import pytest

import oracle


def brute(K, z, boundary):
    dims = z.shape
    y = np.zeros(dims)
    for p in itertools.product(*(range(d) for d in dims)):
        acc = 0.0
        for q in itertools.product(*(range(d) for d in dims)):
            off = tuple(a - b for a, b in zip(p, q))
            if boundary == "circular":
                off = tuple(o % d for o, d in zip(off, dims))
            elif any(o < 0 for o in off):
                continue
            acc += K[off] * z[q]
        y[p] = acc
    return y


@pytest.mark.parametrize("dims", [(4, 8), (8, 2), (2, 4, 4), (3, 5), (1, 6)])
@pytest.mark.parametrize("boundary", ["zero", "circular"])
def test_matches_brute_force(dims, boundary):
    rng = np.random.default_rng(sum(dims) * 7 + len(dims))
    K, z = rng.standard_normal(dims), rng.standard_normal(dims)
    np.testing.assert_allclose(oracle.nd_conv(K, z, boundary), brute(K, z, boundary), rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("boundary", ["zero", "circular"])
def test_delta_and_shifted_delta(boundary):
    rng = np.random.default_rng(3)
    dims = (8, 16, 4)
    z = rng.standard_normal(dims)
    K = np.zeros(dims); K[0, 0, 0] = 1.0
    np.testing.assert_allclose(oracle.nd_conv(K, z, boundary), z, atol=1e-12)
    o = (3, 5, 1)
    K = np.zeros(dims); K[o] = 1.0
    got = oracle.nd_conv(K, z, boundary)
    if boundary == "circular":
        want = np.roll(z, o, axis=(0, 1, 2))
    else:
        want = np.zeros(dims)
        want[o[0]:, o[1]:, o[2]:] = z[:dims[0] - o[0], :dims[1] - o[1], :dims[2] - o[2]]
    np.testing.assert_allclose(got, want, atol=1e-12)


def test_separable_kernel_is_two_causal_sums():
    # K = a (outer) b: the zero-padded 2D convolution is the 1D causal sum of
    # the C oracle along each axis in turn
    rng = np.random.default_rng(5)
    H, W = 16, 32
    a, b = rng.standard_normal(H), rng.standard_normal(W)
    z = rng.standard_normal((H, W))
    rows = np.stack([oracle.causal_conv(b, z[i]) for i in range(H)])
    want = np.stack([oracle.causal_conv(a, rows[:, j]) for j in range(W)], axis=1)
    np.testing.assert_allclose(oracle.nd_conv(np.outer(a, b), z, "zero"), want, rtol=1e-10, atol=1e-10)


def test_one_dimensional_case_is_the_order_n_forward():
    rng = np.random.default_rng(9)
    C, L, N = 3, 64, 3
    v = rng.standard_normal((C, L))
    xs = [rng.standard_normal((C, L)) for _ in range(N)]
    hs = [rng.standard_normal((C, L)) * np.exp(-np.arange(L) / 16) for _ in range(N)]
    want = oracle.hyena_forward(v, xs, hs)
    got = oracle.hyena_nd_forward(v, xs, hs, (L,), "zero")
    np.testing.assert_allclose(got, want, rtol=1e-10, atol=1e-10)


def test_boundaries_agree_without_wrap():
    # kernel and signal inside the first half of every axis: nothing wraps
    rng = np.random.default_rng(11)
    dims = (16, 8)
    K, z = np.zeros(dims), np.zeros(dims)
    K[:8, :4] = rng.standard_normal((8, 4))
    z[:8, :4] = rng.standard_normal((8, 4))
    np.testing.assert_allclose(oracle.nd_conv(K, z, "circular"), oracle.nd_conv(K, z, "zero"), atol=1e-12)


def test_circular_wraps_where_zero_padding_does_not():
    dims = (4, 4)
    K = np.zeros(dims); K[0, 1] = 1.0
    z = np.zeros(dims); z[2, 3] = 1.0
    assert oracle.nd_conv(K, z, "circular")[2, 0] == pytest.approx(1.0)
    assert abs(oracle.nd_conv(K, z, "zero")).max() < 1e-12


def test_order_n_recurrence_on_rows_and_filter_rows():
    rng = np.random.default_rng(13)
    dims = (4, 8)
    P = 32
    v = rng.standard_normal((4, P))
    xs = [rng.standard_normal((4, P)) for _ in range(2)]
    Ks = [rng.standard_normal((2, P)) for _ in range(2)]
    fr = [0, 1, 0, 1]
    got = oracle.hyena_nd_forward(v, xs, Ks, dims, "circular", filter_row=fr)
    for r in range(4):
        z = v[r].reshape(dims)
        for n in range(2):
            z = xs[n][r].reshape(dims) * brute(Ks[n][fr[r]].reshape(dims), z, "circular")
        np.testing.assert_allclose(got[r], z.reshape(-1), rtol=1e-10, atol=1e-10)

"""Pins of the float64 backward oracle to things other than itself.

The pages print no backward formulas, so the backward is pinned to the
(already pinned) forward oracle and to numpy:
- the adjoint of the causal sum is the transpose of its Toeplitz matrix,
  built column by column with numpy.convolve;
- the forward is linear in v, in each x_n and in each h_n separately, so for
  any direction d the gradient satisfies <grad, d> = <dy, y(input <- d)>
  exactly (a dropped term, a wrong index or a transposed operand breaks it);
- closed forms for a delta filter;
- the filter-weight gradients against Richardson-extrapolated central
  differences of the forward filter oracle, with perturbations that are exact
  in float32 (the oracle takes float32 weights), and a closed form for b3.
No GPU is used.
"""
import numpy as np
import pytest

import oracle

rng = np.random.default_rng(2024)


def toeplitz_causal(h):
    """T[t][s] = h[t-s] for s <= t, built from numpy.convolve of unit vectors."""
    L = len(h)
    T = np.zeros((L, L))
    for s in range(L):
        e = np.zeros(L)
        e[s] = 1.0
        T[:, s] = np.convolve(h, e)[:L]
    return T


@pytest.mark.parametrize("L", [1, 2, 3, 7, 16, 33])
def test_corr_is_transpose_of_causal_sum(L):
    h, r = rng.standard_normal(L), rng.standard_normal(L)
    ref = toeplitz_causal(h).T @ r
    np.testing.assert_allclose(oracle.causal_corr(h, r, "direct"), ref, rtol=0, atol=1e-12 * max(L, 1))


@pytest.mark.parametrize("L", [1, 2, 5, 16, 40])
def test_xcorr_is_filter_gradient_of_causal_sum(L):
    # conv(h, z) = T_z h with T_z[t][j] = z[t-j]; d<r, T_z h>/dh = T_z^T r
    r, z = rng.standard_normal(L), rng.standard_normal(L)
    ref = toeplitz_causal(z).T @ r
    np.testing.assert_allclose(oracle.causal_xcorr(r, z, "direct"), ref, rtol=0, atol=1e-12 * max(L, 1))


@pytest.mark.parametrize("L", [1, 2, 8, 64, 1024, 8192, 16384])
def test_corr_fft_branches_match_direct(L):
    h, r, z = rng.standard_normal(L), rng.standard_normal(L), rng.standard_normal(L)
    a = oracle.causal_corr(h, r, "direct")
    b = oracle.causal_corr(h, r, "fft")
    assert np.abs(a - b).max() <= 1e-11 * np.abs(a).max() + 1e-14
    a = oracle.causal_xcorr(r, z, "direct")
    b = oracle.causal_xcorr(r, z, "fft")
    assert np.abs(a - b).max() <= 1e-11 * np.abs(a).max() + 1e-14


def _problem(C, F, L, N, seed):
    g = np.random.default_rng(seed)
    v = g.standard_normal((C, L))
    xs = [g.standard_normal((C, L)) for _ in range(N)]
    decay = np.exp(-0.05 * np.arange(L))
    hs = [g.standard_normal((F, L)) * decay for _ in range(N)]
    fr = g.integers(0, F, C).astype(np.int32)
    fr[:F] = np.arange(F)                       # every filter row used at least once
    dy = g.standard_normal((C, L))
    return v, xs, hs, fr, dy


@pytest.mark.parametrize("C,F,L,N", [(1, 1, 16, 1), (3, 2, 32, 2), (4, 2, 64, 3), (2, 2, 128, 4)])
def test_adjoint_identities_against_forward(C, F, L, N):
    v, xs, hs, fr, dy = _problem(C, F, L, N, seed=C * 100 + L + N)
    dv, dx, dh = oracle.hyena_backward(v, xs, hs, dy, filter_row=fr)

    def fwd(v_, xs_, hs_):
        return oracle.hyena_forward(v_, xs_, hs_, filter_row=fr)

    def close(a, b):
        assert abs(a - b) <= 1e-10 * (abs(a) + abs(b) + 1.0), (a, b)

    d = rng.standard_normal((C, L))
    close(np.vdot(dv, d), np.vdot(dy, fwd(d, xs, hs)))           # y linear in v
    for n in range(N):
        d = rng.standard_normal((C, L))
        xs2 = list(xs)
        xs2[n] = d
        close(np.vdot(dx[n], d), np.vdot(dy, fwd(v, xs2, hs)))   # y linear in x_n
        for f in range(F):
            # y is linear in row f of h_n: replace that row by d, zero every
            # other row of h_n, and keep only the channels that use row f
            d = rng.standard_normal(L)
            hn = np.zeros_like(hs[n])
            hn[f] = d
            hs2 = list(hs)
            hs2[n] = hn
            y2 = fwd(v, xs, hs2)
            use = fr == f
            close(np.vdot(dh[n, f], d), np.vdot(dy[use], y2[use]))


def test_full_jacobian_by_unit_vectors_tiny():
    C, F, L, N = 2, 1, 8, 2
    v, xs, hs, fr, dy = _problem(C, F, L, N, seed=7)
    fr[:] = 0
    dv, dx, dh = oracle.hyena_backward(v, xs, hs, dy, filter_row=fr)
    for r in range(C):
        for i in range(L):
            e = np.zeros((C, L))
            e[r, i] = 1.0
            ref = np.vdot(dy, oracle.hyena_forward(e, xs, hs, filter_row=fr))
            assert abs(dv[r, i] - ref) <= 1e-12 * (abs(ref) + 1)


def test_delta_filter_closed_form():
    # N = 1, h = delta: y = x * v, so dv = dy x, dx = dy v, dh[j] = sum_t dy[t] x[t] v[t-j]
    L = 32
    v, x, dy = rng.standard_normal((1, L)), rng.standard_normal((1, L)), rng.standard_normal((1, L))
    h = np.zeros((1, L))
    h[0, 0] = 1.0
    dv, dx, dh = oracle.hyena_backward(v, [x], [h], dy)
    np.testing.assert_allclose(dv, dy * x, rtol=0, atol=1e-14)
    np.testing.assert_allclose(dx[0], dy * v, rtol=0, atol=1e-14)
    ref = np.array([sum(dy[0, t] * x[0, t] * v[0, t - j] for t in range(j, L)) for j in range(L)])
    np.testing.assert_allclose(dh[0, 0], ref, rtol=0, atol=1e-12)


def test_large_L_fft_branch_backward_matches_adjoint():
    # L > 8192 takes the FFT branches; check one adjoint identity there
    L, N = 16384, 2
    v, xs, hs, fr, dy = _problem(1, 1, L, N, seed=99)
    dv, dx, dh = oracle.hyena_backward(v, xs, hs, dy, filter_row=fr)
    d = rng.standard_normal((1, L))
    a = np.vdot(dv, d)
    b = np.vdot(dy, oracle.hyena_forward(d, xs, hs, filter_row=fr))
    assert abs(a - b) <= 1e-9 * (abs(a) + abs(b))
    d = rng.standard_normal(L)
    hs2 = [hs[0], d[None, :]]
    b = np.vdot(dy, oracle.hyena_forward(v, xs, hs2, filter_row=fr))
    a = np.vdot(dh[1, 0], d)
    assert abs(a - b) <= 1e-9 * (abs(a) + abs(b))


# ---------------------------------------------------- filter weights ------

def _grid_weights(N, D, H=16, E=17, seed=5):
    """Weights on a 2^-8 grid (exact in float32, and so is w +- 2^-12 k)."""
    g = np.random.default_rng(seed)

    def q(shape, scale):
        return (np.round(g.uniform(-scale, scale, shape) * 256) / 256).astype(np.float32)

    return {"W1": q((H, E), 0.8), "b1": q(H, 0.8), "W2": q((H, H), 0.5), "b2": q(H, 0.5),
            "W3": q((N * D, H), 0.5), "b3": q(N * D, 0.5)}


def _loss(w, N, D, L, lo, hi, dh):
    h = oracle.implicit_filter(w, N, D, L, lo, hi)
    return float(np.vdot(dh.reshape(N * D, L), h))


KEYS = ["W1", "b1", "W2", "b2", "W3", "b3"]


@pytest.mark.parametrize("key", KEYS)
def test_filter_backward_matches_central_differences(key):
    N, D, L, lo, hi = 2, 3, 24, 0.5, 20.0
    w = _grid_weights(N, D)
    g = np.random.default_rng(300 + KEYS.index(key))
    dh = g.standard_normal((N, D, L))
    grads = oracle.filter_backward(w, N, D, L, lo, hi, dh)
    direction = g.integers(-2, 3, w[key].shape).astype(np.float64)

    def central(eps):
        wp, wm = dict(w), dict(w)
        wp[key] = (w[key].astype(np.float64) + eps * direction).astype(np.float32)
        wm[key] = (w[key].astype(np.float64) - eps * direction).astype(np.float32)
        assert np.array_equal(wp[key].astype(np.float64) - w[key], eps * direction)   # exact in fp32
        assert np.array_equal(w[key] - wm[key].astype(np.float64), eps * direction)
        return (_loss(wp, N, D, L, lo, hi, dh) - _loss(wm, N, D, L, lo, hi, dh)) / (2 * eps)

    # central differences of a smooth function err by c eps^2 + O(eps^4);
    # Richardson's combination of eps and 2 eps cancels the eps^2 term
    eps = 2.0 ** -12
    fd = (4.0 * central(eps) - central(2 * eps)) / 3.0
    an = float(np.vdot(grads[key], direction))
    assert abs(fd - an) <= 1e-9 * (abs(an) + 1.0), (key, fd, an)


def test_filter_backward_linear_weights_closed_form():
    # h_{n,c}(t) = window_c(t) (W3 s2(t) + b3): the b3 gradient is sum_t dh window
    N, D, L, lo, hi = 1, 4, 32, 0.5, 20.0
    w = _grid_weights(N, D)
    dh = rng.standard_normal((N, D, L))
    grads = oracle.filter_backward(w, N, D, L, lo, hi, dh)
    t = np.arange(L)
    for c in range(D):
        a = oracle.alpha(c, D, lo, hi)
        ref = float(np.sum(dh[0, c] * np.exp(-a * t / L)))
        assert abs(grads["b3"][c] - ref) <= 1e-12 * (abs(ref) + 1)

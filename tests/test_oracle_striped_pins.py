"""Pins of the float64 StripedHyena-form oracle (q . (hG * (k . v)), short
explicit FIR featurizers; "02. 3つの Hyena 演算子", sections 2 and 4) to
things other than itself: numpy.convolve for every FIR, the already-pinned
order-1 Hyena forward oracle when the featurizers are deltas, delta and
shift cases, linearity and causality. No GPU is used."""
import numpy as np
import pytest

import oracle

rng = np.random.default_rng(77)


def np_striped(xq, xk, xv, hT, hH, hK, hG):
    L = len(xq)
    fir = lambda h, x: np.convolve(h, x)[:L]
    return fir(hT, xq) * fir(hG, fir(hH, xk) * fir(hK, xv))


@pytest.mark.parametrize("L,lf,lg", [(1, 1, 1), (5, 3, 2), (64, 4, 7), (300, 7, 128), (40, 16, 64)])
def test_matches_numpy_convolve(L, lf, lg):
    C = 3
    x = [rng.standard_normal((C, L)) for _ in range(3)]
    hs = [rng.standard_normal((C, lf)) for _ in range(3)]
    hG = rng.standard_normal((C, lg))
    y = oracle.striped_forward(*x, *hs, hG)
    for c in range(C):
        ref = np_striped(x[0][c], x[1][c], x[2][c], hs[0][c], hs[1][c], hs[2][c], hG[c])
        np.testing.assert_allclose(y[c], ref, rtol=1e-12, atol=1e-12)


def test_delta_featurizers_reduce_to_order1_hyena():
    # hT = hH = hK = delta: y = xq . (hG * (xk . xv)), the order-1 forward with
    # gate xq on the input xk . xv and filter hG zero-extended to length L
    C, L, lg = 2, 256, 200
    xq, xk, xv = (rng.standard_normal((C, L)) for _ in range(3))
    d = np.zeros((C, 4)); d[:, 0] = 1.0
    hG = rng.standard_normal((C, lg)) * np.exp(-np.arange(lg) / 50.0)
    y = oracle.striped_forward(xq, xk, xv, d, d, d, hG)
    hfull = np.zeros((C, L)); hfull[:, :lg] = hG
    ref = oracle.hyena_forward(xk * xv, [xq], [hfull])
    np.testing.assert_allclose(y, ref, rtol=1e-11, atol=1e-12)


def test_shifted_deltas_shift_the_inputs():
    # hT = delta at 1, hH = delta at 2, hK = delta, hG = delta at 3
    C, L = 1, 50
    xq, xk, xv = (rng.standard_normal((C, L)) for _ in range(3))
    e = lambda n, l: np.eye(1, l, n)
    y = oracle.striped_forward(xq, xk, xv, e(1, 4), e(2, 4), e(0, 4), e(3, 5))[0]
    sh = lambda a, s: np.concatenate([np.zeros(s), a[:L - s]])
    ref = sh(xq[0], 1) * sh(sh(xk[0], 2) * xv[0], 3)
    np.testing.assert_allclose(y, ref, rtol=0, atol=1e-14)


def test_linear_in_xq_and_in_hG_and_causal():
    C, L, lf, lg = 2, 120, 5, 30
    xq, xk, xv = (rng.standard_normal((C, L)) for _ in range(3))
    hT, hH, hK = (rng.standard_normal((C, lf)) for _ in range(3))
    hG = rng.standard_normal((C, lg))
    a, b = 0.7, -1.3
    xq2 = rng.standard_normal((C, L))
    f = lambda q, g: oracle.striped_forward(q, xk, xv, hT, hH, hK, g)
    np.testing.assert_allclose(f(a * xq + b * xq2, hG), a * f(xq, hG) + b * f(xq2, hG), rtol=1e-10, atol=1e-10)
    hG2 = rng.standard_normal((C, lg))
    np.testing.assert_allclose(f(xq, a * hG + b * hG2), a * f(xq, hG) + b * f(xq, hG2), rtol=1e-10, atol=1e-10)
    # perturbing xv at t0 leaves y[t < t0] bit-exact
    t0 = 70
    xv2 = xv.copy(); xv2[:, t0] += 5.0
    y1 = oracle.striped_forward(xq, xk, xv, hT, hH, hK, hG)
    y2 = oracle.striped_forward(xq, xk, xv2, hT, hH, hK, hG)
    assert np.array_equal(y1[:, :t0], y2[:, :t0]) and not np.array_equal(y1[:, t0:], y2[:, t0:])


def test_exponential_filter_matches_first_order_recurrences():
    # conv with h_t = sum_n R_n lam_n^t equals the sum over n of the recurrences
    # s_t = lam_n s_{t-1} + R_n z_t (the page's recurrent form of Hyena-LI)
    L, d = 200, 3
    R = rng.standard_normal((1, d))
    lam = rng.uniform(-0.95, 0.95, (1, d))
    z = rng.standard_normal(L)
    h = oracle.exponential_filter(R, lam, L)[0]
    ref = np.zeros(L)
    for n in range(d):
        s = 0.0
        for t in range(L):
            s = lam[0, n] * s + R[0, n] * z[t]
            ref[t] += s
    np.testing.assert_allclose(oracle.causal_conv(h, z, "direct"), ref, rtol=1e-10, atol=1e-12)
    assert h[0] == pytest.approx(R.sum())

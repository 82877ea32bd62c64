"""The pins catch plausible mistakes: each test plants one mistake in a copy
of an oracle step (on the CPU, in numpy), runs the same kind of check the
pins apply to the oracle, and requires that check to fail, while the oracle
itself passes it."""
import itertools

import numpy as np
import pytest

import oracle


def brute_causal(h, z):
    L = len(z)
    return np.array([sum(h[t - s] * z[s] for s in range(t + 1)) for t in range(L)])


def brute_nd(K, z, boundary):
    dims = z.shape
    y = np.zeros(dims)
    for p in itertools.product(*(range(d) for d in dims)):
        for q in itertools.product(*(range(d) for d in dims)):
            off = tuple(a - b for a, b in zip(p, q))
            if boundary == "circular":
                off = tuple(o % d for o, d in zip(off, dims))
            elif min(off) < 0:
                continue
            y[p] += K[off] * z[q]
    return y


def passes(check):
    try:
        check()
        return True
    except AssertionError:
        return False


RNG = np.random.default_rng(2024)
H, Z = RNG.standard_normal(24), RNG.standard_normal(24)


# ---------------------------------------------------------- causal sum --

CONV_MUTANTS = {
    "off-by-one lag": lambda h, z: np.array([sum(h[t - s - 1] * z[s] for s in range(t)) for t in range(len(z))]),
    "anti-causal (correlation)": lambda h, z: np.array(
        [sum(h[s - t] * z[s] for s in range(t, len(z))) for t in range(len(z))]),
    "circular wrap (no zero padding)": lambda h, z: np.real(np.fft.ifft(np.fft.fft(h) * np.fft.fft(z))),
    "dropped last tap": lambda h, z: np.array([sum(h[t - s] * z[s] for s in range(t)) for t in range(len(z))]),
}


def conv_check(fn):
    def check():
        np.testing.assert_allclose(fn(H, Z), brute_causal(H, Z), rtol=1e-9, atol=1e-9)
    return check


def test_causal_sum_pin_accepts_the_oracle():
    assert passes(conv_check(oracle.causal_conv))


@pytest.mark.parametrize("name", sorted(CONV_MUTANTS))
def test_causal_sum_pin_rejects(name):
    assert not passes(conv_check(CONV_MUTANTS[name])), name


# --------------------------------------------------------- recurrence --

def recurrence(v, xs, hs, mistake=None):
    z = v
    for n, (x, h) in enumerate(zip(xs, hs)):
        if mistake == "gate before convolution":
            z = brute_causal(h, x * z)
        elif mistake == "filters in reverse order":
            z = x * brute_causal(hs[len(hs) - 1 - n], z)
        elif mistake == "gate dropped on the last stage" and n == len(xs) - 1:
            z = brute_causal(h, z)
        elif mistake == "gates in reverse order":
            z = xs[len(xs) - 1 - n] * brute_causal(h, z)
        else:
            z = x * brute_causal(h, z)
    return z


V = RNG.standard_normal(16)
XS = [RNG.standard_normal(16) for _ in range(3)]
HS = [RNG.standard_normal(16) for _ in range(3)]


def recurrence_check(fn):
    def check():
        np.testing.assert_allclose(fn(V, XS, HS), oracle.hyena_forward(V[None], [x[None] for x in XS],
                                                                       [h[None] for h in HS])[0],
                                   rtol=1e-9, atol=1e-9)
    return check


def test_recurrence_pin_accepts_the_written_recurrence():
    assert passes(recurrence_check(recurrence))


@pytest.mark.parametrize("mistake", ["gate before convolution", "filters in reverse order",
                                     "gate dropped on the last stage", "gates in reverse order"])
def test_recurrence_pin_rejects(mistake):
    assert not passes(recurrence_check(lambda v, xs, hs: recurrence(v, xs, hs, mistake))), mistake


# ----------------------------------------------------- ND convolution --

DIMS = (4, 6)
KN, ZN = RNG.standard_normal(DIMS), RNG.standard_normal(DIMS)

ND_MUTANTS = {
    "zero boundary computed circularly": lambda K, z, b: oracle.nd_conv(K, z, "circular" if b == "zero" else b),
    "circular boundary computed with padding": lambda K, z, b: oracle.nd_conv(K, z, "zero" if b == "circular" else b),
    "transposed kernel": lambda K, z, b: (oracle.nd_conv(K.T.reshape(K.shape), z, b)),
    "kernel flipped (correlation)": lambda K, z, b: oracle.nd_conv(np.flip(K), z, b),
}


def nd_check(fn, boundary):
    def check():
        np.testing.assert_allclose(fn(KN, ZN, boundary), brute_nd(KN, ZN, boundary), rtol=1e-9, atol=1e-9)
    return check


@pytest.mark.parametrize("boundary", ["zero", "circular"])
def test_nd_pin_accepts_the_oracle(boundary):
    assert passes(nd_check(oracle.nd_conv, boundary))


@pytest.mark.parametrize("name", sorted(ND_MUTANTS))
def test_nd_pin_rejects(name):
    # each mutant must fail for at least one boundary (the boundary mutants only touch one)
    assert not all(passes(nd_check(ND_MUTANTS[name], b)) for b in ("zero", "circular")), name


# ---------------------------------------------------- filter spectrum --

def test_spectrum_closed_form_rejects_a_wrong_sign_or_scale():
    L = 16
    h = np.zeros(L); h[1] = 1.0                       # delta at lag 1: H[k] = exp(-2 pi i k / 2L)
    k = np.arange(L + 1)
    want = np.exp(-2j * np.pi * k / (2 * L))
    np.testing.assert_allclose(oracle.filter_spectrum(h), want, atol=1e-12)
    wrong_sign = np.conj(oracle.filter_spectrum(h))
    wrong_grid = np.fft.rfft(h)                       # L-point grid instead of 2L: no zero padding
    assert not np.allclose(wrong_sign, want, atol=1e-6)
    assert len(wrong_grid) != len(want) or not np.allclose(wrong_grid, want, atol=1e-6)

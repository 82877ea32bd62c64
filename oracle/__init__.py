"""float64 CPU oracle for the Hyena order-N forward and backward (ctypes wrapper of oracle.c).

TEST INFRASTRUCTURE ONLY: imported by tests/, by ``__graft_entry__.smoke()``
and by the CPU-baseline leg of ``bench.py``. The CUDA library never imports
or links it, and it never imports the CUDA library.

What each function computes, and the passage it follows, is stated in
oracle.c. Parity pins live in tests/test_oracle_pins.py. The implicit-filter
FFN itself has no printed worked example on the pages; it is pinned only
through closed-form special cases of its weights (see the pins).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB = os.path.join(_BUILD, "liboracle.so")

DIRECT_MAX_L = 8192


def build(force: bool = False) -> str:
    """Compile oracle.c with gcc (-O2, no fast-math: the summation order is
    the one written in the source)."""
    os.makedirs(_BUILD, exist_ok=True)
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        l = ctypes.CDLL(build())
        d, i64, i32 = ctypes.c_double, ctypes.c_int64, ctypes.c_int
        P = ctypes.c_void_p
        l.oracle_fft.argtypes = [P, P, i64, i32]
        l.oracle_causal_conv_direct.argtypes = [P, P, i64, P]
        l.oracle_causal_conv_fft.argtypes = [P, P, i64, P]
        l.oracle_causal_conv.argtypes = [P, P, i64, P]
        l.oracle_filter_spectrum.argtypes = [P, i64, P, P]
        l.oracle_embedding.argtypes = [i32, i32, i32, P]
        l.oracle_alpha.argtypes = [i32, i32, d, d]
        l.oracle_alpha.restype = d
        l.oracle_filter.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32, i32, d, d,
                                    i32, P, P, P, i32]
        l.oracle_hyena_forward.argtypes = [P, P, P, P, i64, i32, i64, i32, P, i32]
        l.oracle_hyena_forward.restype = i32
        for name in ("oracle_causal_corr_direct", "oracle_causal_corr_fft", "oracle_causal_corr",
                     "oracle_causal_xcorr_direct", "oracle_causal_xcorr_fft", "oracle_causal_xcorr"):
            getattr(l, name).argtypes = [P, P, i64, P]
        l.oracle_hyena_backward.argtypes = [P, P, P, P, P, i64, i32, i64, i32, P, P, P, i32]
        l.oracle_hyena_backward.restype = i32
        l.oracle_filter_backward.argtypes = [P, P, P, P, P, P, i32, i32, i32, i32, i32, d, d, P,
                                             P, P, P, P, P, P, i32]
        l.oracle_striped_forward.argtypes = [P, P, P, P, P, P, i32, P, i32, P, i64, i64, P, i32]
        l.oracle_striped_forward.restype = i32
        _lib = l
    return _lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float32)


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def default_threads() -> int:
    return os.cpu_count() or 1


def fft(x, sign: int = -1) -> np.ndarray:
    """Unnormalised DFT, X[k] = sum x[n] exp(sign 2 pi i n k / n) (power-of-two n)."""
    x = np.asarray(x, dtype=np.complex128)
    re, im = _f64(x.real).copy(), _f64(x.imag).copy()
    lib().oracle_fft(_p(re), _p(im), len(re), int(sign))
    return re + 1j * im


def causal_conv(h, z, method: str = "auto") -> np.ndarray:
    """(h conv z)[t] = sum_{s<=t} h[t-s] z[s], t < L."""
    h, z = _f64(h), _f64(z)
    assert h.shape == z.shape and h.ndim == 1
    out = np.empty_like(z)
    fn = {"auto": lib().oracle_causal_conv, "direct": lib().oracle_causal_conv_direct,
          "fft": lib().oracle_causal_conv_fft}[method]
    fn(_p(h), _p(z), len(z), _p(out))
    return out


def filter_spectrum(h) -> np.ndarray:
    """H[k] = sum_{t<L} h[t] exp(-2 pi i k t / 2L), k = 0..L (complex128, L+1 values)."""
    h = _f64(h)
    L = len(h)
    re, im = np.empty(L + 1), np.empty(L + 1)
    lib().oracle_filter_spectrum(_p(h), L, _p(re), _p(im))
    return re + 1j * im


def embedding(t: int, L: int, n_bands: int = 8) -> np.ndarray:
    e = np.empty(1 + 2 * n_bands)
    lib().oracle_embedding(int(t), int(L), int(n_bands), _p(e))
    return e


def alpha(c: int, D: int, lo: float, hi: float) -> float:
    return lib().oracle_alpha(int(c), int(D), float(lo), float(hi))


def implicit_filter(weights: dict, N: int, D: int, L: int, alpha_lo: float, alpha_hi: float,
                    rows: list[tuple[int, int]] | None = None, n_bands: int = 8,
                    threads: int | None = None) -> np.ndarray:
    """h rows [len(rows)][L] for (n, c) pairs (n 0-based); all N*D rows in
    [n][c] order when rows is None."""
    W1, b1, W2, b2, W3, b3 = (_f32(weights[k]) for k in ("W1", "b1", "W2", "b2", "W3", "b3"))
    width = W1.shape[0]
    assert W1.shape == (width, 1 + 2 * n_bands) and W2.shape == (width, width)
    assert W3.shape == (N * D, width) and b3.shape == (N * D,)
    if rows is None:
        rows = [(n, c) for n in range(N) for c in range(D)]
    rn = np.ascontiguousarray([r[0] for r in rows], dtype=np.int32)
    rc = np.ascontiguousarray([r[1] for r in rows], dtype=np.int32)
    h = np.empty((len(rows), L))
    lib().oracle_filter(_p(W1), _p(b1), _p(W2), _p(b2), _p(W3), _p(b3), n_bands, width,
                        N, D, L, float(alpha_lo), float(alpha_hi), len(rows), _p(rn), _p(rc),
                        _p(h), threads or default_threads())
    return h


def hyena_forward(v, xs, hs, filter_row=None, threads: int | None = None) -> np.ndarray:
    """Order-N forward on independent channels.

    v: [C][L]; xs: N arrays [C][L]; hs: N arrays [F][L] (filter rows);
    filter_row: per channel the row of each h_n it uses (default: row r).
    Returns y [C][L] (float64).
    """
    v = _f64(np.atleast_2d(v))
    C, L = v.shape
    N = len(xs)
    x = _f64(np.stack([np.atleast_2d(a) for a in xs]))
    h = _f64(np.stack([np.atleast_2d(a) for a in hs]))
    assert x.shape == (N, C, L) and h.shape[0] == N and h.shape[2] == L
    F = h.shape[1]
    fr = np.ascontiguousarray(np.arange(C) if filter_row is None else filter_row, dtype=np.int32)
    assert fr.shape == (C,) and (fr >= 0).all() and (fr < F).all()
    y = np.empty((C, L))
    rc = lib().oracle_hyena_forward(_p(v), _p(x), _p(h), _p(fr), C, F, L, N, _p(y),
                                    threads or default_threads())
    if rc != 0:
        raise ValueError("oracle_hyena_forward rejected its arguments")
    return y


def causal_corr(h, r, method: str = "auto") -> np.ndarray:
    """Transpose of the causal sum: out[s] = sum_{t>=s} h[t-s] r[t], s < L."""
    h, r = _f64(h), _f64(r)
    assert h.shape == r.shape and h.ndim == 1
    out = np.empty_like(r)
    fn = {"auto": lib().oracle_causal_corr, "direct": lib().oracle_causal_corr_direct,
          "fft": lib().oracle_causal_corr_fft}[method]
    fn(_p(h), _p(r), len(r), _p(out))
    return out


def causal_xcorr(r, z, method: str = "auto") -> np.ndarray:
    """Filter-gradient correlation: out[j] = sum_{t>=j} r[t] z[t-j], j < L."""
    r, z = _f64(r), _f64(z)
    assert r.shape == z.shape and r.ndim == 1
    out = np.empty_like(r)
    fn = {"auto": lib().oracle_causal_xcorr, "direct": lib().oracle_causal_xcorr_direct,
          "fft": lib().oracle_causal_xcorr_fft}[method]
    fn(_p(r), _p(z), len(r), _p(out))
    return out


def hyena_backward(v, xs, hs, dy, filter_row=None, threads: int | None = None):
    """Gradients of <dy, y> through the order-N forward on independent channels.

    v, dy: [C][L]; xs: N arrays [C][L]; hs: N arrays [F][L]; filter_row as in
    hyena_forward. Returns (dv [C][L], dx [N][C][L], dh [N][F][L]) where dh sums
    the contributions of every channel that uses a filter row.
    """
    v = _f64(np.atleast_2d(v))
    C, L = v.shape
    N = len(xs)
    x = _f64(np.stack([np.atleast_2d(a) for a in xs]))
    h = _f64(np.stack([np.atleast_2d(a) for a in hs]))
    dy = _f64(np.atleast_2d(dy))
    assert x.shape == (N, C, L) and h.shape[0] == N and h.shape[2] == L and dy.shape == (C, L)
    F = h.shape[1]
    fr = np.ascontiguousarray(np.arange(C) if filter_row is None else filter_row, dtype=np.int32)
    assert fr.shape == (C,) and (fr >= 0).all() and (fr < F).all()
    dv = np.empty((C, L))
    dx = np.empty((N, C, L))
    dh_ch = np.empty((N, C, L))
    rc = lib().oracle_hyena_backward(_p(v), _p(x), _p(h), _p(dy), _p(fr), C, F, L, N,
                                     _p(dv), _p(dx), _p(dh_ch), threads or default_threads())
    if rc != 0:
        raise ValueError("oracle_hyena_backward rejected its arguments")
    dh = np.zeros((N, F, L))
    for r in range(C):
        dh[:, fr[r], :] += dh_ch[:, r, :]
    return dv, dx, dh


def filter_backward(weights: dict, N: int, D: int, L: int, alpha_lo: float, alpha_hi: float, dh,
                    n_bands: int = 8, threads: int | None = None) -> dict:
    """Gradients of <dh, h> w.r.t. the implicit-filter weights (float64 dict
    with keys W1, b1, W2, b2, W3, b3). dh: [N][D][L] or [N*D][L]."""
    W1, b1, W2, b2, W3, b3 = (_f32(weights[k]) for k in ("W1", "b1", "W2", "b2", "W3", "b3"))
    width = W1.shape[0]
    dh = _f64(np.asarray(dh).reshape(N * D, L))
    out = {"W1": np.empty(W1.shape), "b1": np.empty(b1.shape), "W2": np.empty(W2.shape),
           "b2": np.empty(b2.shape), "W3": np.empty(W3.shape), "b3": np.empty(b3.shape)}
    lib().oracle_filter_backward(_p(W1), _p(b1), _p(W2), _p(b2), _p(W3), _p(b3), n_bands, width,
                                 N, D, L, float(alpha_lo), float(alpha_hi), _p(dh),
                                 *(_p(out[k]) for k in ("W1", "b1", "W2", "b2", "W3", "b3")),
                                 threads or default_threads())
    return out


def striped_forward(xq, xk, xv, hT, hH, hK, hG, filter_row=None, threads: int | None = None) -> np.ndarray:
    """StripedHyena-form operator y = (hT*xq) . (hG * ((hH*xk) . (hK*xv))) with
    causal FIR sums. x*: [C][L]; hT, hH, hK: [F][lf]; hG: [F][lg]."""
    xq, xk, xv = (_f64(np.atleast_2d(a)) for a in (xq, xk, xv))
    C, L = xq.shape
    hT, hH, hK, hG = (_f64(np.atleast_2d(a)) for a in (hT, hH, hK, hG))
    F, lf = hT.shape
    lg = hG.shape[1]
    assert hH.shape == hK.shape == (F, lf) and hG.shape[0] == F
    fr = np.ascontiguousarray(np.arange(C) if filter_row is None else filter_row, dtype=np.int32)
    y = np.empty((C, L))
    rc = lib().oracle_striped_forward(_p(xq), _p(xk), _p(xv), _p(hT), _p(hH), _p(hK), lf, _p(hG), lg,
                                      _p(fr), C, L, _p(y), threads or default_threads())
    if rc != 0:
        raise ValueError("oracle_striped_forward rejected its arguments")
    return y


def exponential_filter(R, lam, L: int) -> np.ndarray:
    """Hyena-LI filter ("02. 3つの Hyena 演算子", section 3): h[c][t] =
    sum_n R[c][n] lam[c][n]^t for t < L (0-based lag t; the page writes
    lambda^(t-1) with 1-based t). float64, evaluated term by term."""
    R, lam = _f64(np.atleast_2d(R)), _f64(np.atleast_2d(lam))
    t = np.arange(L, dtype=np.float64)
    return np.einsum("cn,cnt->ct", R, lam[:, :, None] ** t[None, None, :])


# ------------------------------------------------------------------ HyenaND --
# The N-dimensional operator of HyenaND (page "Native Multi-Dimensional
# Subquadratic Operators via Input Dependent Long Convolutions", section 手法:
# a global convolution evaluated on the L_1 x ... x L_N grid
# itself through an N-dimensional FFT, with a circular boundary for periodic
# systems or zero padding of the input to twice the grid for non-periodic
# data). Plain numpy, float64; numpy's FFT is the only library step.

def nd_conv(K, z, boundary: str) -> np.ndarray:
    """ND convolution of z by the kernel K on one grid (both shaped dims).
    circular:  y[p] = sum_q K[(p - q) mod dims] z[q]
    zero:      y[p] = sum_{0 <= q <= p} K[p - q] z[q]   (linear convolution of
               the grid signals, i.e. both zero-padded to 2 x dims; kept on the grid)"""
    K, z = np.asarray(K, dtype=np.float64), np.asarray(z, dtype=np.float64)
    assert K.shape == z.shape
    dims = z.shape
    if boundary == "circular":
        return np.real(np.fft.ifftn(np.fft.fftn(K) * np.fft.fftn(z)))
    if boundary != "zero":
        raise ValueError(boundary)
    s = tuple(2 * d for d in dims)
    axes = tuple(range(len(dims)))
    full = np.fft.irfftn(np.fft.rfftn(K, s, axes=axes) * np.fft.rfftn(z, s, axes=axes), s, axes=axes)
    return full[tuple(slice(0, d) for d in dims)]


def hyena_nd_forward(v, xs, Ks, dims, boundary: str, filter_row=None) -> np.ndarray:
    """Order-N recurrence of the Hyena operator with the ND convolution:
    z_1 = v, z_{n+1} = x_n . (K_n conv z_n), y = z_{N+1}, row by row.
    v, xs[n]: [C][prod(dims)] (grid flattened row-major); Ks[n]: [F][prod(dims)];
    filter_row[r] = the filter row of data row r (default r)."""
    v = _f64(np.atleast_2d(v))
    C = v.shape[0]
    fr = np.arange(C) if filter_row is None else np.asarray(filter_row)
    dims = tuple(int(d) for d in dims)
    Ks = [np.atleast_2d(k) for k in Ks]
    xs = [np.atleast_2d(x) for x in xs]
    y = np.empty_like(v)
    for r in range(C):
        z = v[r].reshape(dims)
        for n, x in enumerate(xs):
            K = _f64(Ks[n][fr[r]]).reshape(dims)
            z = _f64(x[r]).reshape(dims) * nd_conv(K, z, boundary)
        y[r] = z.reshape(-1)
    return y

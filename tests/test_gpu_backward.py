"""Parity of the CUDA backward (through the C ABI) with the float64 oracle.

Tolerances: dv and dx_n per (b, c) row, as for the forward: relative L2
<= 2e-5 for float32 I/O, <= 8e-3 for bfloat16 I/O (float32 arithmetic, bf16
rounding of the outputs). dh_n (float32 output for both I/O types) per
(n, c) row: relative L2 <= 1e-4 -- it chains up to 2N + 1 float32 2L-grid
FFT convolutions (each ~1e-6 relative) and sums the batch, and a row can be
smaller than the terms that cancel in it. Filter-weight gradients per
tensor: relative L2 <= 1e-4 (float32 sums over up to 2^20 taps in fixed
chunks, float32 activations).
"""
import numpy as np
import pytest

import oracle
import synth
from hyena_cases import TOL, rel_l2_rows, upload, weights_to_cuda

pytestmark = pytest.mark.gpu

DH_TOL = 1e-4
W_TOL = 1e-4


@pytest.fixture(scope="module", autouse=True)
def hy():
    from fft_long_convolution_implicit_b200 import build
    build.build()
    import fft_long_convolution_implicit_b200 as m
    m.load()
    return m


def gpu_backward(hy, w):
    wt = synth.filter_weights(w)
    v, xs = synth.inputs(w)
    dy = synth.dy_rows(w)
    tw = weights_to_cuda(wt)
    h = hy.filter_generate(tw, w.N, w.D, w.L, w.alpha_lo, w.alpha_hi)
    hh = [hy.filter_rfft(h[n]) for n in range(w.N)]
    dv, dxs, dh = hy.backward(upload(v, w), [upload(x, w) for x in xs], hh, upload(dy, w))
    import torch
    torch.cuda.synchronize()
    C, L = w.channels, w.L
    out = (dv.float().cpu().numpy().reshape(C, L), [d.float().cpu().numpy().reshape(C, L) for d in dxs],
           dh.cpu().numpy())
    return out, (v, xs, dy, wt, tw, dh)


def oracle_backward(w, cs, v, xs, dy, wt):
    """Oracle gradients for every batch item of the channels cs."""
    rows = [b * w.D + c for b in range(w.B) for c in cs]
    pairs = [(n, c) for n in range(w.N) for c in cs]
    hrows = oracle.implicit_filter(wt, w.N, w.D, w.L, w.alpha_lo, w.alpha_hi, rows=pairs)
    hs = [hrows[n * len(cs):(n + 1) * len(cs)] for n in range(w.N)]
    fr = [cs.index(r % w.D) for r in rows]
    dv, dx, dh = oracle.hyena_backward(np.asarray(v)[rows], [np.asarray(x)[rows] for x in xs], hs,
                                       np.asarray(dy)[rows], filter_row=fr)
    return rows, dv, dx, dh


def check(w, got, cs, v, xs, dy, wt):
    dv, dxs, dh = got
    rows, rv, rx, rh = oracle_backward(w, cs, v, xs, dy, wt)
    tol = TOL[w.dtype]
    e = rel_l2_rows(dv[rows], rv)
    assert e.max() <= tol, ("dv", e.max())
    for n in range(w.N):
        e = rel_l2_rows(dxs[n][rows], rx[n])
        assert e.max() <= tol, ("dx", n, e.max())
        e = rel_l2_rows(dh[n][cs], rh[n])
        assert e.max() <= DH_TOL, ("dh", n, e.max())


SWEEP = [
    # N, dtype, B, D, L
    (1, "f32", 1, 1, 16),        # zero-extended 128-point grid
    (2, "f32", 2, 3, 64),
    (3, "f32", 1, 2, 512),
    (2, "bf16", 2, 3, 1024),
    (2, "f32", 3, 2, 2048),
    (3, "bf16", 2, 2, 8192),
    (2, "f32", 1, 2, 16384),     # fused, 1024 threads per channel
    (2, "f32", 1, 2, 32768),     # four-step
    (2, "bf16", 2, 1, 32768),    # four-step
]


@pytest.mark.parametrize("N,dtype,B,D,L", SWEEP)
def test_backward_shapes(hy, N, dtype, B, D, L):
    w = synth.custom(N, dtype, B, D, L, seed=11 + L + N)
    got, (v, xs, dy, wt, _, _) = gpu_backward(hy, w)
    assert all(np.isfinite(a).all() for a in (got[0], got[2]))
    check(w, got, list(range(D)), v, xs, dy, wt)


@pytest.mark.parametrize("cfg_i,nc", [(0, None), (1, 4), (2, 3), (3, 2), (4, 1)])
def test_backward_workload(hy, cfg_i, nc):
    w = synth.workload(cfg_i)
    got, (v, xs, dy, wt, _, _) = gpu_backward(hy, w)
    cs = list(range(w.D)) if nc is None else sorted({0, w.D - 1, *[(w.D * k) // nc for k in range(nc)]})[:max(nc, 2)]
    check(w, got, cs, v, xs, dy, wt)


def test_backward_is_deterministic(hy):
    w = synth.custom(2, "bf16", 2, 3, 2048, seed=5)
    a, _ = gpu_backward(hy, w)
    b, _ = gpu_backward(hy, w)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[2], b[2])


# ------------------------------------------------------ filter weights ---

def _rel(a, b):
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(np.asarray(a, dtype=np.float64) - b) / np.linalg.norm(b))


@pytest.mark.parametrize("N,D,L", [(2, 16, 1024), (3, 1024, 8192), (2, 256, 131072), (1, 3, 16)])
def test_filter_backward_matches_oracle(hy, N, D, L):
    import torch
    w = synth.custom(N, "f32", 1, D, L, seed=40 + N)
    wt = synth.filter_weights(w)
    dh = synth.dh_rows(w)
    g = hy.filter_backward(weights_to_cuda(wt), N, D, L, w.alpha_lo, w.alpha_hi, torch.from_numpy(dh).cuda())
    ref = oracle.filter_backward(wt, N, D, L, w.alpha_lo, w.alpha_hi, dh.astype(np.float64))
    for k in ("W1", "b1", "W2", "b2", "W3", "b3"):
        e = _rel(g[k].cpu().numpy(), ref[k])
        assert e <= W_TOL, (k, e)


def test_backward_then_filter_backward_chain(hy):
    """Weight gradients of <dy, y> end to end, against the oracle chain."""
    w = synth.workload(0)
    got, (v, xs, dy, wt, tw, dh_gpu) = gpu_backward(hy, w)
    g = hy.filter_backward(tw, w.N, w.D, w.L, w.alpha_lo, w.alpha_hi, dh_gpu)
    cs = list(range(w.D))
    _, _, _, rh = oracle_backward(w, cs, v, xs, dy, wt)
    ref = oracle.filter_backward(wt, w.N, w.D, w.L, w.alpha_lo, w.alpha_hi, rh)
    for k in ("W1", "b1", "W2", "b2", "W3", "b3"):
        e = _rel(g[k].cpu().numpy(), ref[k])
        assert e <= W_TOL, (k, e)

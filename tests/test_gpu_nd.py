"""HyenaND parity: the CUDA path (through the C ABI) against the float64
oracle's ND convolution recurrence (page "Native Multi-Dimensional
Subquadratic Operators via Input Dependent Long Convolutions", section 手法).

Tolerance: per (b, c) row relative L2 <= 2e-5 for float32 I/O and <= 8e-3 for
bfloat16 I/O, the bar of the 1-D forward (the same float32 transform
arithmetic, the same output rounding). Small shapes are compared on every row;
the workloads at full size on a seeded sample of rows, plus a delta-kernel
identity that holds at any size.
"""
import numpy as np
import pytest

import oracle
import synth
from hyena_cases import TOL, rel_l2_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def hy():
    from fft_long_convolution_implicit_b200 import build
    build.build()
    import fft_long_convolution_implicit_b200 as m
    m.load()
    return m


def _up(a, w, dt):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).view(w.B, w.D, w.grid).cuda().to(dt)


def run_nd(hy, w, K=None, nsample=None):
    import torch
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    if K is None:
        K = synth.nd_kernels(w)
    v, xs = synth.nd_inputs(w)
    kh = [hy.nd_filter_spectrum(torch.from_numpy(K[n]).cuda(), w.dims, w.boundary) for n in range(w.N)]
    y = hy.nd_forward(_up(v, w, dt), [_up(x, w, dt) for x in xs], kh, w.dims, w.boundary)
    torch.cuda.synchronize()
    y = y.float().cpu().numpy().reshape(w.channels, w.grid)
    assert np.isfinite(y).all()
    rows = list(range(w.channels)) if nsample is None else synth.sample_rows(w.flat(), nsample)
    fr = [r % w.D for r in rows]
    ref = oracle.hyena_nd_forward(v[rows], [x[rows] for x in xs], [K[n] for n in range(w.N)], w.dims, w.boundary,
                                  filter_row=fr)
    return rel_l2_rows(y[rows], ref), y, (v, xs)


SHAPES = [
    # N, dtype, B, D, dims, boundary
    (1, "f32", 1, 2, (16,), "zero"),
    (2, "f32", 2, 2, (64,), "circular"),
    (2, "f32", 3, 2, (8, 16), "zero"),
    (3, "f32", 2, 3, (16, 8), "circular"),
    (2, "f32", 1, 2, (1, 32), "zero"),
    (2, "f32", 2, 2, (4, 8, 8), "zero"),
    (2, "f32", 2, 2, (8, 4, 16), "circular"),
    (1, "f32", 2, 1, (2, 2, 2), "circular"),
    (2, "f32", 2, 2, (1, 64), "circular"),     # unit axes are dropped
    (2, "f32", 1, 2, (8, 1, 16), "circular"),
    (2, "f32", 3, 1, (1, 1, 1), "circular"),   # a single point: y = x_N ... K^ v
    (2, "f32", 2, 2, (64, 64), "zero"),
    (2, "f32", 1, 2, (128, 128), "circular"),
    (2, "f32", 2, 1, (512,), "zero"),          # longest padded axis (1024)
    (2, "f32", 2, 1, (8192, 2), "circular"),   # rejected: padded axis above 1024
    (2, "bf16", 3, 3, (32, 32), "zero"),
    (4, "bf16", 2, 2, (8, 16, 8), "zero"),
    (2, "bf16", 2, 2, (16, 16, 64), "circular"),
]


@pytest.mark.parametrize("N,dtype,B,D,dims,boundary", SHAPES)
def test_nd_shapes(hy, N, dtype, B, D, dims, boundary):
    w = synth.nd_custom(N, dtype, B, D, dims, boundary, seed=41 + sum(dims) + N)
    if hy.nd_spectrum_bytes(D, dims, boundary) == 0:
        with pytest.raises(hy.HyenaError):
            run_nd(hy, w)
        return
    err, _, _ = run_nd(hy, w)
    assert err.max() <= TOL[dtype], err.max()


@pytest.mark.parametrize("i,nsample", [(0, None), (1, 8), (2, 6), (3, 8), (4, 6)])
def test_nd_workload(hy, i, nsample):
    w = synth.nd_workload(i)
    err, _, _ = run_nd(hy, w, nsample=nsample)
    print(f"{w.name}: max rel-L2 {err.max():.3e}")
    assert err.max() <= TOL[w.dtype], err.max()


@pytest.mark.parametrize("i", [1, 2, 3])
def test_nd_delta_kernel_identity(hy, i):
    # K_n = delta at offset 0: y = x_N ... x_1 v exactly up to the transform's rounding
    w = synth.nd_workload(i)
    K = np.zeros((w.N, w.D, w.grid), dtype=np.float32)
    K[:, :, 0] = 1.0
    _, y, (v, xs) = run_nd(hy, w, K=K, nsample=2)
    want = v.astype(np.float64)
    for x in xs:
        want = want * x
    err = rel_l2_rows(y, want)
    assert err.max() <= TOL[w.dtype], err.max()


def test_nd_spectrum_is_the_padded_dft(hy):
    import torch
    rng = np.random.default_rng(3)
    for dims, boundary in [((8, 16), "zero"), ((4, 8, 16), "circular"), ((32,), "zero")]:
        D = 3
        G = int(np.prod(dims))
        K = rng.standard_normal((D, G)).astype(np.float32)
        blk = hy.nd_filter_spectrum(torch.from_numpy(K).cuda(), dims, boundary).cpu().numpy()
        pdims = tuple(2 * d if boundary == "zero" else d for d in dims)
        P = int(np.prod(pdims))
        got = blk[: 8 * D * P].view(np.complex64).reshape(D, P)
        for c in range(D):
            full = np.fft.fftn(K[c].astype(np.float64).reshape(dims), s=pdims) / P
            # transform order: every axis index bit-reversed
            perm = [np.array([int(format(k, f"0{max(1, int(np.log2(n)))}b")[::-1], 2) if n > 1 else 0
                              for k in range(n)]) for n in pdims]
            want = full[np.ix_(*perm)].reshape(-1)
            err = np.linalg.norm(got[c] - want) / np.linalg.norm(want)
            assert err < 2e-6, (dims, boundary, c, err)


def test_nd_output_may_alias_input(hy):
    import torch
    w = synth.nd_custom(2, "f32", 2, 2, (16, 16), "zero", seed=5)
    K = synth.nd_kernels(w)
    v, xs = synth.nd_inputs(w)
    kh = [hy.nd_filter_spectrum(torch.from_numpy(K[n]).cuda(), w.dims, w.boundary) for n in range(w.N)]
    tv = _up(v, w, torch.float32)
    txs = [_up(x, w, torch.float32) for x in xs]
    y_ref = hy.nd_forward(tv, txs, kh, w.dims, w.boundary).cpu().numpy()
    hy.nd_forward(tv, txs, kh, w.dims, w.boundary, y=tv)
    np.testing.assert_array_equal(tv.cpu().numpy(), y_ref)

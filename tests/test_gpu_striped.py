"""Parity of the StripedHyena-form operator (CUDA, through the C ABI) with the
float64 oracle: y = (hT*xq) . (hG * ((hH*xk) . (hK*xv))), SE and MR inner
filters on the fused FIR kernel, LI (sum of exponentials) through the
featurizer and the order-1 FFT forward. Tolerance per (b, c) row: relative L2
<= 2e-5 for float32 I/O, <= 8e-3 for bfloat16 I/O (float32 arithmetic; in the
LI form q and u are stored in the I/O type between the two calls)."""
import numpy as np
import pytest

import oracle
import synth
from hyena_cases import TOL, rel_l2_rows, upload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def hy():
    from fft_long_convolution_implicit_b200 import build
    build.build()
    import fft_long_convolution_implicit_b200 as m
    m.load()
    return m


def cuda(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def run_fir(hy, w, lf, lg, rows=None):
    import torch
    xv, (xq, xk) = synth.inputs(w)
    hT, hH, hK, hG = synth.striped_filters(w, lf, lg)
    y = hy.striped_forward(upload(xq, w), upload(xk, w), upload(xv, w), cuda(hT), cuda(hH), cuda(hK), cuda(hG))
    torch.cuda.synchronize()
    got = y.float().cpu().numpy().reshape(w.channels, w.L)
    rows = list(range(w.channels)) if rows is None else rows
    fr = [r % w.D for r in rows]
    ref = oracle.striped_forward(xq[rows], xk[rows], xv[rows], hT, hH, hK, hG, filter_row=fr)
    return rel_l2_rows(got[rows], ref)


SHAPES = [
    # dtype, B, D, L, lf, lg
    ("f32", 2, 3, 100, 4, 7),        # SE, one ragged tile
    ("bf16", 2, 3, 100, 4, 7),
    ("f32", 1, 2, 5000, 7, 5),       # three tiles, ragged tail
    ("bf16", 4, 8, 2048, 4, 7),
    ("f32", 1, 2, 5000, 4, 7),       # SE sizes on the unrolled kernel: three tiles, ragged tail
    ("bf16", 2, 2, 6144, 4, 7),
    ("f32", 2, 2, 4096, 3, 128),     # MR
    ("bf16", 1, 3, 6000, 5, 1024),   # longest inner filter, halo past a tile
    ("f32", 1, 1, 1, 1, 1),          # degenerate
    ("f32", 1, 2, 30, 16, 64),       # filters longer than the row
]


@pytest.mark.parametrize("dtype,B,D,L,lf,lg", SHAPES)
def test_striped_fir_shapes(hy, dtype, B, D, L, lf, lg):
    w = synth.custom(2, dtype, B, D, L, seed=31 + L + lg)
    err = run_fir(hy, w, lf, lg)
    assert err.max() <= TOL[dtype], err.max()


def test_striped_fir_workload_shape_sampled(hy):
    """The order-2 bench workload's shape (B=4, D=768, L=2048, bf16) with SE
    filters (lf = 4, lg = 7), sampled rows."""
    w = synth.workload(1)
    err = run_fir(hy, w, 4, 7, rows=synth.sample_rows(w, 24))
    assert err.max() <= TOL[w.dtype], err.max()


@pytest.mark.parametrize("dtype,B,D,L,d", [("f32", 2, 3, 2048, 4), ("bf16", 2, 2, 8192, 3), ("bf16", 1, 2, 32768, 2)])
def test_striped_li_through_fft_forward(hy, dtype, B, D, L, d):
    import torch
    w = synth.custom(1, dtype, B, D, L, seed=91 + L)
    xv, (xq,) = synth.inputs(w)
    xk = synth.v_rows(synth.custom(1, dtype, B, D, L, seed=92 + L))
    hT, hH, hK, _ = synth.striped_filters(w, 4, 1)
    R, lam = synth.exponential_params(w, d)
    h = hy.filter_exponential(cuda(R), cuda(lam), L)
    hh = hy.filter_rfft(h)
    q, u = hy.striped_featurize(upload(xq, w), upload(xk, w), upload(xv, w), cuda(hT), cuda(hH), cuda(hK))
    y = hy.forward(u, [q], [hh])
    torch.cuda.synchronize()
    got = y.float().cpu().numpy().reshape(w.channels, L)
    hG = oracle.exponential_filter(R, lam, L)
    ref = oracle.striped_forward(xq, xk, xv, hT, hH, hK, hG, filter_row=[r % D for r in range(w.channels)])
    err = rel_l2_rows(got, ref)
    assert err.max() <= TOL[dtype], err.max()
    # the generated filter itself
    np.testing.assert_allclose(h.cpu().numpy(), hG, rtol=2e-5, atol=1e-6 * np.abs(hG).max())

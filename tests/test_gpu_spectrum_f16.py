"""Reduced-precision filter spectra: the f16 block and the forward that reads it.

The conversion is checked bit for bit against its plain definition (a
power-of-two scale per channel that puts the largest component in
[2^14, 2^15), then round to nearest even to f16, numpy's own float16 cast).

The forward (bf16 I/O only; float32 I/O is refused) is compared with the
float64 oracle, which keeps exact spectra, at the bf16 bar of the float32
spectra, 8e-3: each bin of each stage's spectrum moves by at most 2^-11 of
its own magnitude (the scaled components sit in f16's normal range unless
they are below 2^-29 of the channel's largest one), so a stage's convolution
moves by at most 2^-11 in relative L2 (Parseval), below the bf16 output
rounding (2^-9) that the bar is set for.
"""
import numpy as np
import pytest

import synth
from hyena_cases import TOL, oracle_rows, rel_l2_rows, upload, weights_to_cuda

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def hy():
    from fft_long_convolution_implicit_b200 import build
    build.build()
    import fft_long_convolution_implicit_b200 as m
    m.load()
    return m


def tol_f16(w) -> float:
    assert w.dtype == "bf16"
    return TOL["bf16"]


@pytest.mark.parametrize("L", [16, 1024, 8192, 16384, 131072])
def test_conversion_is_exact_scaled_rounding(hy, L):
    import torch
    rng = np.random.default_rng(100 + L)
    D = 4
    h = (rng.standard_normal((D, L)) * np.exp(-np.arange(L) / (0.1 * L))).astype(np.float32)
    h[1] *= 1e-30      # scale far below one
    h[2] = 0.0         # all-zero channel: scale 1
    h[3] *= 3e4        # components well above the f16 range before scaling
    hh = hy.filter_rfft(torch.from_numpy(h).cuda())
    h16 = hy.spectrum_to_f16(hh, D, L)
    torch.cuda.synchronize()
    M, _, _ = hy.spectrum_layout(L)
    f32 = hh.cpu().numpy()
    b16 = h16.cpu().numpy()
    assert b16.nbytes == hy.load().hyena_filter_spectrum_bytes_f16(D, L)
    bins = f32[: 8 * D * M].view(np.float32).reshape(D, 2 * M)
    got = b16[: 4 * D * M].view(np.float16).reshape(D, 2 * M)
    inv = b16[4 * D * M: 4 * D * M + 4 * D].view(np.float32)
    for c in range(D):
        mx = np.abs(bins[c]).max()
        if mx == 0:
            assert inv[c] == 1.0        # bins stay signed zeros (a zero filter's bins may be -0)
        else:
            m, e = np.frexp(np.float64(inv[c]))
            assert m == 0.5, inv[c]                 # a power of two
            assert 2.0 ** 14 <= mx / np.float64(inv[c]) < 2.0 ** 15, (c, mx / inv[c])
        s = 1.0 / np.float64(inv[c])
        want = (bins[c].astype(np.float64) * s).astype(np.float32).astype(np.float16)
        np.testing.assert_array_equal(got[c].view(np.uint16), want.view(np.uint16))
    # the FFT tables close both blocks and travel unchanged
    t16 = (4 * D * M + 4 * D + 15) // 16 * 16
    tb = b16.nbytes - t16
    assert tb > 0
    np.testing.assert_array_equal(b16[t16:], f32[f32.nbytes - tb:])


def run_f16(hy, w, nsample=None):
    import torch
    wt = synth.filter_weights(w)
    v, xs = synth.inputs(w)
    h = hy.filter_generate(weights_to_cuda(wt), w.N, w.D, w.L, w.alpha_lo, w.alpha_hi)
    hh16 = [hy.spectrum_to_f16(hy.filter_rfft(h[n]), w.D, w.L) for n in range(w.N)]
    y = hy.forward_f16_spectra(upload(v, w), [upload(x, w) for x in xs], hh16)
    torch.cuda.synchronize()
    hy.check_device_timeouts()
    y = y.float().cpu().numpy().reshape(w.channels, w.L)
    assert np.isfinite(y).all()
    rows = list(range(w.channels)) if nsample is None else synth.sample_rows(w, nsample)
    ref = oracle_rows(w, rows, v, xs, wt)
    err = rel_l2_rows(y[rows], ref)
    print(f"f16 spectra {w.name}: max rel-L2 {err.max():.3e} (bar {tol_f16(w):.3e})")
    return err


@pytest.mark.parametrize("cfg_i,nsample", [(1, 16), (2, 8), (3, 4), (4, 2)])
def test_forward_f16_workload(hy, cfg_i, nsample):
    w = synth.workload(cfg_i)
    err = run_f16(hy, w, nsample)
    assert err.max() <= tol_f16(w), err.max()


def test_forward_f16_refuses_f32_io(hy):
    import torch
    w = synth.workload(0)          # the float32 workload
    wt = synth.filter_weights(w)
    v, xs = synth.inputs(w)
    h = hy.filter_generate(weights_to_cuda(wt), w.N, w.D, w.L, w.alpha_lo, w.alpha_hi)
    hh16 = [hy.spectrum_to_f16(hy.filter_rfft(h[n]), w.D, w.L) for n in range(w.N)]
    y = torch.full((w.B, w.D, w.L), float("nan"), device="cuda")
    with pytest.raises(hy.HyenaError) as e:
        hy.forward_f16_spectra(upload(v, w), [upload(x, w) for x in xs], hh16, y=y)
    assert e.value.status == hy.HYENA_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert torch.isnan(y).all()    # nothing was launched


@pytest.mark.parametrize("N,dtype,B,D,L", [
    (1, "bf16", 1, 2, 16),
    (3, "bf16", 2, 3, 128),
    (2, "bf16", 2, 2, 1024),      # would take the tensor-core kernel with float32 spectra
    (2, "bf16", 2, 3, 2048),
    (2, "bf16", 1, 2, 8192),
    (3, "bf16", 1, 2, 16384),
    (2, "bf16", 1, 2, 65536),
    (1, "bf16", 1, 1, 262144),
])
def test_forward_f16_shapes(hy, N, dtype, B, D, L):
    w = synth.custom(N, dtype, B, D, L, seed=31 + L + N)
    err = run_f16(hy, w)
    assert err.max() <= tol_f16(w), err.max()


"""hyena_forward_static_workspace: the long-sequence forward for callers that
cannot allocate device memory (pool-owned devices, fixed budgets, paths that
cannot take cudaMalloc's implicit synchronisation). It runs with the
library's own static device scratch instead of a caller workspace.

Checked through the C ABI against hyena_forward with a caller workspace, on
two calls in a row (the scratch keeps the previous call's contents, which
must not leak into the next result). This file is collected last.
"""
import ctypes

import numpy as np
import pytest

import synth
from hyena_cases import TOL, rel_l2_rows, upload, weights_to_cuda

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("N,dtype,B,D,L", [(2, "bf16", 2, 3, 32768), (2, "bf16", 1, 40, 131072),
                                           (3, "f32", 1, 2, 16384)])
def test_static_workspace_matches_workspace_forward(N, dtype, B, D, L):
    import torch
    from fft_long_convolution_implicit_b200 import build
    build.build()
    import fft_long_convolution_implicit_b200 as hy
    lib = hy.load()

    w = synth.custom(N, dtype, B, D, L, seed=21 + L)
    wt = synth.filter_weights(w)
    v, xs = synth.inputs(w)
    h = hy.filter_generate(weights_to_cuda(wt), w.N, w.D, w.L, w.alpha_lo, w.alpha_hi)
    hh = [hy.filter_rfft(h[n]) for n in range(w.N)]
    tv = upload(v, w)
    txs = [upload(x, w) for x in xs]
    y_ref = hy.forward(tv, txs, hh)          # caller-provided workspace
    torch.cuda.synchronize()
    ref = y_ref.double().cpu().numpy().reshape(w.channels, L)

    code = hy.HYENA_BF16 if dtype == "bf16" else hy.HYENA_F32
    xarr = (ctypes.c_void_p * N)(*[x.data_ptr() for x in txs])
    harr = (ctypes.c_void_p * N)(*[t.data_ptr() for t in hh])
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        y = torch.full_like(tv, float("nan"))
        st = lib.hyena_forward_static_workspace(ctypes.c_void_p(tv.data_ptr()), xarr, harr, B, D, L, N, code,
                                                ctypes.c_void_p(y.data_ptr()), stream)
        assert st == hy.HYENA_OK, lib.hyena_status_string(st)
        torch.cuda.synchronize()
        got = y.double().cpu().numpy().reshape(w.channels, L)
        assert np.isfinite(got).all(), call
        err = rel_l2_rows(got, ref)
        assert err.max() <= TOL[dtype], (call, err.max())


def test_static_workspace_rejects_short_lengths():
    import torch
    import fft_long_convolution_implicit_b200 as hy
    lib = hy.load()
    t = torch.zeros(16, device="cuda")
    p = ctypes.c_void_p(t.data_ptr())
    arr = (ctypes.c_void_p * 2)(t.data_ptr(), t.data_ptr())
    assert lib.hyena_forward_static_workspace(p, arr, arr, 1, 1, 2048, 2, hy.HYENA_F32, p, None) \
        == hy.HYENA_ERR_UNSUPPORTED
    assert lib.hyena_forward_static_workspace(p, arr, arr, 1, 1, 3000, 2, hy.HYENA_F32, p, None) \
        == hy.HYENA_ERR_UNSUPPORTED

"""hyena_forward_static_workspace: the long-sequence forward for callers that
cannot allocate device memory (pool-owned devices, fixed budgets, paths that
cannot take cudaMalloc's implicit synchronisation). It runs with the
library's own static device scratch instead of a caller workspace.

Checked through the C ABI against hyena_forward with a caller workspace, on
two calls in a row (the scratch keeps the previous call's contents, which
must not leak into the next result): the results are bit for bit equal (the
two calls differ only in how many channels a wave holds, and every channel's
arithmetic is the same whatever the wave), one row is checked against the
float64 oracle, and the device's free memory is the same before and after a
call (nothing is allocated). The shapes include L = 2^20: in float32 the
16 MiB scratch holds two channels per wave and the last wave is partial; in
bf16 (order <= 3) the row pass runs on the tensor cores and also keeps the
column pass's per-channel maxima in the scratch, so a wave holds one channel.
This file is collected last.
"""
import ctypes

import numpy as np
import pytest

import synth
from hyena_cases import TOL, oracle_rows, rel_l2_rows, upload, weights_to_cuda

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("N,dtype,B,D,L", [(2, "bf16", 2, 3, 32768), (2, "bf16", 1, 40, 131072),
                                           (3, "f32", 1, 2, 32768), (2, "bf16", 1, 3, 1 << 20),
                                           (2, "f32", 1, 3, 1 << 20)])
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
    ref_bits = y_ref.view(torch.int16 if dtype == "bf16" else torch.int32).cpu().numpy()

    code = hy.HYENA_BF16 if dtype == "bf16" else hy.HYENA_F32
    xarr = (ctypes.c_void_p * N)(*[x.data_ptr() for x in txs])
    harr = (ctypes.c_void_p * N)(*[t.data_ptr() for t in hh])
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    ys = [torch.full_like(tv, float("nan")) for _ in range(2)]
    # a warm-up call loads the library module that holds the scratch
    assert lib.hyena_forward_static_workspace(ctypes.c_void_p(tv.data_ptr()), xarr, harr, B, D, L, N, code,
                                              ctypes.c_void_p(ys[0].data_ptr()), stream) == hy.HYENA_OK
    torch.cuda.synchronize()
    for call in range(2):
        y = ys[call]
        y.fill_(float("nan"))
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        reserved_before = torch.cuda.memory_reserved()
        st = lib.hyena_forward_static_workspace(ctypes.c_void_p(tv.data_ptr()), xarr, harr, B, D, L, N, code,
                                                ctypes.c_void_p(y.data_ptr()), stream)
        assert st == hy.HYENA_OK, lib.hyena_status_string(st)
        torch.cuda.synchronize()
        assert torch.cuda.mem_get_info()[0] == free_before, call
        assert torch.cuda.memory_reserved() == reserved_before, call
        got_bits = y.view(torch.int16 if dtype == "bf16" else torch.int32).cpu().numpy()
        np.testing.assert_array_equal(got_bits, ref_bits, err_msg=f"call {call}")
    hy.check_device_timeouts()
    # one row against the float64 oracle (the last row: the last, partial wave)
    row = w.channels - 1
    got = ys[1].float().cpu().numpy().reshape(w.channels, L)[[row]]
    ref = oracle_rows(w, [row], v, xs, wt)
    err = rel_l2_rows(got, ref)
    assert err.max() <= TOL[dtype], err.max()


def test_static_workspace_rejects_short_lengths():
    import torch
    import fft_long_convolution_implicit_b200 as hy
    lib = hy.load()
    t = torch.zeros(16, device="cuda")
    p = ctypes.c_void_p(t.data_ptr())
    arr = (ctypes.c_void_p * 2)(t.data_ptr(), t.data_ptr())
    assert lib.hyena_forward_static_workspace(p, arr, arr, 1, 1, 2048, 2, hy.HYENA_F32, p, None) \
        == hy.HYENA_ERR_UNSUPPORTED
    assert lib.hyena_forward_static_workspace(p, arr, arr, 1, 1, 16384, 2, hy.HYENA_F32, p, None) \
        == hy.HYENA_ERR_UNSUPPORTED
    assert lib.hyena_forward_static_workspace(p, arr, arr, 1, 1, 3000, 2, hy.HYENA_F32, p, None) \
        == hy.HYENA_ERR_UNSUPPORTED
    # misaligned or null pointers are refused on the host, before any lookup
    mis = ctypes.c_void_p(t.data_ptr() + 4)
    assert lib.hyena_forward_static_workspace(mis, arr, arr, 1, 1, 32768, 2, hy.HYENA_F32, p, None) \
        == hy.HYENA_ERR_INVALID_ARG
    assert lib.hyena_forward_static_workspace(p, None, arr, 1, 1, 32768, 2, hy.HYENA_F32, p, None) \
        == hy.HYENA_ERR_INVALID_ARG

"""C-ABI checks that need no GPU: the library builds and loads, exports every
function include/hyena.h declares, and rejects bad arguments on the host
before touching CUDA."""
import ctypes
import os
import re

import pytest

import fft_long_convolution_implicit_b200 as hy
from fft_long_convolution_implicit_b200 import build as hybuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    hybuild.build()
    return hy.load()


def declared_functions():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names += re.findall(r"\b(hyena_[a-z0-9_]+)\s*\(", src)
    return sorted(set(names))


def test_header_declares_the_binding_exports():
    assert set(declared_functions()) == set(hy.EXPORTS)


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_host_queries(lib):
    assert hy.abi_version() == 2
    assert lib.hyena_status_string(0) == b"ok"
    # spectrum block: D*M complex64 + tables
    M, M1, MV = hy.spectrum_layout(2048)
    assert (M, M1, MV) == (2048, 1, 2048)
    assert hy.filter_spectrum_bytes(768, 2048) >= 768 * 2048 * 8
    assert hy.spectrum_layout(16)[0] == 128                  # small L is zero-extended to 128 points
    M, M1, MV = hy.spectrum_layout(1 << 20)
    assert M == 1 << 20 and M1 * MV == M and MV <= 4096
    # rows of 4096 (L = 2^19, 2^20): spectrum, tables (MV-point plan, w_2MV, M1-point
    # plan), [D] float maxima padded to 16 bytes, then the [D][L] __half2 copy
    for L in (1 << 19, 1 << 20):
        M, M1, MV = hy.spectrum_layout(L)
        assert MV == 4096
        for D in (1, 3, 4, 5):
            tables = 8 * (2 * MV + M1)
            assert hy.filter_spectrum_bytes(D, L) == 8 * D * M + tables + 16 * ((D + 3) // 4) + 4 * D * L
    M, M1, MV = hy.spectrum_layout(131072)
    assert (M1, MV) == (128, 1024)
    assert hy.forward_workspace_bytes(4, 768, 2048, 2, True) == 0
    ws = hy.forward_workspace_bytes(1, 256, 131072, 2, True)
    assert ws % (131072 * 8) == 0 and ws >= 131072 * 8
    # SIMT rows: all channels in one wave, up to 1 GiB
    assert ws == 256 * 131072 * 8
    assert hy.forward_workspace_bytes(8, 256, 131072, 2, True) == 1024 * 131072 * 8
    # tensor-core rows of 4096 (bf16, order <= 3): 5/8 of the L2, 8 more bytes per channel
    per = 8 * (1 << 20) + 8
    ws_t = hy.forward_workspace_bytes(1, 256, 1 << 20, 2, True)
    assert ws_t % per == 0 and 1 <= ws_t // per <= 20
    ws_s = hy.forward_workspace_bytes(1, 256, 1 << 20, 2, False)   # float32 I/O: SIMT rows
    assert ws_s % per == 0 and ws_s // per == (1 << 30) // per
    assert hy.forward_workspace_bytes(1, 256, 1 << 20, 4, True) == ws_s   # order 4: SIMT rows
    assert hy.forward_workspace_bytes(1, 1, 1000, 2, True) == 0       # unsupported L
    assert hy.filter_spectrum_bytes(4, 3000) == 0


@pytest.mark.parametrize("L", [0, 8, 1000, 3 << 10, 1 << 21])
def test_unsupported_lengths_rejected_before_launch(lib, L):
    p = ctypes.c_void_p(16)      # never dereferenced: the call must fail on the host
    xs = (ctypes.c_void_p * 2)(16, 16)
    st = lib.hyena_forward(p, xs, xs, 1, 1, L, 2, hy.HYENA_BF16, p, None, 0, None)
    assert st == hy.HYENA_ERR_UNSUPPORTED
    assert lib.hyena_filter_rfft(p, 1, L, p, None) == hy.HYENA_ERR_UNSUPPORTED


def test_invalid_arguments_rejected_before_launch(lib):
    p = ctypes.c_void_p(16)
    xs = (ctypes.c_void_p * 2)(16, 16)
    f = lib.hyena_forward
    assert f(None, xs, xs, 1, 1, 1024, 2, 0, p, None, 0, None) == hy.HYENA_ERR_INVALID_ARG
    assert f(p, None, xs, 1, 1, 1024, 2, 0, p, None, 0, None) == hy.HYENA_ERR_INVALID_ARG
    assert f(p, xs, xs, 1, 1, 1024, 0, 0, p, None, 0, None) == hy.HYENA_ERR_INVALID_ARG
    assert f(p, xs, xs, 1, 1, 1024, 9, 0, p, None, 0, None) == hy.HYENA_ERR_INVALID_ARG
    assert f(p, xs, xs, 0, 1, 1024, 2, 0, p, None, 0, None) == hy.HYENA_ERR_INVALID_ARG
    assert f(p, xs, xs, 1, 1, 1024, 2, 7, p, None, 0, None) == hy.HYENA_ERR_INVALID_ARG
    mis = ctypes.c_void_p(24)    # 8-byte aligned only
    assert f(mis, xs, xs, 1, 1, 1024, 2, 0, p, None, 0, None) == hy.HYENA_ERR_INVALID_ARG
    # long L needs a workspace of at least 8 L bytes
    assert f(p, xs, xs, 1, 1, 1 << 15, 2, 0, p, None, 0, None) == hy.HYENA_ERR_WORKSPACE
    assert f(p, xs, xs, 1, 1, 1 << 15, 2, 0, p, p, 8 * (1 << 15) - 16, None) == hy.HYENA_ERR_WORKSPACE
    fp = hy.FilterParams(16, 16, 16, 16, 16, 16, 8, 64)
    g = lib.hyena_filter_generate
    assert g(None, 2, 4, 1024, 0.5, 20.0, p, None) == hy.HYENA_ERR_INVALID_ARG
    assert g(ctypes.byref(fp), 2, 4, 1000, 0.5, 20.0, p, None) == hy.HYENA_ERR_UNSUPPORTED
    bad = hy.FilterParams(16, 16, 16, 16, 16, 16, 8, 512)
    assert g(ctypes.byref(bad), 2, 4, 1024, 0.5, 20.0, p, None) == hy.HYENA_ERR_INVALID_ARG


def test_status_strings(lib):
    for s in range(5):
        assert lib.hyena_status_string(s)
    assert lib.hyena_last_cuda_error() == b""


def test_backward_queries_and_host_rejections(lib):
    ws = hy.backward_workspace_bytes(2, 3, 1024, 2, False)
    # u_1..u_N, z and rev(r), g, unit gates: (N + 4) float32 tensors, plus spectra of 2BD rows
    assert ws >= (2 + 4) * 4 * 2 * 3 * 1024 + 2 * 2 * 3 * 1024 * 8
    assert hy.backward_workspace_bytes(2, 3, 1000, 2, False) == 0
    assert hy.backward_workspace_bytes(2, 3, 1024, 9, False) == 0
    assert hy.filter_backward_workspace_bytes(2, 16, 1024) > 0
    assert hy.filter_backward_workspace_bytes(2, 16, 1000) == 0
    p = ctypes.c_void_p(16)
    xs = (ctypes.c_void_p * 2)(16, 16)
    f = lib.hyena_backward
    # unsupported length, bad order, null arrays, misaligned pointer, small workspace
    assert f(p, xs, xs, p, 1, 1, 1000, 2, 0, p, xs, xs, p, 1 << 30, None) == hy.HYENA_ERR_UNSUPPORTED
    assert f(p, xs, xs, p, 1, 1, 1024, 0, 0, p, xs, xs, p, 1 << 30, None) == hy.HYENA_ERR_INVALID_ARG
    assert f(p, xs, xs, p, 1, 1, 1024, 2, 0, p, None, xs, p, 1 << 30, None) == hy.HYENA_ERR_INVALID_ARG
    assert f(p, xs, xs, ctypes.c_void_p(24), 1, 1, 1024, 2, 0, p, xs, xs, p, 1 << 30, None) == hy.HYENA_ERR_INVALID_ARG
    need = hy.backward_workspace_bytes(1, 1, 1024, 2, False)
    assert f(p, xs, xs, p, 1, 1, 1024, 2, 0, p, xs, xs, p, need - 1, None) == hy.HYENA_ERR_WORKSPACE
    assert f(p, xs, xs, p, 1, 1, 1024, 2, 0, p, xs, xs, None, need, None) == hy.HYENA_ERR_WORKSPACE
    fp = hy.FilterParams(16, 16, 16, 16, 16, 16, 8, 64)
    g = hy.FilterGrads(16, 16, 16, 16, 16, 16)
    fb = lib.hyena_filter_backward
    need = hy.filter_backward_workspace_bytes(2, 4, 256)
    assert fb(ctypes.byref(fp), 2, 4, 256, 0.5, 20.0, p, ctypes.byref(g), p, need - 1, None) == hy.HYENA_ERR_WORKSPACE
    assert fb(ctypes.byref(fp), 2, 4, 300, 0.5, 20.0, p, ctypes.byref(g), p, need, None) == hy.HYENA_ERR_UNSUPPORTED
    assert fb(None, 2, 4, 256, 0.5, 20.0, p, ctypes.byref(g), p, need, None) == hy.HYENA_ERR_INVALID_ARG
    bad = hy.FilterGrads(16, 16, 16, 16, None, 16)
    assert fb(ctypes.byref(fp), 2, 4, 256, 0.5, 20.0, p, ctypes.byref(bad), p, need, None) == hy.HYENA_ERR_INVALID_ARG


def test_striped_host_rejections(lib):
    p = ctypes.c_void_p(16)
    f = lib.hyena_striped_forward
    ok = (p, p, p, p, p, p, 4, p, 7, 2, 3, 100, hy.HYENA_BF16, p, None)
    bad_lf = (p, p, p, p, p, p, 17, p, 7, 2, 3, 100, hy.HYENA_BF16, p, None)
    bad_lg = (p, p, p, p, p, p, 4, p, 1025, 2, 3, 100, hy.HYENA_BF16, p, None)
    bad_L = (p, p, p, p, p, p, 4, p, 7, 2, 3, 0, hy.HYENA_BF16, p, None)
    mis = (ctypes.c_void_p(24), p, p, p, p, p, 4, p, 7, 2, 3, 100, hy.HYENA_BF16, p, None)
    for args in (bad_lf, bad_lg, bad_L, mis):
        assert f(*args) == hy.HYENA_ERR_INVALID_ARG
    assert lib.hyena_striped_featurize(p, p, p, p, p, p, 0, 2, 3, 100, 0, p, p, None) == hy.HYENA_ERR_INVALID_ARG
    assert lib.hyena_filter_exponential(p, p, 0, 3, 100, p, None) == hy.HYENA_ERR_INVALID_ARG
    assert lib.hyena_filter_exponential(p, p, 65, 3, 100, p, None) == hy.HYENA_ERR_INVALID_ARG
    del ok


def test_f16_spectra_queries_and_host_rejections(lib):
    p, mis = ctypes.c_void_p(1 << 20), ctypes.c_void_p((1 << 20) + 8)
    assert lib.hyena_filter_spectrum_bytes_f16(0, 1024) == 0
    assert lib.hyena_filter_spectrum_bytes_f16(4, 1000) == 0
    # bins, per-channel inverse scales (padded to 16 bytes), then the float32
    # block's tables (a length without the tensor-core copy: bins, then tables)
    M = 4096
    f32 = lib.hyena_filter_spectrum_bytes(4, M)
    tables = f32 - 8 * 4 * M
    assert lib.hyena_filter_spectrum_bytes_f16(4, M) == 4 * 4 * M + 16 + tables
    assert lib.hyena_filter_spectrum_to_f16(mis, 4, 1024, p, None) == hy.HYENA_ERR_INVALID_ARG
    assert lib.hyena_filter_spectrum_to_f16(p, 4, 1024, mis, None) == hy.HYENA_ERR_INVALID_ARG
    assert lib.hyena_filter_spectrum_to_f16(p, 0, 1024, p, None) == hy.HYENA_ERR_INVALID_ARG
    assert lib.hyena_filter_spectrum_to_f16(p, 4, 1000, p, None) == hy.HYENA_ERR_UNSUPPORTED
    f = lib.hyena_forward_f16_spectra
    xs = (ctypes.c_void_p * 2)(p, p)
    assert f(p, xs, xs, 1, 1, 1024, 0, 1, p, None, 0, None) == hy.HYENA_ERR_INVALID_ARG
    assert f(p, xs, xs, 1, 1, 1024, 2, 7, p, None, 0, None) == hy.HYENA_ERR_INVALID_ARG
    assert f(mis, xs, xs, 1, 1, 1024, 2, 1, p, None, 0, None) == hy.HYENA_ERR_INVALID_ARG
    assert f(p, xs, xs, 1, 1, 1000, 2, 1, p, None, 0, None) == hy.HYENA_ERR_UNSUPPORTED
    assert f(p, xs, xs, 1, 1, 32768, 2, 1, p, None, 0, None) == hy.HYENA_ERR_WORKSPACE
    # float32 I/O is refused: f16 spectra cannot meet the float32 accuracy
    assert f(p, xs, xs, 1, 1, 1024, 2, hy.HYENA_F32, p, None, 0, None) == hy.HYENA_ERR_UNSUPPORTED
    assert f(p, xs, xs, 1, 1, 32768, 2, hy.HYENA_F32, p, p, 1 << 20, None) == hy.HYENA_ERR_UNSUPPORTED


def test_nd_queries_and_host_rejections(lib):
    p, mis = ctypes.c_void_p(1 << 20), ctypes.c_void_p((1 << 20) + 8)
    I3 = ctypes.c_int * 3
    # [D][P] float2 then the twiddle table (one entry per point of the longest padded axis, at least 2)
    assert lib.hyena_nd_spectrum_bytes(4, 2, I3(64, 64, 0), 0) == 8 * (4 * 128 * 128 + 128)
    assert lib.hyena_nd_spectrum_bytes(4, 2, I3(128, 128, 0), 1) == 8 * (4 * 128 * 128 + 128)
    assert lib.hyena_nd_spectrum_bytes(1, 3, I3(2, 2, 2), 1) == 8 * (8 + 2)
    assert lib.hyena_nd_spectrum_bytes(1, 1, I3(1, 0, 0), 1) == 8 * (1 + 2)
    assert lib.hyena_nd_spectrum_bytes(4, 2, I3(128, 128, 0), 0) == 0      # padded grid above 16384 points
    assert lib.hyena_nd_spectrum_bytes(4, 1, I3(1024, 0, 0), 0) == 0       # padded axis above 1024
    assert lib.hyena_nd_spectrum_bytes(4, 2, I3(12, 16, 0), 0) == 0        # not a power of two
    assert lib.hyena_nd_spectrum_bytes(4, 4, I3(2, 2, 2), 0) == 0          # nd above 3
    assert lib.hyena_nd_spectrum_bytes(4, 2, I3(8, 8, 0), 2) == 0          # unknown boundary
    assert lib.hyena_nd_spectrum_bytes(0, 2, I3(8, 8, 0), 0) == 0
    f = lib.hyena_nd_filter_spectrum
    assert f(mis, 4, 2, I3(8, 8, 0), 0, p, None) == hy.HYENA_ERR_INVALID_ARG
    assert f(p, 4, 2, I3(8, 8, 0), 0, mis, None) == hy.HYENA_ERR_INVALID_ARG
    assert f(p, 4, 2, I3(12, 8, 0), 0, p, None) == hy.HYENA_ERR_UNSUPPORTED
    g = lib.hyena_nd_forward
    xs = (ctypes.c_void_p * 2)(p, p)
    ok = I3(8, 8, 0)
    assert g(p, xs, xs, 1, 1, 2, ok, 0, 0, 0, p, None) == hy.HYENA_ERR_INVALID_ARG
    assert g(p, xs, xs, 1, 1, 2, ok, 0, 2, 7, p, None) == hy.HYENA_ERR_INVALID_ARG
    assert g(mis, xs, xs, 1, 1, 2, ok, 0, 2, 0, p, None) == hy.HYENA_ERR_INVALID_ARG
    assert g(p, xs, xs, 0, 1, 2, ok, 0, 2, 0, p, None) == hy.HYENA_ERR_INVALID_ARG
    assert g(p, xs, xs, 1, 1, 2, I3(8, 6, 0), 0, 2, 0, p, None) == hy.HYENA_ERR_UNSUPPORTED
    assert g(p, xs, xs, 1, 1, 0, ok, 0, 2, 0, p, None) == hy.HYENA_ERR_UNSUPPORTED


def test_header_is_plain_c_and_links_from_c(lib, tmp_path):
    """include/hyena.h compiles as strict C99, and a C program linked against
    the library calls its host-side queries (no device needed)."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    inc = os.path.join(hy._PKG, os.pardir, "include")
    src = tmp_path / "probe.c"
    src.write_text(
        '#include <stdio.h>\n#include "hyena.h"\n'
        "int main(void) {\n"
        "  int dims[2] = {64, 64}, M = 0, M1 = 0, MV = 0;\n"
        "  if (hyena_spectrum_layout(131072, &M, &M1, &MV) != HYENA_OK) return 2;\n"
        '  printf("%d %zu %zu %zu %d %d %d\\n", hyena_abi_version(), hyena_filter_spectrum_bytes(768, 2048),\n'
        "         hyena_filter_spectrum_bytes_f16(768, 2048), hyena_nd_spectrum_bytes(4, 2, dims, HYENA_ND_ZERO),\n"
        "         M, M1, MV);\n"
        "  return 0;\n}\n")
    exe = tmp_path / "probe"
    libdir = os.path.dirname(hy.LIB_PATH)
    r = subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", f"-I{inc}", str(src), "-o",
                        str(exe), f"-L{libdir}", "-lhyena_b200", f"-Wl,-rpath,{libdir}"],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.split()
    I2 = ctypes.c_int * 2
    assert int(out[0]) == hy.abi_version()
    assert int(out[1]) == lib.hyena_filter_spectrum_bytes(768, 2048)
    assert int(out[2]) == lib.hyena_filter_spectrum_bytes_f16(768, 2048)
    assert int(out[3]) == lib.hyena_nd_spectrum_bytes(4, 2, I2(64, 64), 0)
    assert tuple(int(t) for t in out[4:7]) == hy.spectrum_layout(131072)


def test_binding_rejects_short_spectrum_blocks():
    """The binding checks every spectrum block against the bytes the library
    reads for (D, L) before anything reaches the device (CPU tensors here)."""
    import torch
    v = torch.zeros(1, 2, 1 << 19, dtype=torch.bfloat16)
    xs = [torch.zeros_like(v)]
    short = [torch.zeros(hy.filter_spectrum_bytes(2, 1 << 19) - 16, dtype=torch.uint8)]
    for call in (lambda: hy.forward(v, xs, short), lambda: hy.forward_static_workspace(v, xs, short),
                 lambda: hy.backward(v, xs, short, v), lambda: hy.PreparedForward(v, xs, short)):
        with pytest.raises(ValueError, match="spectrum block 0"):
            call()
    short16 = [torch.zeros(hy.load().hyena_filter_spectrum_bytes_f16(2, 1 << 19) - 16, dtype=torch.uint8)]
    with pytest.raises(ValueError, match="spectrum block 0"):
        hy.forward_f16_spectra(v, xs, short16)

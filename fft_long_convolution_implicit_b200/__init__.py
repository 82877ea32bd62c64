"""Hyena order-N forward and backward on B200 (sm_100a): thin Python binding of libhyena_b200.so.

Every function here marshals arguments (torch CUDA tensors -> device
pointers, the current CUDA stream) and calls the C ABI declared in
include/hyena.h; all computation happens in the library's CUDA kernels.
There is no CPU fallback: if the shared library is missing or a call fails,
an exception is raised.

    h    = filter_generate(weights, N, D, L, alpha_lo, alpha_hi)      # [N][D][L] fp32
    hhat = [filter_rfft(h[n]) for n in range(N)]                      # cached spectra
    y    = forward(v, [x1, ..., xN], hhat)                            # [B][D][L]
    dv, dxs, dh = backward(v, [x1, ..., xN], hhat, dy)                # gradients
    grads = filter_backward(weights, N, D, L, alpha_lo, alpha_hi, dh) # FFN weight gradients

    h16  = [spectrum_to_f16(t, D, L) for t in hhat]                   # f16 spectra
    y    = forward_f16_spectra(v, [x1, ..., xN], h16)
    y    = striped_forward(xq, xk, xv, hT, hH, hK, hG)                # q . (hG * (k . v))
    kh   = [nd_filter_spectrum(K[n], dims, "zero") for n in range(N)] # HyenaND kernels
    y    = nd_forward(v, [x1, ..., xN], kh, dims, "zero")             # [B][D][*dims]
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "lib", "libhyena_b200.so")

HYENA_OK, HYENA_ERR_INVALID_ARG, HYENA_ERR_UNSUPPORTED, HYENA_ERR_WORKSPACE, HYENA_ERR_CUDA, HYENA_ERR_TIMEOUT = range(6)
HYENA_F32, HYENA_BF16 = 0, 1

# exported symbols (kept in step with include/hyena.h)
EXPORTS = (
    "hyena_filter_generate", "hyena_filter_spectrum_bytes", "hyena_filter_rfft", "hyena_spectrum_layout",
    "hyena_forward_workspace_bytes", "hyena_forward", "hyena_status_string", "hyena_last_cuda_error",
    "hyena_abi_version", "hyena_forward_static_workspace", "hyena_backward_workspace_bytes", "hyena_backward",
    "hyena_filter_backward_workspace_bytes", "hyena_filter_backward", "hyena_device_timeouts",
    "hyena_striped_forward", "hyena_striped_featurize", "hyena_filter_exponential",
    "hyena_filter_spectrum_bytes_f16", "hyena_filter_spectrum_to_f16", "hyena_forward_f16_spectra",
    "hyena_nd_spectrum_bytes", "hyena_nd_filter_spectrum", "hyena_nd_forward",
)


class HyenaError(RuntimeError):
    def __init__(self, status: int, where: str):
        lib = load()
        msg = lib.hyena_status_string(status).decode()
        if status == HYENA_ERR_CUDA:
            msg += ": " + lib.hyena_last_cuda_error().decode()
        super().__init__(f"{where}: {msg}")
        self.status = status


class FilterGrads(ctypes.Structure):
    _fields_ = [("W1", ctypes.c_void_p), ("b1", ctypes.c_void_p), ("W2", ctypes.c_void_p),
                ("b2", ctypes.c_void_p), ("W3", ctypes.c_void_p), ("b3", ctypes.c_void_p)]


class FilterParams(ctypes.Structure):
    _fields_ = [("W1", ctypes.c_void_p), ("b1", ctypes.c_void_p), ("W2", ctypes.c_void_p),
                ("b2", ctypes.c_void_p), ("W3", ctypes.c_void_p), ("b3", ctypes.c_void_p),
                ("n_bands", ctypes.c_int), ("width", ctypes.c_int)]


_lib = None


def load() -> ctypes.CDLL:
    """Load libhyena_b200.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m fft_long_convolution_implicit_b200.build`")
    l = ctypes.CDLL(LIB_PATH)
    i, sz, P = ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p
    l.hyena_filter_generate.argtypes = [ctypes.POINTER(FilterParams), i, i, i, ctypes.c_float, ctypes.c_float, P, P]
    l.hyena_filter_generate.restype = i
    l.hyena_filter_spectrum_bytes.argtypes = [i, i]
    l.hyena_filter_spectrum_bytes.restype = sz
    l.hyena_filter_rfft.argtypes = [P, i, i, P, P]
    l.hyena_filter_rfft.restype = i
    l.hyena_spectrum_layout.argtypes = [i, ctypes.POINTER(i), ctypes.POINTER(i), ctypes.POINTER(i)]
    l.hyena_spectrum_layout.restype = i
    l.hyena_filter_spectrum_bytes_f16.argtypes = [i, i]
    l.hyena_filter_spectrum_bytes_f16.restype = sz
    l.hyena_filter_spectrum_to_f16.argtypes = [P, i, i, P, P]
    l.hyena_filter_spectrum_to_f16.restype = i
    l.hyena_forward_f16_spectra.argtypes = [P, P, P, i, i, i, i, i, P, P, sz, P]
    l.hyena_forward_f16_spectra.restype = i
    l.hyena_nd_spectrum_bytes.argtypes = [i, i, ctypes.POINTER(i), i]
    l.hyena_nd_spectrum_bytes.restype = sz
    l.hyena_nd_filter_spectrum.argtypes = [P, i, i, ctypes.POINTER(i), i, P, P]
    l.hyena_nd_filter_spectrum.restype = i
    l.hyena_nd_forward.argtypes = [P, P, P, i, i, i, ctypes.POINTER(i), i, i, i, P, P]
    l.hyena_nd_forward.restype = i
    l.hyena_forward_workspace_bytes.argtypes = [i, i, i, i, i]
    l.hyena_forward_workspace_bytes.restype = sz
    l.hyena_forward.argtypes = [P, P, P, i, i, i, i, i, P, P, sz, P]
    l.hyena_forward.restype = i
    l.hyena_forward_static_workspace.argtypes = [P, P, P, i, i, i, i, i, P, P]
    l.hyena_forward_static_workspace.restype = i
    l.hyena_backward_workspace_bytes.argtypes = [i, i, i, i, i]
    l.hyena_backward_workspace_bytes.restype = sz
    l.hyena_backward.argtypes = [P, P, P, P, i, i, i, i, i, P, P, P, P, sz, P]
    l.hyena_backward.restype = i
    l.hyena_filter_backward_workspace_bytes.argtypes = [i, i, i, i, i]
    l.hyena_filter_backward_workspace_bytes.restype = sz
    l.hyena_filter_backward.argtypes = [ctypes.POINTER(FilterParams), i, i, i, ctypes.c_float, ctypes.c_float, P,
                                        ctypes.POINTER(FilterGrads), P, sz, P]
    l.hyena_filter_backward.restype = i
    l.hyena_status_string.argtypes = [i]
    l.hyena_status_string.restype = ctypes.c_char_p
    l.hyena_last_cuda_error.argtypes = []
    l.hyena_last_cuda_error.restype = ctypes.c_char_p
    l.hyena_striped_forward.argtypes = [P, P, P, P, P, P, i, P, i, i, i, i, i, P, P]
    l.hyena_striped_forward.restype = i
    l.hyena_striped_featurize.argtypes = [P, P, P, P, P, P, i, i, i, i, i, P, P, P]
    l.hyena_striped_featurize.restype = i
    l.hyena_filter_exponential.argtypes = [P, P, i, i, i, P, P]
    l.hyena_filter_exponential.restype = i
    l.hyena_device_timeouts.argtypes = []
    l.hyena_device_timeouts.restype = i
    l.hyena_abi_version.argtypes = []
    l.hyena_abi_version.restype = i
    _lib = l
    return l


def _check(status: int, where: str):
    if status != HYENA_OK:
        raise HyenaError(status, where)


def _torch():
    import torch
    return torch


def _stream(stream):
    torch = _torch()
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.float32:
        return HYENA_F32
    if t.dtype == torch.bfloat16:
        return HYENA_BF16
    raise TypeError(f"unsupported activation dtype {t.dtype} (float32 or bfloat16)")


def _dev(t, name):
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")
    return ctypes.c_void_p(t.data_ptr())


def _check_spectra(hhats, D: int, L: int, f16: bool = False):
    """Each spectrum block must hold at least the bytes the library reads for
    (D, L): hyena_filter_spectrum_bytes, or its f16 counterpart."""
    lib = load()
    need = lib.hyena_filter_spectrum_bytes_f16(D, L) if f16 else lib.hyena_filter_spectrum_bytes(D, L)
    if need == 0:
        return   # unsupported (D, L): the library call reports it
    for n, hh in enumerate(hhats):
        have = hh.numel() * hh.element_size()
        if have < need:
            raise ValueError(f"spectrum block {n} holds {have} bytes; (D={D}, L={L}) needs {need}")


# ------------------------------------------------------------------ queries --

def abi_version() -> int:
    return load().hyena_abi_version()


def check_device_timeouts():
    """Raise HyenaError(HYENA_ERR_TIMEOUT) if a bounded device wait ran out
    since the last check (synchronises with the device; clears the flag)."""
    _check(load().hyena_device_timeouts(), "hyena_device_timeouts")


def filter_spectrum_bytes(D: int, L: int) -> int:
    return load().hyena_filter_spectrum_bytes(D, L)


def forward_workspace_bytes(B: int, D: int, L: int, N: int, bf16: bool) -> int:
    return load().hyena_forward_workspace_bytes(B, D, L, N, HYENA_BF16 if bf16 else HYENA_F32)


def backward_workspace_bytes(B: int, D: int, L: int, N: int, bf16: bool) -> int:
    return load().hyena_backward_workspace_bytes(B, D, L, N, HYENA_BF16 if bf16 else HYENA_F32)


def filter_backward_workspace_bytes(N: int, D: int, L: int, n_bands: int = 8, width: int = 64) -> int:
    return load().hyena_filter_backward_workspace_bytes(N, D, L, n_bands, width)


def spectrum_layout(L: int) -> tuple[int, int, int]:
    """(M, M1, MV): bin k < M of channel c sits at float2 index c*M + (k % M1)*MV + k // M1."""
    M, M1, MV = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    _check(load().hyena_spectrum_layout(L, ctypes.byref(M), ctypes.byref(M1), ctypes.byref(MV)),
           "hyena_spectrum_layout")
    return M.value, M1.value, MV.value


# ------------------------------------------------------------------- calls --

def filter_generate(weights: dict, N: int, D: int, L: int, alpha_lo: float, alpha_hi: float,
                    h=None, n_bands: int = 8, stream=None):
    """Implicit filters h [N][D][L] (float32) from FFN weights (CUDA float32
    tensors W1 [H][1+2K], b1, W2 [H][H], b2, W3 [N*D][H], b3)."""
    torch = _torch()
    W1 = weights["W1"]
    dev = W1.device
    if h is None:
        h = torch.empty((N, D, L), dtype=torch.float32, device=dev)
    p = FilterParams(*(ctypes.c_void_p(_dev(weights[k], k).value) for k in ("W1", "b1", "W2", "b2", "W3", "b3")),
                     n_bands, W1.shape[0])
    _check(load().hyena_filter_generate(ctypes.byref(p), N, D, L, alpha_lo, alpha_hi, _dev(h, "h"),
                                        _stream(stream)), "hyena_filter_generate")
    return h


def filter_rfft(h, hhat=None, stream=None):
    """Spectrum block (uint8 CUDA tensor, library order) of one filter h [D][L] float32."""
    torch = _torch()
    D, L = h.shape
    nbytes = filter_spectrum_bytes(D, L)
    if nbytes == 0:
        _check(HYENA_ERR_UNSUPPORTED, "hyena_filter_spectrum_bytes")
    if hhat is None:
        hhat = torch.empty(nbytes, dtype=torch.uint8, device=h.device)
    _check(load().hyena_filter_rfft(_dev(h, "h"), D, L, _dev(hhat, "hhat"), _stream(stream)), "hyena_filter_rfft")
    return hhat


def forward(v, xs, hhats, y=None, workspace=None, stream=None):
    """y = z_{N+1} of the order-N recurrence for v, gates xs[0..N-1] ([B][D][L],
    float32 or bfloat16) and cached spectra hhats[0..N-1]."""
    torch = _torch()
    B, D, L = v.shape
    N = len(xs)
    if len(hhats) != N:
        raise ValueError("need one spectrum per gate")
    _check_spectra(hhats, D, L)
    code = _dtype_code(v)
    for x in xs:
        if x.shape != v.shape or x.dtype != v.dtype:
            raise ValueError("gates must match v in shape and dtype")
    if y is None:
        y = torch.empty_like(v)
    ws_need = forward_workspace_bytes(B, D, L, N, code == HYENA_BF16)
    if workspace is None and ws_need:
        workspace = torch.empty(ws_need, dtype=torch.uint8, device=v.device)
    xarr = (ctypes.c_void_p * N)(*[_dev(x, "x").value for x in xs])
    harr = (ctypes.c_void_p * N)(*[_dev(hh, "hhat").value for hh in hhats])
    ws_ptr = ctypes.c_void_p(workspace.data_ptr()) if workspace is not None else ctypes.c_void_p(0)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(load().hyena_forward(_dev(v, "v"), xarr, harr, B, D, L, N, code, _dev(y, "y"), ws_ptr, ws_bytes,
                                _stream(stream)), "hyena_forward")
    return y


def spectrum_to_f16(hhat, D: int, L: int, hhat16=None, stream=None):
    """f16 copy (uint8 CUDA tensor) of a float32 spectrum block from filter_rfft."""
    torch = _torch()
    nbytes = load().hyena_filter_spectrum_bytes_f16(D, L)
    if nbytes == 0:
        _check(HYENA_ERR_UNSUPPORTED, "hyena_filter_spectrum_bytes_f16")
    if hhat.numel() * hhat.element_size() < filter_spectrum_bytes(D, L):
        raise ValueError("hhat is smaller than a float32 spectrum block for (D, L)")
    if hhat16 is None:
        hhat16 = torch.empty(nbytes, dtype=torch.uint8, device=hhat.device)
    _check(load().hyena_filter_spectrum_to_f16(_dev(hhat, "hhat"), D, L, _dev(hhat16, "hhat16"), _stream(stream)),
           "hyena_filter_spectrum_to_f16")
    return hhat16


def forward_f16_spectra(v, xs, hhats16, y=None, workspace=None, stream=None):
    """forward() with f16 spectrum blocks from spectrum_to_f16."""
    torch = _torch()
    B, D, L = v.shape
    N = len(xs)
    if len(hhats16) != N:
        raise ValueError("need one spectrum per gate")
    _check_spectra(hhats16, D, L, f16=True)
    code = _dtype_code(v)
    for x in xs:
        if x.shape != v.shape or x.dtype != v.dtype:
            raise ValueError("gates must match v in shape and dtype")
    if y is None:
        y = torch.empty_like(v)
    ws_need = forward_workspace_bytes(B, D, L, N, code == HYENA_BF16)
    if workspace is None and ws_need:
        workspace = torch.empty(ws_need, dtype=torch.uint8, device=v.device)
    xarr = (ctypes.c_void_p * N)(*[_dev(x, "x").value for x in xs])
    harr = (ctypes.c_void_p * N)(*[_dev(hh, "hhat16").value for hh in hhats16])
    ws_ptr = ctypes.c_void_p(workspace.data_ptr()) if workspace is not None else ctypes.c_void_p(0)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(load().hyena_forward_f16_spectra(_dev(v, "v"), xarr, harr, B, D, L, N, code, _dev(y, "y"), ws_ptr,
                                            ws_bytes, _stream(stream)), "hyena_forward_f16_spectra")
    return y


def forward_static_workspace(v, xs, hhats, y=None, stream=None):
    """hyena_forward_static_workspace: the long-sequence forward (16384 < L)
    with the library's static device scratch instead of a caller workspace,
    for callers that cannot allocate device memory. Calls whose GPU work
    overlaps race on that scratch; the first call on a device must come
    before any stream capture on it."""
    torch = _torch()
    B, D, L = v.shape
    N = len(xs)
    if len(hhats) != N:
        raise ValueError("need one spectrum per gate")
    _check_spectra(hhats, D, L)
    code = _dtype_code(v)
    if y is None:
        y = torch.empty_like(v)
    xarr = (ctypes.c_void_p * N)(*[_dev(x, "x").value for x in xs])
    harr = (ctypes.c_void_p * N)(*[_dev(hh, "hhat").value for hh in hhats])
    _check(load().hyena_forward_static_workspace(_dev(v, "v"), xarr, harr, B, D, L, N, code, _dev(y, "y"),
                                                 _stream(stream)), "hyena_forward_static_workspace")
    return y


def backward(v, xs, hhats, dy, dv=None, dxs=None, dh=None, workspace=None, stream=None):
    """Gradients of <dy, y> for y = forward(v, xs, hhats): returns (dv, dxs, dh)
    with dv and dxs[n] like v, and dh float32 [N][D][L] (filter gradients
    summed over the batch)."""
    torch = _torch()
    B, D, L = v.shape
    N = len(xs)
    if len(hhats) != N:
        raise ValueError("need one spectrum per gate")
    _check_spectra(hhats, D, L)
    code = _dtype_code(v)
    for t in list(xs) + [dy]:
        if t.shape != v.shape or t.dtype != v.dtype:
            raise ValueError("gates and dy must match v in shape and dtype")
    dv = torch.empty_like(v) if dv is None else dv
    dxs = [torch.empty_like(v) for _ in range(N)] if dxs is None else list(dxs)
    dh = torch.empty((N, D, L), dtype=torch.float32, device=v.device) if dh is None else dh
    need = backward_workspace_bytes(B, D, L, N, code == HYENA_BF16)
    if need == 0:
        _check(HYENA_ERR_INVALID_ARG, "hyena_backward_workspace_bytes")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=v.device)
    xarr = (ctypes.c_void_p * N)(*[_dev(x, "x").value for x in xs])
    harr = (ctypes.c_void_p * N)(*[_dev(hh, "hhat").value for hh in hhats])
    dxarr = (ctypes.c_void_p * N)(*[_dev(t, "dx").value for t in dxs])
    dharr = (ctypes.c_void_p * N)(*[_dev(dh[n], "dh").value for n in range(N)])
    _check(load().hyena_backward(_dev(v, "v"), xarr, harr, _dev(dy, "dy"), B, D, L, N, code, _dev(dv, "dv"),
                                 dxarr, dharr, _dev(workspace, "workspace"),
                                 workspace.numel() * workspace.element_size(), _stream(stream)), "hyena_backward")
    return dv, dxs, dh


def filter_backward(weights: dict, N: int, D: int, L: int, alpha_lo: float, alpha_hi: float, dh,
                    n_bands: int = 8, grads=None, workspace=None, stream=None) -> dict:
    """Gradients of sum(dh * h) w.r.t. the FFN weights (float32 CUDA tensors
    shaped like the weights). dh: float32 [N][D][L]."""
    torch = _torch()
    W1 = weights["W1"]
    keys = ("W1", "b1", "W2", "b2", "W3", "b3")
    if grads is None:
        grads = {k: torch.empty_like(weights[k]) for k in keys}
    width = W1.shape[0]
    need = filter_backward_workspace_bytes(N, D, L, n_bands, width)
    if need == 0:
        _check(HYENA_ERR_INVALID_ARG, "hyena_filter_backward_workspace_bytes")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=W1.device)
    p = FilterParams(*(ctypes.c_void_p(_dev(weights[k], k).value) for k in keys), n_bands, width)
    g = FilterGrads(*(ctypes.c_void_p(_dev(grads[k], "grad " + k).value) for k in keys))
    _check(load().hyena_filter_backward(ctypes.byref(p), N, D, L, alpha_lo, alpha_hi, _dev(dh, "dh"),
                                        ctypes.byref(g), _dev(workspace, "workspace"),
                                        workspace.numel() * workspace.element_size(), _stream(stream)),
           "hyena_filter_backward")
    return grads


def spectrum_natural(hhat, D: int, L: int):
    """View a spectrum block in natural bin order: complex [D][M+1] (torch,
    on the block's device), M = max(L, 128). Index permutation only."""
    torch = _torch()
    M, M1, MV = spectrum_layout(L)
    blk = hhat[: D * M * 8].view(torch.float32).view(D, M, 2)
    k = torch.arange(M, device=hhat.device)
    idx = (k % M1) * MV + k // M1
    nat = blk[:, idx, :]
    out = torch.complex(nat[..., 0], nat[..., 1])
    out = torch.cat([out, torch.zeros(D, 1, dtype=out.dtype, device=out.device)], dim=1)
    out[:, M] = blk[:, 0, 1].to(out.dtype)       # packed Nyquist bin
    out[:, 0] = blk[:, 0, 0].to(out.dtype)
    return out


# ----------------------------------------------------------------- HyenaND --

ND_BOUNDARY = {"zero": 0, "circular": 1}


def _nd_dims(dims):
    dims = tuple(int(d) for d in dims)
    return dims, (ctypes.c_int * len(dims))(*dims)


def nd_spectrum_bytes(D: int, dims, boundary: str) -> int:
    dims, arr = _nd_dims(dims)
    return load().hyena_nd_spectrum_bytes(D, len(dims), arr, ND_BOUNDARY[boundary])


def nd_filter_spectrum(K, dims, boundary: str, khat=None, stream=None):
    """Spectrum block (uint8 CUDA tensor) of one HyenaND kernel K: float32
    [D][grid] (or [D][*dims]) on the grid dims, boundary "zero" or "circular"."""
    torch = _torch()
    dims, arr = _nd_dims(dims)
    D = K.shape[0]
    nbytes = nd_spectrum_bytes(D, dims, boundary)
    if nbytes == 0:
        _check(HYENA_ERR_UNSUPPORTED, "hyena_nd_spectrum_bytes")
    if khat is None:
        khat = torch.empty(nbytes, dtype=torch.uint8, device=K.device)
    _check(load().hyena_nd_filter_spectrum(_dev(K, "K"), D, len(dims), arr, ND_BOUNDARY[boundary], _dev(khat, "khat"),
                                           _stream(stream)), "hyena_nd_filter_spectrum")
    return khat


class PreparedND:
    """hyena_nd_forward with its arguments marshalled once: v and xs are
    [B][D][grid] (or [B][D][*dims]) float32 or bfloat16, khats from
    nd_filter_spectrum; calling it issues the C call only."""

    def __init__(self, v, xs, khats, dims, boundary: str, y=None, stream=None):
        torch = _torch()
        B, D = v.shape[0], v.shape[1]
        N = len(xs)
        if len(khats) != N:
            raise ValueError("need one spectrum per gate")
        code = _dtype_code(v)
        for x in xs:
            if x.shape != v.shape or x.dtype != v.dtype:
                raise ValueError("gates must match v in shape and dtype")
        self.y = torch.empty_like(v) if y is None else y
        self.dims, self._dims = _nd_dims(dims)
        self._keep = (v, list(xs), list(khats))
        self._x = (ctypes.c_void_p * N)(*[_dev(x, "x").value for x in xs])
        self._h = (ctypes.c_void_p * N)(*[_dev(h, "khat").value for h in khats])
        self._args = (_dev(v, "v"), self._x, self._h, B, D, len(self.dims), self._dims, ND_BOUNDARY[boundary], N, code,
                      _dev(self.y, "y"), _stream(stream))
        self._fn = load().hyena_nd_forward

    def __call__(self):
        st = self._fn(*self._args)
        if st != HYENA_OK:
            raise HyenaError(st, "hyena_nd_forward")
        return self.y


def nd_forward(v, xs, khats, dims, boundary: str, y=None, stream=None):
    """HyenaND order-N forward: y = z_{N+1} with z_{n+1} = x_n . (K_n conv z_n)
    on the grid dims (boundary "zero" or "circular")."""
    return PreparedND(v, xs, khats, dims, boundary, y=y, stream=stream)()


class PreparedForward:
    """hyena_forward with its arguments marshalled once (fixed tensors and
    stream); calling it issues the C call only. Keeps host overhead per
    call to a few microseconds for back-to-back launches. With
    f16_spectra=True, hhats are f16 blocks (spectrum_to_f16) and the call is
    hyena_forward_f16_spectra."""

    def __init__(self, v, xs, hhats, y=None, workspace=None, stream=None, f16_spectra: bool = False):
        torch = _torch()
        B, D, L = v.shape
        N = len(xs)
        if len(hhats) != N:
            raise ValueError("need one spectrum per gate")
        _check_spectra(hhats, D, L, f16=f16_spectra)
        code = _dtype_code(v)
        self.y = torch.empty_like(v) if y is None else y
        need = forward_workspace_bytes(B, D, L, N, code == HYENA_BF16)
        if workspace is None and need:
            workspace = torch.empty(need, dtype=torch.uint8, device=v.device)
        self._keep = (v, list(xs), list(hhats), workspace)
        self._x = (ctypes.c_void_p * N)(*[_dev(x, "x").value for x in xs])
        self._h = (ctypes.c_void_p * N)(*[_dev(h, "hhat").value for h in hhats])
        ws_ptr = ctypes.c_void_p(workspace.data_ptr()) if workspace is not None else ctypes.c_void_p(0)
        ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
        self._args = (_dev(v, "v"), self._x, self._h, B, D, L, N, code, _dev(self.y, "y"), ws_ptr, ws_bytes,
                      _stream(stream))
        self._name = "hyena_forward_f16_spectra" if f16_spectra else "hyena_forward"
        self._fn = getattr(load(), self._name)

    def __call__(self):
        st = self._fn(*self._args)
        if st != HYENA_OK:
            raise HyenaError(st, self._name)
        return self.y


class PreparedBackward:
    """hyena_backward with its arguments marshalled once (fixed tensors,
    workspace and stream); calling it issues the C call only."""

    def __init__(self, v, xs, hhats, dy, dv=None, dxs=None, dh=None, workspace=None, stream=None):
        torch = _torch()
        B, D, L = v.shape
        N = len(xs)
        if len(hhats) != N:
            raise ValueError("need one spectrum per gate")
        _check_spectra(hhats, D, L)
        code = _dtype_code(v)
        self.dv = torch.empty_like(v) if dv is None else dv
        self.dxs = [torch.empty_like(v) for _ in range(N)] if dxs is None else list(dxs)
        self.dh = torch.empty((N, D, L), dtype=torch.float32, device=v.device) if dh is None else dh
        need = backward_workspace_bytes(B, D, L, N, code == HYENA_BF16)
        if need == 0:
            _check(HYENA_ERR_INVALID_ARG, "hyena_backward_workspace_bytes")
        if workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=v.device)
        self._keep = (v, list(xs), list(hhats), dy, workspace)
        self._x = (ctypes.c_void_p * N)(*[_dev(x, "x").value for x in xs])
        self._h = (ctypes.c_void_p * N)(*[_dev(h, "hhat").value for h in hhats])
        self._dx = (ctypes.c_void_p * N)(*[_dev(t, "dx").value for t in self.dxs])
        self._dh = (ctypes.c_void_p * N)(*[_dev(self.dh[n], "dh").value for n in range(N)])
        self._args = (_dev(v, "v"), self._x, self._h, _dev(dy, "dy"), B, D, L, N, code, _dev(self.dv, "dv"),
                      self._dx, self._dh, _dev(workspace, "workspace"),
                      workspace.numel() * workspace.element_size(), _stream(stream))
        self._fn = load().hyena_backward

    def __call__(self):
        st = self._fn(*self._args)
        if st != HYENA_OK:
            raise HyenaError(st, "hyena_backward")
        return self.dv, self.dxs, self.dh


def striped_forward(xq, xk, xv, hT, hH, hK, hG, y=None, stream=None):
    """StripedHyena-form operator y = (hT*xq) . (hG * ((hH*xk) . (hK*xv))) with
    causal FIR sums (SE / MR inner filters). x*: [B][D][L] float32 or bfloat16;
    hT, hH, hK: float32 [D][lf]; hG: float32 [D][lg]."""
    torch = _torch()
    B, D, L = xq.shape
    code = _dtype_code(xq)
    for t in (xk, xv):
        if t.shape != xq.shape or t.dtype != xq.dtype:
            raise ValueError("xq, xk, xv must match in shape and dtype")
    lf, lg = hT.shape[1], hG.shape[1]
    y = torch.empty_like(xq) if y is None else y
    _check(load().hyena_striped_forward(_dev(xq, "xq"), _dev(xk, "xk"), _dev(xv, "xv"), _dev(hT, "hT"),
                                        _dev(hH, "hH"), _dev(hK, "hK"), lf, _dev(hG, "hG"), lg, B, D, L, code,
                                        _dev(y, "y"), _stream(stream)), "hyena_striped_forward")
    return y


def striped_featurize(xq, xk, xv, hT, hH, hK, q=None, u=None, stream=None):
    """(q, u) = (hT*xq, (hH*xk) . (hK*xv)) for the long-filter (LI) form:
    y = forward(u, [q], [filter_rfft(hG)])."""
    torch = _torch()
    B, D, L = xq.shape
    code = _dtype_code(xq)
    lf = hT.shape[1]
    q = torch.empty_like(xq) if q is None else q
    u = torch.empty_like(xq) if u is None else u
    _check(load().hyena_striped_featurize(_dev(xq, "xq"), _dev(xk, "xk"), _dev(xv, "xv"), _dev(hT, "hT"),
                                          _dev(hH, "hH"), _dev(hK, "hK"), lf, B, D, L, code, _dev(q, "q"),
                                          _dev(u, "u"), _stream(stream)), "hyena_striped_featurize")
    return q, u


def filter_exponential(R, lam, L: int, h=None, stream=None):
    """Hyena-LI filter h[c][t] = sum_n R[c][n] lam[c][n]^t, float32 [D][L]."""
    torch = _torch()
    D, d = R.shape
    h = torch.empty((D, L), dtype=torch.float32, device=R.device) if h is None else h
    _check(load().hyena_filter_exponential(_dev(R, "R"), _dev(lam, "lambda"), d, D, L, _dev(h, "h"),
                                           _stream(stream)), "hyena_filter_exponential")
    return h


class PreparedStriped:
    """hyena_striped_forward with its arguments marshalled once."""

    def __init__(self, xq, xk, xv, hT, hH, hK, hG, y=None, stream=None):
        torch = _torch()
        B, D, L = xq.shape
        self.y = torch.empty_like(xq) if y is None else y
        self._keep = (xq, xk, xv, hT, hH, hK, hG)
        self._args = (_dev(xq, "xq"), _dev(xk, "xk"), _dev(xv, "xv"), _dev(hT, "hT"), _dev(hH, "hH"),
                      _dev(hK, "hK"), hT.shape[1], _dev(hG, "hG"), hG.shape[1], B, D, L, _dtype_code(xq),
                      _dev(self.y, "y"), _stream(stream))
        self._fn = load().hyena_striped_forward

    def __call__(self):
        st = self._fn(*self._args)
        if st != HYENA_OK:
            raise HyenaError(st, "hyena_striped_forward")
        return self.y

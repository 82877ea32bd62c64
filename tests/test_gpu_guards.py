"""Bounds and initialisation checks of the CUDA path (in place of a memory
sanitizer): every output, spectrum block and workspace is carved out of a
larger buffer whose guard bytes on both sides hold a canary pattern, and
every workspace and spectrum block is prefilled with NaN bytes.

After each call: the guard bytes are unchanged (no write outside the
buffers the call was given), the inputs are unchanged bit for bit, the
outputs are finite (no NaN from a workspace or spectrum byte that was read
before being written), and the outputs equal bit for bit those of the same
call on zero-prefilled buffers.
"""
import numpy as np
import pytest

import synth
from hyena_cases import upload, weights_to_cuda

pytestmark = pytest.mark.gpu

GUARD = 4096          # bytes on each side
CANARY = 0xA5


@pytest.fixture(scope="module")
def hy():
    from fft_long_convolution_implicit_b200 import build
    build.build()
    import fft_long_convolution_implicit_b200 as m
    m.load()
    return m


class Guarded:
    """A byte buffer of `nbytes` (rounded up to 16) between two canary guards."""

    def __init__(self, nbytes, fill):
        import torch
        self.n = (nbytes + 15) // 16 * 16
        self.raw = torch.full((self.n + 2 * GUARD,), CANARY, dtype=torch.uint8, device="cuda")
        self.body = self.raw[GUARD:GUARD + self.n]
        self.body.fill_(fill)

    def view(self, dtype, shape):
        import torch
        elems = int(np.prod(shape))
        return self.body.view(dtype)[:elems].view(*shape)

    def guards_intact(self):
        g = self.raw.cpu().numpy()
        return bool((g[:GUARD] == CANARY).all() and (g[GUARD + self.n:] == CANARY).all())


def run_guarded(hy, w, fill, f16=False):
    """Spectra, workspace and y in guarded buffers; returns (y bytes, guard status, inputs unchanged)."""
    import torch
    wt = synth.filter_weights(w)
    v, xs = synth.inputs(w)
    h = hy.filter_generate(weights_to_cuda(wt), w.N, w.D, w.L, w.alpha_lo, w.alpha_hi)
    specs = []
    for n in range(w.N):
        g = Guarded(hy.filter_spectrum_bytes(w.D, w.L), fill)
        hy.filter_rfft(h[n], hhat=g.body[:hy.filter_spectrum_bytes(w.D, w.L)])
        specs.append(g)
    hh = [g.body[:hy.filter_spectrum_bytes(w.D, w.L)] for g in specs]
    if f16:
        nb = hy.load().hyena_filter_spectrum_bytes_f16(w.D, w.L)
        g16 = [Guarded(nb, fill) for _ in range(w.N)]
        for n in range(w.N):
            hy.spectrum_to_f16(hh[n], w.D, w.L, hhat16=g16[n].body[:nb])
        specs += g16
        hh = [g.body[:nb] for g in g16]
    tv = upload(v, w)
    txs = [upload(x, w) for x in xs]
    before = [t.clone() for t in [tv] + txs]
    ws_bytes = hy.forward_workspace_bytes(w.B, w.D, w.L, w.N, w.dtype == "bf16")
    ws = Guarded(max(ws_bytes, 16), fill)
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    yb = Guarded(w.channels * w.L * (4 if w.dtype == "f32" else 2), fill)
    y = yb.view(dt, (w.B, w.D, w.L))
    fwd = hy.forward_f16_spectra if f16 else hy.forward
    fwd(tv, txs, hh, y=y, workspace=ws.body[:ws_bytes] if ws_bytes else None)
    torch.cuda.synchronize()
    hy.check_device_timeouts()
    intact = all(g.guards_intact() for g in specs) and ws.guards_intact() and yb.guards_intact()
    unchanged = all(torch.equal(a.view(torch.uint8) if a.dtype == torch.bfloat16 else a, b.view(torch.uint8)
                                if b.dtype == torch.bfloat16 else b) for a, b in zip([tv] + txs, before))
    return y.float().cpu().numpy(), y.view(torch.uint8).cpu().numpy().copy(), intact, unchanged


@pytest.mark.parametrize("N,dtype,B,D,L,f16", [
    (2, "f32", 1, 3, 1024, False),       # fused SIMT
    (2, "bf16", 2, 3, 2048, False),      # tensor-core fused
    (3, "bf16", 3, 2, 8192, False),      # fused SIMT, staged spectra
    (3, "bf16", 2, 3, 8192, False),      # tcgen05 GEMM levels
    (2, "f32", 2, 2, 16384, False),      # fused SIMT, 1024 threads per channel
    (2, "bf16", 1, 3, 32768, False),     # four-step
    (2, "bf16", 1, 5, 131072, False),    # four-step, rows of 1024
    (2, "bf16", 1, 3, 524288, False),    # four-step, rows of 4096 on the tensor cores
    (2, "bf16", 2, 2, 8192, True),       # f16 spectra, fused
    (2, "bf16", 1, 2, 65536, True),      # f16 spectra, four-step
])
def test_forward_guards_and_initialisation(hy, N, dtype, B, D, L, f16):
    w = synth.custom(N, dtype, B, D, L, seed=77 + L)
    y_nan, bytes_nan, intact, unchanged = run_guarded(hy, w, 0xFF, f16)
    assert intact, "a guard byte changed: a write outside the given buffers"
    assert unchanged, "an input changed"
    assert np.isfinite(y_nan).all(), "NaN in y: a prefilled byte was read before it was written"
    _, bytes_zero, intact0, _ = run_guarded(hy, w, 0x00, f16)
    assert intact0
    np.testing.assert_array_equal(bytes_nan, bytes_zero)

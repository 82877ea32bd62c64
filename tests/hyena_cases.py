"""Shared helpers of the GPU parity tests: run the CUDA path through the
binding on seeded inputs, run the float64 oracle on the same inputs, and
compare per (b, c) row."""
from __future__ import annotations

import numpy as np

import oracle
import synth

TOL = {"f32": 2e-5, "bf16": 8e-3}


def torch_dtype(dtype: str):
    import torch
    return torch.float32 if dtype == "f32" else torch.bfloat16


def weights_to_cuda(wt: dict):
    import torch
    return {k: torch.from_numpy(np.ascontiguousarray(a)).cuda() for k, a in wt.items()}


def upload(arr: np.ndarray, w: synth.Workload):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(arr)).view(w.B, w.D, w.L)
    return t.to("cuda").to(torch_dtype(w.dtype))


def gpu_run(w: synth.Workload, v=None, xs=None, keep_h: bool = False):
    """Full CUDA pipeline: filter generation, spectra, forward. Returns
    (y as float32 numpy [C][L], h numpy or None, inputs)."""
    import torch
    import fft_long_convolution_implicit_b200 as hy
    wt = synth.filter_weights(w)
    if v is None:
        v, xs = synth.inputs(w)
    tw = weights_to_cuda(wt)
    h = hy.filter_generate(tw, w.N, w.D, w.L, w.alpha_lo, w.alpha_hi)
    hh = [hy.filter_rfft(h[n]) for n in range(w.N)]
    tv = upload(v, w)
    txs = [upload(x, w) for x in xs]
    y = hy.forward(tv, txs, hh)
    torch.cuda.synchronize()
    hy.check_device_timeouts()
    y_np = y.float().cpu().numpy().reshape(w.channels, w.L)
    h_np = h.cpu().numpy() if keep_h else None
    return y_np, h_np, (v, xs, wt)


def oracle_rows(w: synth.Workload, rows, v, xs, wt):
    """float64 oracle y for flat channel rows (b*D + c) of already generated inputs."""
    cs = sorted({r % w.D for r in rows})
    pairs = [(n, c) for n in range(w.N) for c in cs]
    hrows = oracle.implicit_filter(wt, w.N, w.D, w.L, w.alpha_lo, w.alpha_hi, rows=pairs)
    hs = [hrows[n * len(cs):(n + 1) * len(cs)] for n in range(w.N)]
    fr = [cs.index(r % w.D) for r in rows]
    vr = np.asarray(v)[rows]
    xr = [np.asarray(x)[rows] for x in xs]
    return oracle.hyena_forward(vr, xr, hs, filter_row=fr)


def rel_l2_rows(got: np.ndarray, ref: np.ndarray) -> np.ndarray:
    num = np.linalg.norm(got.astype(np.float64) - ref, axis=-1)
    den = np.linalg.norm(ref, axis=-1)
    return np.where(den > 0, num / np.where(den > 0, den, 1), num)


def wave_rows(w: synth.Workload, wave_channels: int, seed: int = 0, min_rows: int = 8) -> list[int]:
    """Rows (b*D + c) that put at least one checked row in every wave of the
    four-step path: channels are taken in waves of `wave_channels` in
    c-major order (channel index c*B + b); rows are drawn (seeded) from every
    wave, enough per wave that at least `min_rows` are drawn in all, and the
    first and last rows are always included."""
    rng = np.random.default_rng(1234 + seed)
    C = w.channels
    waves = -(-C // wave_channels)
    per_wave = max(1, -(-min_rows // waves))
    picks = {0, C - 1}
    for start in range(0, C, wave_channels):
        stop = min(C, start + wave_channels)
        for ch in rng.choice(np.arange(start, stop), size=min(per_wave, stop - start), replace=False):
            c, b = divmod(int(ch), w.B)
            picks.add(b * w.D + c)
    return sorted(picks)

"""Seeded synthetic inputs for the Hyena order-N forward.

This module is the only code shared by the float64 oracle side and the CUDA
side. It holds no arithmetic of the method itself: it draws numbers, rounds
them to the storage type the kernels receive, and describes the workload
shapes. Everything the method computes (filter generation, spectra, causal
convolution, gating) lives separately in ``oracle/`` and in the CUDA library.

Random numbers come from a counter-based generator so that any slice of any
tensor can be regenerated on its own:

* splitmix64 output function (Steele, Lea & Flood, "Fast splittable
  pseudorandom number generators", OOPSLA 2014) applied to
  ``key(seed, tensor_id) + (index + 1) * golden_gamma``;
* uniform doubles in (0, 1) from the top 53 bits;
* standard normals by Box-Muller (cosine branch) from the uniforms at
  counter indices ``2 i`` and ``2 i + 1``.

Tensor ids: 0 = v, n = x_n (n = 1..N), 101..106 = W1, b1, W2, b2, W3, b3,
200 = the 4 x D embedding table E, 201 = the symbol stream, 300 = the loss
gradient dy fed to the backward, 301 = a filter gradient dh fed to the
filter-weight backward on its own, 400..403 = the StripedHyena-form filters
hT, hH, hK, hG, 404/405 = the Hyena-LI exponential weights R and rates lambda.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

GOLDEN_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

TID_V = 0
TID_W1, TID_B1, TID_W2, TID_B2, TID_W3, TID_B3 = 101, 102, 103, 104, 105, 106
TID_EMBED = 200
TID_SYMBOLS = 201
TID_DY = 300
TID_DH = 301


def _mix64(z: np.ndarray) -> np.ndarray:
    """splitmix64 output function on a uint64 array (wrapping arithmetic)."""
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def _stream_key(seed: int, tensor_id: int) -> np.uint64:
    base = np.array([(seed * 0x9E3779B97F4A7C15 + tensor_id) & 0xFFFFFFFFFFFFFFFF],
                    dtype=np.uint64)
    return _mix64(base)[0]


def raw_u64(seed: int, tensor_id: int, start: int, count: int) -> np.ndarray:
    """Counter outputs for indices start .. start+count-1 of one tensor stream."""
    idx = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix64(_stream_key(seed, tensor_id) + idx * GOLDEN_GAMMA)


def uniform(seed: int, tensor_id: int, start: int, count: int) -> np.ndarray:
    """Uniform float64 in the open interval (0, 1)."""
    u = raw_u64(seed, tensor_id, start, count) >> np.uint64(11)
    return (u.astype(np.float64) + 0.5) * (1.0 / 9007199254740992.0)


def normal(seed: int, tensor_id: int, start: int, count: int) -> np.ndarray:
    """Standard normal float64 values for elements start .. start+count-1."""
    u = uniform(seed, tensor_id, 2 * start, 2 * count)
    u1, u2 = u[0::2], u[1::2]
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * math.pi * u2)


def round_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns (uint16), round to nearest even."""
    bits = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    lsb = (bits >> np.uint32(16)) & np.uint32(1)
    with np.errstate(over="ignore"):
        r = (bits + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """bfloat16 bit patterns (uint16) -> exact float32 values."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# --------------------------------------------------------------------------
# Workloads
# --------------------------------------------------------------------------

@dataclass(frozen=True)
class Workload:
    """Shape and input recipe of one Hyena order-N forward workload.

    ``v_kind``: "normal" (N(0,1)) or "onehot4" (one-hot over a uniform
    4-symbol alphabet times a 4 x D N(0,1) table).
    ``x_kind``: "normal" or "sigmoid_normal" (sigmoid of N(0,1)).
    """
    name: str
    N: int
    dtype: str          # "f32" or "bf16": storage type of v, x_n and y
    B: int
    D: int
    L: int
    alpha_lo: float
    alpha_hi: float
    v_kind: str = "normal"
    x_kind: str = "normal"
    seed: int = 1000
    n_bands: int = 8
    width: int = 64

    @property
    def channels(self) -> int:
        return self.B * self.D

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    def roofline_bytes(self) -> int:
        """(N+2) B D L elem + N D (L+1) complex64: every input, output and
        cached filter spectrum touched exactly once."""
        return ((self.N + 2) * self.B * self.D * self.L * self.elem_bytes
                + self.N * self.D * (self.L + 1) * 8)


WORKLOADS = [
    Workload("hyena2_f32_B1_D16_L1024", 2, "f32", 1, 16, 1024, 0.5, 20.0, seed=1000),
    Workload("hyena2_bf16_B4_D768_L2048", 2, "bf16", 4, 768, 2048, 0.5, 20.0, seed=1001),
    Workload("hyena3_bf16_B2_D1024_L8192", 3, "bf16", 2, 1024, 8192, 0.5, 20.0, seed=1002),
    Workload("hyena2_bf16_B1_D256_L131072", 2, "bf16", 1, 256, 131072, 0.1, 10.0,
             x_kind="sigmoid_normal", seed=1003),
    Workload("hyena2_bf16_B1_D256_L1048576", 2, "bf16", 1, 256, 1048576, 0.05, 5.0,
             v_kind="onehot4", seed=1004),
]


def workload(i: int) -> Workload:
    return WORKLOADS[i]


def custom(N: int, dtype: str, B: int, D: int, L: int, alpha_lo: float = 0.5,
           alpha_hi: float = 20.0, seed: int = 7, v_kind: str = "normal",
           x_kind: str = "normal", name: str | None = None) -> Workload:
    return Workload(name or f"custom_N{N}_{dtype}_B{B}_D{D}_L{L}", N, dtype, B, D, L,
                    alpha_lo, alpha_hi, v_kind=v_kind, x_kind=x_kind, seed=seed)


# --------------------------------------------------------------------------
# Generators. Each returns float32 values exactly representable in the
# workload's storage type (bf16-rounded when dtype == "bf16").
# --------------------------------------------------------------------------

def _to_storage_f32(a: np.ndarray, dtype: str) -> np.ndarray:
    a = a.astype(np.float32)
    if dtype == "bf16":
        a = bf16_bits_to_f32(round_to_bf16_bits(a))
    return a


def filter_weights(w: Workload) -> dict[str, np.ndarray]:
    """FFN weights, row-major [out][in], each ~ U(-1/sqrt(fan_in), 1/sqrt(fan_in));
    biases drawn from the same range as their layer's weights."""
    E = 1 + 2 * w.n_bands
    H = w.width
    O = w.N * w.D

    def U(tid, shape, fan_in):
        n = int(np.prod(shape))
        u = uniform(w.seed, tid, 0, n)
        return ((2.0 * u - 1.0) / math.sqrt(fan_in)).astype(np.float32).reshape(shape)

    return {
        "W1": U(TID_W1, (H, E), E), "b1": U(TID_B1, (H,), E),
        "W2": U(TID_W2, (H, H), H), "b2": U(TID_B2, (H,), H),
        "W3": U(TID_W3, (O, H), H), "b3": U(TID_B3, (O,), H),
    }


def _rows(w: Workload, tensor_id: int, rows: list[int] | None, kind: str) -> np.ndarray:
    """Rows (flattened channel index b*D + c) of a [B][D][L] input tensor."""
    L = w.L
    if rows is None:
        rows = list(range(w.channels))
    out = np.empty((len(rows), L), dtype=np.float32)

    if kind == "onehot4":
        table = normal(w.seed, TID_EMBED, 0, 4 * w.D).reshape(4, w.D)

    def fill(i):
        r = rows[i]
        if kind == "normal":
            a = normal(w.seed, tensor_id, r * L, L)
        elif kind == "sigmoid_normal":
            g = normal(w.seed, tensor_id, r * L, L)
            a = 1.0 / (1.0 + np.exp(-g))
        elif kind == "onehot4":
            b, c = divmod(r, w.D)
            sym = (raw_u64(w.seed, TID_SYMBOLS, b * L, L) >> np.uint64(62)).astype(np.int64)
            a = table[sym, c]
        else:
            raise ValueError(kind)
        out[i] = _to_storage_f32(a, w.dtype)

    n = len(rows)
    if n * L >= (1 << 22):
        with ThreadPoolExecutor(max_workers=min(16, os.cpu_count() or 1)) as ex:
            list(ex.map(fill, range(n)))
    else:
        for i in range(n):
            fill(i)
    return out


def v_rows(w: Workload, rows: list[int] | None = None) -> np.ndarray:
    return _rows(w, TID_V, rows, w.v_kind)


def x_rows(w: Workload, n: int, rows: list[int] | None = None) -> np.ndarray:
    """Gate x_n (n = 1..N)."""
    assert 1 <= n <= w.N
    return _rows(w, n, rows, w.x_kind)


def inputs(w: Workload, rows: list[int] | None = None) -> tuple[np.ndarray, list[np.ndarray]]:
    """(v, [x_1..x_N]) as float32 arrays of shape [len(rows)][L]
    (all channels in b-major order when rows is None)."""
    return v_rows(w, rows), [x_rows(w, n, rows) for n in range(1, w.N + 1)]


def dy_rows(w: Workload, rows: list[int] | None = None) -> np.ndarray:
    """Loss gradient dL/dy [len(rows)][L]: N(0,1) in the storage type."""
    return _rows(w, TID_DY, rows, "normal")


def dh_rows(w: Workload) -> np.ndarray:
    """A filter gradient dL/dh, float32 [N][D][L] of N(0,1) values."""
    return normal(w.seed, TID_DH, 0, w.N * w.D * w.L).astype(np.float32).reshape(w.N, w.D, w.L)


def striped_filters(w: Workload, lf: int, lg: int):
    """Featurizers hT, hH, hK: float32 [D][lf] of N(0,1)/sqrt(lf); inner hG:
    float32 [D][lg] of N(0,1)/sqrt(lg) times exp(-4 t / lg) (an MR-style decay)."""
    def nrm(tid, cols, scale):
        return (normal(w.seed, tid, 0, w.D * cols).reshape(w.D, cols) * scale).astype(np.float32)
    hT, hH, hK = (nrm(400 + i, lf, 1 / math.sqrt(lf)) for i in range(3))
    decay = np.exp(-4.0 * np.arange(lg) / lg)
    hG = (nrm(403, lg, 1 / math.sqrt(lg)) * decay).astype(np.float32)
    return hT, hH, hK, hG


def exponential_params(w: Workload, d: int):
    """Hyena-LI weights: R [D][d] of N(0,1)/sqrt(d), rates lambda [D][d]
    uniform in (0.5, 1 - 2/L) (decaying within the sequence)."""
    R = (normal(w.seed, 404, 0, w.D * d).reshape(w.D, d) / math.sqrt(d)).astype(np.float32)
    u = uniform(w.seed, 405, 0, w.D * d).reshape(w.D, d)
    lam = (0.5 + (0.5 - 2.0 / max(w.L, 4)) * u).astype(np.float32)
    return R, lam


def sample_rows(w: Workload, count: int, salt: int = 0) -> list[int]:
    """A fixed, seeded sample of channel rows, always including the first and
    the last channel."""
    C = w.channels
    if count >= C:
        return list(range(C))
    u = raw_u64(w.seed + 7919 * (salt + 1), 999, 0, 4 * count)
    picks = {0, C - 1}
    for val in u:
        if len(picks) >= count:
            break
        picks.add(int(val % np.uint64(C)))
    return sorted(picks)


# --------------------------------------------------------------------------
# HyenaND workloads: the order-N recurrence on a 2-D or 3-D grid. Inputs use
# the 1-D generators on the flattened grid (row-major, last axis contiguous);
# kernels K_n are N(0,1) values under a Gaussian window (the summary's kernel
# carries a learnable Gaussian window), one width per channel.
# --------------------------------------------------------------------------

@dataclass(frozen=True)
class NDWorkload:
    name: str
    N: int
    dtype: str
    B: int
    D: int
    dims: tuple
    boundary: str          # "zero" or "circular"
    gamma_lo: float = 2.0
    gamma_hi: float = 32.0
    seed: int = 1100

    @property
    def grid(self) -> int:
        return int(np.prod(self.dims))

    @property
    def padded(self) -> int:
        return int(np.prod([2 * d if self.boundary == "zero" else d for d in self.dims]))

    @property
    def channels(self) -> int:
        return self.B * self.D

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    def flat(self) -> Workload:
        return Workload(self.name, self.N, self.dtype, self.B, self.D, self.grid, 0.5, 20.0, seed=self.seed)

    def roofline_bytes(self) -> int:
        """(N+2) B D grid elem (v, x_n, y) + N D P complex64 (the cached padded-grid
        spectra), each touched once."""
        return (self.N + 2) * self.B * self.D * self.grid * self.elem_bytes + self.N * self.D * self.padded * 8


ND_WORKLOADS = [
    NDWorkload("hyenand2_f32_B3_D4_8x16_zero", 2, "f32", 3, 4, (8, 16), "zero", seed=1100),
    NDWorkload("hyenand2_bf16_B2_D256_64x64_zero", 2, "bf16", 2, 256, (64, 64), "zero", seed=1101),
    NDWorkload("hyenand2_bf16_B2_D256_128x128_circular", 2, "bf16", 2, 256, (128, 128), "circular", seed=1102),
    NDWorkload("hyenand2_bf16_B2_D256_8x16x16_zero", 2, "bf16", 2, 256, (8, 16, 16), "zero", seed=1103),
    NDWorkload("hyenand2_bf16_B2_D256_16x32x32_circular", 2, "bf16", 2, 256, (16, 32, 32), "circular", seed=1104),
]


def nd_workload(i: int) -> NDWorkload:
    return ND_WORKLOADS[i]


def nd_custom(N: int, dtype: str, B: int, D: int, dims, boundary: str, seed: int = 17) -> NDWorkload:
    dims = tuple(int(d) for d in dims)
    return NDWorkload(f"custom_nd_N{N}_{dtype}_B{B}_D{D}_{'x'.join(map(str, dims))}_{boundary}", N, dtype, B, D,
                      dims, boundary, seed=seed)


def nd_inputs(w: NDWorkload, rows: list[int] | None = None):
    """(v, [x_1..x_N]) as float32 [len(rows)][grid] (storage-rounded)."""
    return inputs(w.flat(), rows)


def nd_kernels(w: NDWorkload) -> np.ndarray:
    """K float32 [N][D][grid]: N(0,1) times exp(-gamma_c sum_a (d_a / L_a)^2),
    d_a the offset along axis a (circular: the periodic distance), gamma_c
    geometric from gamma_lo to gamma_hi over the channels; each kernel scaled
    to unit L2 norm of its window."""
    coords = np.meshgrid(*[np.arange(d, dtype=np.float64) for d in w.dims], indexing="ij")
    r2 = np.zeros(w.dims)
    for a, d in enumerate(w.dims):
        off = coords[a]
        if w.boundary == "circular":
            off = np.minimum(off, d - off)
        r2 += (off / d) ** 2
    r2 = r2.reshape(-1)
    K = np.empty((w.N, w.D, w.grid), dtype=np.float32)
    for c in range(w.D):
        gamma = w.gamma_lo * (w.gamma_hi / w.gamma_lo) ** (c / max(1, w.D - 1))
        win = np.exp(-gamma * r2)
        win /= np.linalg.norm(win)
        for n in range(w.N):
            K[n, c] = normal(w.seed, 500 + n, c * w.grid, w.grid) * win
    return K

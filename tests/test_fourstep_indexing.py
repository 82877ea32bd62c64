"""Bounds and coverage of the global-memory indexing of the four-step kernels
and of the tcgen05 pair kernel, replayed on the CPU over their launch grids
(no GPU; the device sanitizer is not available, so this is the bounds
evidence for their indexing).

For each layout of the four-step path (L = 2^15 .. 2^20, from the library's
own hyena_spectrum_layout), the index formulas of
- col_kernel (csrc/fourstep.cu): input/gate/output elements of a channel row
  and the scratch elements (row n1, column n2) each pass reads and writes, and
- row_kernel (csrc/fourstep.cu): the rows of each CTA's pair and the
  elements of a row each thread reads and writes,
- tcr_row_kernel (csrc/tc_rows.cu): the scratch elements of a row pair each
  thread reads and writes, the spectrum bins of the product and their mirror
  partners, and the row pairs the items of a channel cover,
and of tcg_forward_kernel (csrc/tc_gemm.cu, L = 8192) are enumerated for
every thread of the launch and checked to stay inside the buffers and to
touch every element exactly once. The formulas are restated
from the kernels; a change to a kernel's indexing must be made here too.
"""
import numpy as np
import pytest

import fft_long_convolution_implicit_b200 as hy

LS = [1 << 15, 1 << 16, 1 << 17, 1 << 18, 1 << 19, 1 << 20]


def col_cfg(MB: int):
    """Columns per CTA and threads per CTA of col_kernel<MB> (ColCfg)."""
    CW = 128 if MB == 1 else (64 if MB == 2 else 16)
    return CW, CW * MB


@pytest.mark.parametrize("L", LS)
def test_column_pass_indexing(L):
    M, M1, MV = hy.spectrum_layout(L)
    assert M == L and M1 * MV == M and M1 % 16 == 0
    MB = M1 // 16
    CW, threads = col_cfg(MB)
    assert MV % CW == 0
    gx = MV // CW                                       # grid.x; grid.y = channels of the wave
    tid = np.arange(threads)
    col, j = tid % CW, tid // CW
    bx = np.arange(gx)[:, None]
    n2 = (bx * CW + col[None, :]).ravel()               # column of each (CTA, thread)
    jj = np.broadcast_to(j[None, :], (gx, threads)).ravel()
    assert n2.min() >= 0 and n2.max() < MV

    # first pass reads v, middle and last passes read the gate, the last writes y:
    # element pairs 2m, 2m + 1 of the channel row with m = MV (j + r MB) + n2, r < 8
    m = (MV * (jj[:, None] + np.arange(8)[None, :] * MB) + n2[:, None]).ravel()
    elems = np.concatenate([2 * m, 2 * m + 1])
    assert elems.min() >= 0 and elems.max() < L
    assert np.bincount(elems, minlength=L).tolist() == [1] * L

    # scratch rows read (middle and last passes) and written (first and middle):
    # row j + q MB + 16 r (q < 16 / MB, r < MB) of column n2; MB = 1: row r < 16
    if MB == 1:
        rows = np.arange(16)[None, :].repeat(len(n2), 0)
    else:
        q = np.arange(16 // MB)
        r = np.arange(MB)
        rows = (jj[:, None, None] + q[None, :, None] * MB + 16 * r[None, None, :]).reshape(len(n2), -1)
    idx = (rows * MV + n2[:, None]).ravel()
    assert idx.min() >= 0 and idx.max() < M1 * MV
    assert np.bincount(idx, minlength=M1 * MV).tolist() == [1] * (M1 * MV)


@pytest.mark.parametrize("L", LS)
def test_simt_row_pass_indexing(L):
    """row_kernel (csrc/fourstep.cu): CTA p < M1 / 2 of a channel transforms
    rows kA = p and kB = M1 - p (CTA 0: rows 0 and M1 / 2); its 2 TV threads
    (TV = MV / 16) read and write elements tl + r MV / 16 (r < 16) of their row,
    and the staged spectrum rows are 16-byte aligned bulk copies."""
    M, M1, MV = hy.spectrum_layout(L)
    rows = np.zeros(M1, int)
    for p in range(M1 // 2):
        kA, kB = p, (M1 // 2 if p == 0 else M1 - p)
        rows[kA] += 1
        rows[kB] += 1
        for k in (kA, kB):
            for elem in (8, 4):      # float32 and f16 spectrum rows
                assert (elem * k * MV) % 16 == 0 and (elem * MV) % 16 == 0
    assert rows.tolist() == [1] * M1
    TV = MV // 16
    idx = (np.arange(TV)[:, None] + np.arange(16)[None, :] * (MV // 16)).ravel()
    assert idx.min() >= 0 and idx.max() < MV
    assert np.bincount(idx, minlength=MV).tolist() == [1] * MV


def tcr_items(M1: int):
    """(kA, kB, kind) of the items of one channel (tcr_row_kernel)."""
    out = []
    for q in range(M1 // 2 + 1):
        if q < M1 // 2 - 1:
            out.append((q + 1, M1 - q - 1, 0))
        elif q == M1 // 2 - 1:
            out.append((0, 0, 1))
        else:
            out.append((M1 // 2, M1 // 2, 2))
    return out


@pytest.mark.parametrize("L", [1 << 19, 1 << 20])
def test_tensor_row_pass_indexing(L):
    M, M1, MV = hy.spectrum_layout(L)
    assert MV == 4096
    # the items cover every row of the channel once: a mirror pair (kA, M1 - kA),
    # or a self-mirrored row 0 or M1/2 as its own item
    seen = np.zeros(M1, int)
    for kA, kB, kind in tcr_items(M1):
        assert 0 <= kA < M1 and 0 <= kB < M1
        seen[kA] += 1
        if kind == 0:
            assert kA + kB == M1
            seen[kB] += 1
    assert seen.tolist() == [1] * M1

    tid = np.arange(128)
    w, l = tid >> 5, tid & 31
    # scratch row elements (input of F1, output of I1): m0 + 8 t + 256 n3 with
    # m0 = (l & 7) + 16 n2f, n2f = ((l >> 3) & 3) + 4 w, t < 2, n3 < 16
    n2f = ((l >> 3) & 3) + 4 * w
    m0 = (l & 7) + 16 * n2f
    idx = (m0[:, None, None] + 8 * np.arange(2)[None, :, None] + 256 * np.arange(16)[None, None, :]).ravel()
    assert idx.min() >= 0 and idx.max() < MV
    assert np.bincount(idx, minlength=MV).tolist() == [1] * MV

    # spectrum bins of the product: j = (l & 7) + 8 t + 16 k2 + 256 (8 h + e), k2 = ((l >> 3) & 3) + 4 w;
    # partners MV - 1 - j (mirror pair, and row M1/2) or (MV - j) mod MV (row 0)
    k2 = ((l >> 3) & 3) + 4 * w
    j = ((l & 7)[:, None, None, None] + 8 * np.arange(2)[None, :, None, None] + 16 * k2[:, None, None, None]
         + 256 * (8 * np.arange(2)[None, None, :, None] + np.arange(8)[None, None, None, :])).ravel()
    assert np.bincount(j, minlength=MV).tolist() == [1] * MV
    for partner in ((MV - 1 - j), (MV - j) & (MV - 1)):
        assert partner.min() >= 0 and partner.max() < MV
        assert np.bincount(partner, minlength=MV).tolist() == [1] * MV

    # staged spectrum rows: one or two rows of MV f16x2 words (16 KB each) at word
    # offset c M + kA MV of the f16 copy, 16-byte aligned for the bulk copies
    for kA, kB, kind in tcr_items(M1):
        for k in ((kA, kB) if kind == 0 else (kA,)):
            off_bytes = 4 * k * MV
            assert off_bytes % 16 == 0 and off_bytes + 4 * MV <= 4 * M


def test_tcgen05_pair_kernel_indexing():
    """tcg_forward_kernel (csrc/tc_gemm.cu, L = 8192, 256 threads, warp w, lane
    l, q = w & 3, hw = w >> 2): the times t = l + 128 w + 32 i + 1024 n3
    (i < 4, n3 < 8) of its v / gate loads and y stores, and the spectrum-copy
    words (128 hw + 32 q + l + 256 t) * 32 + 16 hn + 4 k + e (t, hn < 2, k, e < 4)
    of its product, each cover their row exactly once; 1 / f_c sits after the
    2L words, inside the copy's row of 4 * 2L + 16 bytes."""
    L = 8192
    P = 2 * L
    tid = np.arange(256)
    w, l = tid >> 5, tid & 31
    q, hw = w & 3, w >> 2
    t = (l[:, None, None] + 128 * w[:, None, None] + 32 * np.arange(4)[None, :, None]
         + 1024 * np.arange(8)[None, None, :]).ravel()
    assert t.min() >= 0 and t.max() < L
    assert np.bincount(t, minlength=L).tolist() == [1] * L
    r = 128 * hw + 32 * q + l
    words = ((r[:, None, None, None, None] + 256 * np.arange(2)[None, :, None, None, None]) * 32
             + 16 * np.arange(2)[None, None, :, None, None] + 4 * np.arange(4)[None, None, None, :, None]
             + np.arange(4)[None, None, None, None, :]).ravel()
    assert words.min() >= 0 and words.max() < P
    assert np.bincount(words, minlength=P).tolist() == [1] * P
    row_bytes = 4 * P + 16
    assert 4 * P + 4 <= row_bytes and row_bytes % 16 == 0

"""The tcgen05 forward (bf16 I/O, B even, L = 8192, order N <= 3): every DFT
level of the 2L-point pair transform is a GEMM on the tensor cores (f16
operands scaled by exact powers of two, float32 accumulation in TMEM).

Checked through the binding (C ABI) against the float64 oracle on every row
of small shapes (orders 1 to 3 with even B; odd B and orders 4 to 8 run the
float32 SIMT kernel, whose results are checked the same way), its
spectrum copy against the oracle spectrum, its dispatch (one launch of the
tcgen05 kernel per forward, read from a CUDA-graph capture), exact
power-of-two scaling, and the cleared timeout flag. The full-size workload at
this length (order 3, B = 2, D = 1024) is covered by the workload tests of
test_gpu_parity.py, which run the same dispatch.
"""
import numpy as np
import pytest

import oracle
import synth
from hyena_cases import TOL, gpu_run, oracle_rows, rel_l2_rows, upload, weights_to_cuda

pytestmark = pytest.mark.gpu

L = 8192


@pytest.fixture(scope="module", autouse=True)
def hy():
    from fft_long_convolution_implicit_b200 import build
    build.build()
    import fft_long_convolution_implicit_b200 as m
    m.load()
    return m


@pytest.mark.parametrize("N,B,D", [(1, 2, 3), (2, 2, 2), (3, 2, 3), (4, 4, 2), (2, 6, 1), (8, 2, 1), (3, 3, 2)])
def test_forward_matches_oracle(hy, N, B, D):
    w = synth.custom(N, "bf16", B, D, L, seed=100 + N + 7 * B)
    y, _, (v, xs, wt) = gpu_run(w)
    rows = list(range(w.channels))
    ref = oracle_rows(w, rows, v, xs, wt)
    err = rel_l2_rows(y, ref)
    print(f"N={N} B={B} D={D}: max rel-L2 {err.max():.3e}")
    assert err.max() <= TOL["bf16"], err.max()


def _kernel_names(hy, w, tv, txs, hh):
    """Names of the kernels one forward launches (CUDA-graph capture)."""
    import torch
    import cuda.bindings.driver as dr
    y = torch.empty_like(tv)
    side = torch.cuda.Stream()
    with torch.cuda.stream(side):
        hy.forward(tv, txs, hh, y=y, stream=side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph(keep_graph=True)
    with torch.cuda.graph(g, stream=side, capture_error_mode="relaxed"):
        hy.forward(tv, txs, hh, y=y, stream=side)
    graph = dr.CUgraph(init_value=g.raw_cuda_graph())
    err, _, n = dr.cuGraphGetNodes(graph, 0)
    err, nodes, n = dr.cuGraphGetNodes(graph, n)
    names = []
    for nd in nodes[:n]:
        err, t = dr.cuGraphNodeGetType(nd)
        if t != dr.CUgraphNodeType.CU_GRAPH_NODE_TYPE_KERNEL:
            continue
        err, prm = dr.cuGraphKernelNodeGetParams(nd)
        assert err == dr.CUresult.CUDA_SUCCESS, err
        err, name = dr.cuFuncGetName(prm.func)
        assert err == dr.CUresult.CUDA_SUCCESS, err
        names.append(name.decode() if isinstance(name, bytes) else str(name))
    g.reset()
    return names


@pytest.mark.parametrize("N,B,expect", [(2, 2, "tcg_forward_kernel"), (3, 4, "tcg_forward_kernel"),
                                         (2, 3, "fused_forward_kernel"), (4, 2, "fused_forward_kernel")])
def test_dispatch(hy, N, B, expect):
    w = synth.custom(N, "bf16", B, 2, L, seed=3)
    wt = synth.filter_weights(w)
    v, xs = synth.inputs(w)
    h = hy.filter_generate(weights_to_cuda(wt), w.N, w.D, w.L, w.alpha_lo, w.alpha_hi)
    hh = [hy.filter_rfft(h[n]) for n in range(w.N)]
    names = _kernel_names(hy, w, upload(v, w), [upload(x, w) for x in xs], hh)
    assert len(names) == 1 and expect in names[0], names


def test_spectrum_copy_matches_oracle(hy):
    """The copy holds f_c H[k] as f16 pairs in F3-row order: word r * 32 + k1
    of channel c is bin k = k3 + 16 k2 + 512 k1 of row r = 128 T + p with
    k3 = 8 (T & 1) + ((p >> 2) & 7), k2 = (p & 3) + 4 (p >> 5) + 16 (T >> 1),
    followed by 1 / f_c (a power of two) as float32."""
    import torch
    D = 3
    rng = np.random.default_rng(8)
    h = (rng.standard_normal((D, L)) * np.exp(-np.arange(L) / 1500.0)).astype(np.float32)
    hh = hy.filter_rfft(torch.from_numpy(h).cuda())
    M = L
    row_bytes = 8 * (L + 2)
    base = 8 * D * M
    blk = hh.cpu().numpy()
    idx = np.arange(2 * L)
    r, k1 = idx >> 5, idx & 31
    T, p = r >> 7, r & 127
    k3 = 8 * (T & 1) + ((p >> 2) & 7)
    k2 = (p & 3) + 4 * (p >> 5) + 16 * (T >> 1)
    k = k3 + 16 * k2 + 512 * k1
    assert sorted(k.tolist()) == list(range(2 * L))
    for c in range(D):
        row = blk[base + c * row_bytes: base + (c + 1) * row_bytes]
        words = row[: 8 * L].view(np.float16).astype(np.float64)
        got = words[0::2] + 1j * words[1::2]
        inv_f = float(row[8 * L: 8 * L + 4].view(np.float32)[0])
        assert inv_f > 0 and np.log2(inv_f) == np.round(np.log2(inv_f))
        top = np.abs(np.concatenate([got.real, got.imag])).max()
        assert 2.0 ** 14 <= top < 2.0 ** 15, top
        half = oracle.filter_spectrum(h[c])               # k = 0..L
        full = np.concatenate([half, np.conj(half[1:L][::-1])])
        ref = full[k]
        err = np.linalg.norm(got * inv_f - ref) / np.linalg.norm(ref)
        assert err < 5e-4, (c, err)


def test_power_of_two_scaling_and_timeouts(hy):
    """Scaling v by 4 scales y by exactly 4 (the operand scaling is by exact
    powers of two and sees the same mantissas); no bounded wait ran out."""
    import torch
    w = synth.custom(3, "bf16", 2, 4, L, seed=21)
    wt = synth.filter_weights(w)
    v, xs = synth.inputs(w)
    h = hy.filter_generate(weights_to_cuda(wt), w.N, w.D, w.L, w.alpha_lo, w.alpha_hi)
    hh = [hy.filter_rfft(h[n]) for n in range(w.N)]
    tv = upload(v, w)
    txs = [upload(x, w) for x in xs]
    y1 = hy.forward(tv, txs, hh)
    y4 = hy.forward(tv * 4, txs, hh)
    y1b = hy.forward(tv, txs, hh)
    torch.cuda.synchronize()
    hy.check_device_timeouts()
    assert torch.equal(y1, y1b)
    assert torch.equal(y4, y1 * 4)


@pytest.mark.parametrize("L,D", [(1 << 19, 3), (1 << 20, 2)])
def test_row_pass_spectrum_copy(hy, L, D):
    """Rows of 4096 (L = 2^19, 2^20): the spectrum block ends with each
    channel's largest spectrum component ([D] float, padded to 16 bytes) and
    an f16 copy of the bins ([D][L] __half2); the copy is f_c times the
    float32 bins rounded to nearest, f_c the power of two that puts the
    channel's largest component in [2^14, 2^15)."""
    import torch
    rng = np.random.default_rng(L + D)
    h = (rng.standard_normal((D, L)) * np.exp(-np.arange(L) / (L / 8))).astype(np.float32)
    hh = hy.filter_rfft(torch.from_numpy(h).cuda())
    torch.cuda.synchronize()
    blk = hh.cpu().numpy()
    assert blk.size == hy.filter_spectrum_bytes(D, L)
    half = blk[blk.size - 4 * D * L:].view(np.float16).reshape(D, 2 * L)
    hmax_at = blk.size - 4 * D * L - 16 * ((D + 3) // 4)
    hmax = blk[hmax_at: hmax_at + 4 * D].view(np.float32)
    bins = blk[: 8 * D * L].view(np.float32).reshape(D, 2 * L)
    for c in range(D):
        top = np.abs(bins[c]).max()
        assert hmax[c] == top, (c, hmax[c], top)
        f_c = 2.0 ** (14 - np.floor(np.log2(top)))
        assert 2.0 ** 14 <= top * f_c < 2.0 ** 15
        want = (bins[c].astype(np.float64) * f_c).astype(np.float32).astype(np.float16)
        assert np.array_equal(half[c].view(np.uint16), want.view(np.uint16)), c

#!/usr/bin/env python
"""Benchmark of the Hyena order-N forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--config I]
                    [--pass forward|backward]

A step is one hyena_forward over one batch of the workload (default: the
largest one-GPU workload, order 2, bf16, B=1, D=256, L=2^20), with the filter
spectra already cached (they depend only on the weights; filter generation
and the spectrum are timed on their own and reported beside the line, not in
it). Inputs are resident in HBM when the
timed region starts and are rotated over enough buffer sets that the step's
working set is not in L2. The metric is B*D*L processed per second (x1e9)
and the fraction of the HBM roofline; one JSON line is printed by rank 0.

--gpus N > 1 runs under torchrun: every rank processes its own batch
(weak scaling, no collective on the data path); time is the max over ranks.
--impl reference times the float64 CPU oracle (rank 0 only): every one of
its W warm-up and K timed steps is one pass of the oracle over the same
bounded sample of rows of the workload, sized so the whole run takes a few
minutes; its config is the one the GPU arm prints.
The e2e figure times steps through the public API with every step's inputs
copied in from pinned host memory and its result copied back; forward,
striped and ND steps rotate over three CUDA streams so that one step's
copies overlap its neighbours' kernels (the backward, which shares one
workspace, runs its steps on one stream).
--pass backward times hyena_backward instead (dv, dx_n and dh_n from a loss
gradient dy), same workload and conventions; its roofline counts the bytes
the gradients must move at least: v, x_n, dy and the spectra in, dv, dx_n
and dh_n out.
--pass striped times the StripedHyena-form operator q . (hG * (k . v)) with
Hyena-SE filters (featurizers of 4 taps, inner filter of 7) on the workload's
B, D, L: three inputs and one output of B*D*L elements each.
--pass nd times the HyenaND forward (order-N recurrence with a 2-D or 3-D
convolution, circular or zero-padded) on the ND workload --nd-config I; the
metric counts B*D*grid points per second, the roofline v, x_n, y and the
padded-grid spectra.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

METRIC = "Hyena order-N fwd B·D·L/s (×1e9) and % of HBM roofline, 1 B200"
METRIC_BWD = "Hyena order-N bwd B·D·L/s (×1e9) and % of HBM roofline, 1 B200"
METRIC_STRIPED = "StripedHyena-SE fwd B·D·L/s (×1e9) and % of HBM roofline, 1 B200"
METRIC_ND = "HyenaND order-N fwd B·D·grid/s (×1e9) and % of HBM roofline, 1 B200"
UNIT_ND = "1e9 B*D*grid/s"
STRIPED_LF, STRIPED_LG = 4, 7
UNIT = "1e9 B*D*L/s"
KERNEL_SOURCES = os.path.join(ROOT, "fft_long_convolution_implicit_b200", "csrc")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 2 ** 20


# sources the dominant kernel of each path is compiled from
KERNEL_FILES = {
    "fused": ("fused.cu", "fft_engine.cuh", "paired.cuh", "layout.h"),
    "fourstep": ("fourstep.cu", "tc_rows.cu", "tcgen05.cuh", "mbar.cuh", "fft_engine.cuh", "paired.cuh", "layout.h",
                 "api.cu"),   # api.cu sizes the waves, which set the DRAM traffic
    "tc": ("tc_fused.cu", "tc_dft.cuh", "fft_engine.cuh", "layout.h"),
    "tcg": ("tc_gemm.cu", "tcgen05.cuh", "mbar.cuh", "fft_engine.cuh", "layout.h"),
}


def dominant_kernel(w: synth.Workload, spec16: bool = False) -> tuple[str, str]:
    """(kernel name, source set) of the launch that dominates one forward."""
    if w.L > 16384:
        return "four-step column/row kernels (whole step)", "fourstep"
    if spec16:
        return "fused_forward_kernel (f16 spectra)", "fused"
    if w.dtype == "bf16" and w.B % 2 == 0 and 1024 <= w.L <= 2048:
        return "tc_forward_kernel", "tc"
    if w.dtype == "bf16" and w.B % 2 == 0 and w.L == 8192:
        return "tcg_forward_kernel", "tcg"
    return "fused_forward_kernel", "fused"


def backward_bytes(w: synth.Workload) -> int:
    """Algorithmic bytes of one backward: v, x_1..x_N and dy read, dv and
    dx_1..x_N written (storage type), the N spectra read (8 B per bin, as in
    the forward), the N float32 filter gradients written."""
    return ((2 * w.N + 3) * w.channels * w.L * w.elem_bytes + w.N * w.D * (w.L + 1) * 8
            + 4 * w.N * w.D * w.L)


def count_kernel_nodes(make_call) -> int:
    """Kernels one call launches: capture it (on a side stream) into a CUDA
    graph and count the kernel nodes."""
    import torch
    import cuda.bindings.runtime as rt
    side = torch.cuda.Stream()
    fn = make_call(side)
    with torch.cuda.stream(side):
        fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph(keep_graph=True)
    with torch.cuda.graph(g, stream=side, capture_error_mode="relaxed"):
        fn()
    graph = rt.cudaGraph_t(init_value=g.raw_cuda_graph())
    err, _, n = rt.cudaGraphGetNodes(graph, 0)
    err, nodes, n = rt.cudaGraphGetNodes(graph, n)
    kernel = rt.cudaGraphNodeType.cudaGraphNodeTypeKernel
    count = sum(1 for nd in nodes[:n] if rt.cudaGraphNodeGetType(nd)[1] == kernel)
    g.reset()
    return count


def kernel_source_sha(path: str = "fused") -> str:
    h = hashlib.sha256()
    for fn in KERNEL_FILES[path]:
        with open(os.path.join(KERNEL_SOURCES, fn), "rb") as f:
            h.update(fn.encode() + f.read())
    return h.hexdigest()[:16]


def hbm_peak():
    try:
        with open(PEAKS_FILE) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def measured_traffic(workload_name: str):
    """DRAM bytes per launch of the dominant kernel from a committed ncu
    capture, or None when absent or taken on different kernel sources."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
        e = t.get(workload_name)
        if e and e.get("source_sha") == kernel_source_sha(e.get("path", "fused")):
            return int(e["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


# ------------------------------------------------------------ clocks -----

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
            os.close(fd)
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        loaded = [s for s in sm if smax and s > 0.5 * max(smax)] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": reasons, "samples": len(rows)}


# ------------------------------------------------------- replica helpers --

def rank_workload(w: synth.Workload, rank: int) -> synth.Workload:
    """Every rank processes its own batch of the same shape (weak scaling):
    same workload, inputs seeded per rank."""
    return synth.Workload(**{**w.__dict__, "seed": w.seed + 7919 * rank})


def default_steps(torch, step, stream, target_s: float = 20.0) -> int:
    """Timed steps when --steps is not given: enough for about target_s
    seconds of timed work, from the mean of three untimed steps (at least 20,
    at most 20000). Under several ranks the smallest count is taken (a MIN
    all-reduce before the timed region), so that every rank times the same
    number of steps."""
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for i in range(3):
        step(i)
    b.record(stream)
    torch.cuda.synchronize()
    per = max(a.elapsed_time(b) / 3.0, 1e-3) * 1e-3
    k = int(min(20000, max(20, target_s / per)))
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        t = torch.tensor([k], device=torch.device("cuda", torch.cuda.current_device()), dtype=torch.int64)
        dist.all_reduce(t, op=dist.ReduceOp.MIN)
        k = int(t.item())
    return k


def max_over_ranks(value: float, dist, device) -> float:
    """Max of a per-rank float over all ranks (identity without a process group)."""
    if dist is None or not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(value)
    import torch
    t = torch.tensor([float(value)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_throughput(units_per_rank: float, world: int, elapsed_ms: float) -> float:
    """Units processed by all ranks / max-over-ranks elapsed time, in 1e9 units/s."""
    return units_per_rank * world / (elapsed_ms * 1e-3) / 1e9


# ----------------------------------------------------------- oracle arm --

def oracle_sample(w: synth.Workload, target_core_seconds: float = 12.0, backward: bool = False):
    """Time the float64 oracle (as it stands) on a bounded sample of rows of
    the workload; filters are computed beforehand and not timed."""
    import oracle
    threads = host_cores()
    wt = synth.filter_weights(w)

    def run(rows, n_threads):
        v, xs = synth.inputs(w, rows)
        cs = sorted({r % w.D for r in rows})
        hrows = oracle.implicit_filter(wt, w.N, w.D, w.L, w.alpha_lo, w.alpha_hi,
                                       rows=[(n, c) for n in range(w.N) for c in cs], threads=threads)
        hs = [hrows[n * len(cs):(n + 1) * len(cs)] for n in range(w.N)]
        fr = [cs.index(r % w.D) for r in rows]
        dy = synth.dy_rows(w, rows) if backward else None
        t0 = time.perf_counter()
        if backward:
            oracle.hyena_backward(v, xs, hs, dy, filter_row=fr, threads=n_threads)
        else:
            oracle.hyena_forward(v, xs, hs, filter_row=fr, threads=n_threads)
        return time.perf_counter() - t0

    # calibrate on one row, then size the sample for ~target core-seconds
    per_row = max(run([0], 1), 1e-4)
    nrows = int(min(w.channels, max(threads, target_core_seconds / per_row)))
    dt = run(list(range(nrows)), threads)
    value = nrows * w.L / dt / 1e9
    what = "backward (forward again, then gradients)" if backward else "forward"
    sample = (f"{nrows} of {w.channels} (b,c) rows of {w.name}, {what}, all N={w.N} stages, "
              f"{'direct O(L^2)' if w.L <= 8192 else 'radix-2 FFT'} causal sums, filters precomputed")
    return {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample,
            "seconds": dt}


def oracle_passes(w: synth.Workload, steps: int, warmup: int, backward: bool = False,
                  striped: bool = False, budget_s: float = 120.0):
    """Reference arm: `warmup` untimed and `steps` timed passes of the float64
    oracle (as it stands) over one bounded sample of rows of the workload,
    one row per host core at least; every pass recomputes the whole sample.
    The sample is sized so that all passes take about budget_s seconds of
    wall time. Returns (seconds of each timed pass, rows per pass, cores)."""
    import oracle
    threads = host_cores()
    if striped:
        hT, hH, hK, hG = synth.striped_filters(w, STRIPED_LF, STRIPED_LG)
    else:
        wt = synth.filter_weights(w)

    def prepare(rows):
        if striped:
            xv, (xq, xk) = synth.inputs(synth.Workload(**{**w.__dict__, "N": 2}), rows)
            fr = [r % w.D for r in rows]
            return lambda n_threads: oracle.striped_forward(xq, xk, xv, hT, hH, hK, hG, filter_row=fr,
                                                            threads=n_threads)
        v, xs = synth.inputs(w, rows)
        cs = sorted({r % w.D for r in rows})
        hrows = oracle.implicit_filter(wt, w.N, w.D, w.L, w.alpha_lo, w.alpha_hi,
                                       rows=[(n, c) for n in range(w.N) for c in cs], threads=threads)
        hs = [hrows[n * len(cs):(n + 1) * len(cs)] for n in range(w.N)]
        fr = [cs.index(r % w.D) for r in rows]
        dy = synth.dy_rows(w, rows) if backward else None
        if backward:
            return lambda n_threads: oracle.hyena_backward(v, xs, hs, dy, filter_row=fr, threads=n_threads)
        return lambda n_threads: oracle.hyena_forward(v, xs, hs, filter_row=fr, threads=n_threads)

    one = prepare([0])
    t0 = time.perf_counter()
    one(1)
    per_row = max(time.perf_counter() - t0, 1e-5)
    per_pass = max(per_row, budget_s / max(1, steps + warmup))
    nrows = int(min(w.channels, threads * max(1, int(per_pass / per_row))))
    run = prepare(list(range(nrows)))
    for _ in range(warmup):
        run(threads)
    times = []
    for _ in range(steps):
        t0 = time.perf_counter()
        run(threads)
        times.append(time.perf_counter() - t0)
    return times, nrows, threads


def oracle_striped_sample(w: synth.Workload, target_core_seconds: float = 8.0):
    """The float64 StripedHyena-form oracle on a bounded sample of rows."""
    import oracle
    threads = host_cores()
    hT, hH, hK, hG = synth.striped_filters(w, STRIPED_LF, STRIPED_LG)

    def run(rows, n_threads):
        xv, (xq, xk) = synth.inputs(synth.Workload(**{**w.__dict__, "N": 2}), rows)
        t0 = time.perf_counter()
        oracle.striped_forward(xq, xk, xv, hT, hH, hK, hG, filter_row=[r % w.D for r in rows], threads=n_threads)
        return time.perf_counter() - t0

    per_row = max(run([0], 1), 1e-5)
    nrows = int(min(w.channels, max(threads, target_core_seconds / per_row)))
    dt = run(list(range(nrows)), threads)
    return {"value": nrows * w.L / dt / 1e9, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{nrows} of {w.channels} (b,c) rows, StripedHyena-SE (lf={STRIPED_LF}, lg={STRIPED_LG}), "
                      f"direct FIR sums", "seconds": dt}


E2E_SLOTS = 3


def pipelined_e2e(torch, dev, main_stream, pinned_in, make_slot, steps, world, dist):
    """Device time (ms, max over ranks) of `steps` end-to-end steps through the
    public API, rotated over E2E_SLOTS CUDA streams: step i runs on slot
    i % E2E_SLOTS and copies its pinned host inputs into that slot's device
    buffers, makes the library call, and copies the result into that slot's
    pinned host buffers. Every step moves all of its inputs in and its result
    out; the rotation lets one step's uploads overlap its neighbours' kernels
    and downloads (each direction has its own copy engine).
    make_slot(stream) -> (device input tensors, call returning the outputs,
    pinned host output tensors)."""
    slots = []
    for _ in range(E2E_SLOTS):
        st = torch.cuda.Stream(device=dev)
        slots.append((st, make_slot(st)))

    def step(i):
        st, (dins, call, pouts) = slots[i % E2E_SLOTS]
        with torch.cuda.stream(st):
            for d, p in zip(dins, pinned_in):
                d.copy_(p, non_blocking=True)
            for p, o in zip(pouts, call()):
                p.copy_(o, non_blocking=True)

    for i in range(3 * E2E_SLOTS):
        step(i)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(main_stream)
    for st, _ in slots:
        st.wait_event(e0)
    for i in range(steps):
        step(i)
    for st, _ in slots:
        done = torch.cuda.Event()
        done.record(st)
        main_stream.wait_event(done)
    e1.record(main_stream)
    torch.cuda.synchronize()
    return max_over_ranks(e0.elapsed_time(e1), dist if world > 1 else None, dev)


def oracle_nd_sample(w: "synth.NDWorkload", target_core_seconds: float = 8.0):
    """The float64 HyenaND oracle (numpy FFT, one thread) on a bounded sample of rows."""
    import oracle
    K = synth.nd_kernels(w)

    def run(rows):
        v, xs = synth.nd_inputs(w, rows)
        t0 = time.perf_counter()
        oracle.hyena_nd_forward(v, xs, [K[n] for n in range(w.N)], w.dims, w.boundary,
                                filter_row=[r % w.D for r in rows])
        return time.perf_counter() - t0

    per_row = max(run([0]), 1e-5)
    nrows = int(min(w.channels, max(1, target_core_seconds / per_row)))
    dt = run(list(range(nrows)))
    return {"value": nrows * w.grid / dt / 1e9, "unit": UNIT_ND, "cores": 1, "kind": "oracle",
            "sample": f"{nrows} of {w.channels} (b,c) rows of {w.name}, all N={w.N} stages, numpy FFT "
                      f"({w.boundary} boundary)", "seconds": dt}


def nd_rotation(w: "synth.NDWorkload") -> tuple[int, int]:
    """(bytes of one ND input set, number of sets rotated over): the step's algorithmic bytes set the size."""
    set_bytes = w.roofline_bytes()
    nsets = max(2, math.ceil(3 * L2_BYTES / set_bytes)) if set_bytes < 3 * L2_BYTES else 1
    return set_bytes, nsets


def nd_config(w: "synth.NDWorkload", world: int) -> dict:
    """The config dict both arms print for an ND workload."""
    set_bytes, nsets = nd_rotation(w)
    return {"workload": w.name, "B": w.B, "D": w.D, "dims": list(w.dims), "boundary": w.boundary, "N": w.N,
            "io": w.dtype, "pass": "nd", "global_batch": w.B * world, "parallelism": f"replicas x{world}",
            "l2": (f"inputs rotated over {nsets} buffer sets of {set_bytes / 2**20:.0f} MiB "
                   f"(> L2 {L2_BYTES / 2**20:.0f} MiB between reuses)") if nsets > 1 else
                  f"inputs of {set_bytes / 2**20:.0f} MiB per step, larger than L2"}


def run_nd(args) -> int:
    w = synth.nd_workload(args.nd_config)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank != 0:
            return 0
        if args.steps is None:
            args.steps = 20
        import oracle
        K = synth.nd_kernels(w)

        def prepare(rows):
            v, xs = synth.nd_inputs(w, rows)
            fr = [r % w.D for r in rows]
            return lambda: oracle.hyena_nd_forward(v, xs, [K[n] for n in range(w.N)], w.dims, w.boundary,
                                                   filter_row=fr)

        one = prepare([0])
        t0 = time.perf_counter()
        one()
        per_row = max(time.perf_counter() - t0, 1e-5)
        per_pass = max(per_row, 120.0 / max(1, args.steps + args.warmup))
        nrows = int(min(w.channels, max(1, int(per_pass / per_row))))
        run = prepare(list(range(nrows)))
        for _ in range(args.warmup):
            run()
        times = []
        for _ in range(args.steps):
            t0 = time.perf_counter()
            run()
            times.append(time.perf_counter() - t0)
        mean_s = statistics.mean(times)
        value = nrows * w.grid / mean_s / 1e9
        sample = (f"each of the {args.steps} timed steps (after {args.warmup} warm-up steps) is one oracle pass over "
                  f"the same {nrows} of {w.channels} (b,c) rows of {w.name}, all N={w.N} stages, numpy FFT "
                  f"({w.boundary} boundary), one thread")
        print(json.dumps({"impl": "reference", "metric": METRIC_ND, "value": value, "unit": UNIT_ND,
                          "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                          "ms_per_step": mean_s * 1e3, "higher_is_better": True,
                          "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                          "config": nd_config(w, world),
                          "cpu_baseline": {"value": value, "unit": UNIT_ND, "cores": 1, "kind": "oracle",
                                           "sample": sample},
                          "e2e": {"value": value, "unit": UNIT_ND, "h2d_bytes_per_step": 0,
                                  "d2h_bytes_per_step": 0}}))
        return 0

    import torch
    import torch.distributed as dist
    import fft_long_convolution_implicit_b200 as hy
    from fft_long_convolution_implicit_b200 import build as hybuild

    if world > 1:
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    else:
        torch.cuda.set_device(0)
    if rank == 0:
        hybuild.build()
    if world > 1:
        dist.barrier()
    hy.load()
    dev = torch.device("cuda", local_rank if world > 1 else 0)
    stream = torch.cuda.current_stream(dev)
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    wr = synth.NDWorkload(**{**w.__dict__, "seed": w.seed + 7919 * rank})
    v_np, xs_np = synth.nd_inputs(wr)
    K = synth.nd_kernels(wr)
    base_v = torch.from_numpy(v_np).view(w.B, w.D, w.grid).to(dev).to(dt)
    base_x = [torch.from_numpy(x).view(w.B, w.D, w.grid).to(dev).to(dt) for x in xs_np]
    base_k = [hy.nd_filter_spectrum(torch.from_numpy(K[n]).to(dev), w.dims, w.boundary) for n in range(w.N)]
    set_bytes, nsets = nd_rotation(w)
    sets = []
    for i in range(nsets):
        if i == 0:
            v_s, x_s, k_s = base_v, base_x, base_k
        else:
            v_s, x_s, k_s = base_v.clone(), [x.clone() for x in base_x], [t.clone() for t in base_k]
        sets.append(hy.PreparedND(v_s, x_s, k_s, w.dims, w.boundary, stream=stream))
    torch.cuda.synchronize()
    launches_per_step = count_kernel_nodes(lambda st: hy.PreparedND(base_v, base_x, base_k, w.dims, w.boundary,
                                                                    stream=st))
    for i in range(args.warmup):
        sets[i % nsets]()
    torch.cuda.synchronize()
    if args.steps is None:
        args.steps = default_steps(torch, lambda i: sets[i % nsets](), stream)
    sampler = ClockSampler(local_rank if world > 1 else 0)
    sampler.start()
    time.sleep(0.2)
    K_steps = args.steps
    ev_pre = [torch.cuda.Event(enable_timing=True) for _ in range(K_steps)]
    ev_post = [torch.cuda.Event(enable_timing=True) for _ in range(K_steps)]
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    start.record(stream)
    for i in range(K_steps):
        ev_pre[i].record(stream)
        sets[i % nsets]()
        ev_post[i].record(stream)
    end.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    elapsed_ms = max_over_ranks(start.elapsed_time(end), dist if world > 1 else None, dev)
    value = whole_job_throughput(K_steps * w.channels * w.grid, world, elapsed_ms)
    kernel_ms = statistics.mean(a.elapsed_time(b) for a, b in zip(ev_pre, ev_post))
    peak, peak_kind = hbm_peak()
    alg_bytes = w.roofline_bytes()
    achieved = alg_bytes / (kernel_ms * 1e-3) / 1e9

    # end to end: pinned host inputs in, y out, through the same public call
    pinned_in = [base_v.cpu().pin_memory()] + [x.cpu().pin_memory() for x in base_x]

    def nd_slot(st):
        dv = torch.empty_like(base_v)
        dxs = [torch.empty_like(x) for x in base_x]
        call = hy.PreparedND(dv, dxs, base_k, w.dims, w.boundary, stream=st)
        return [dv, *dxs], lambda: [call()], [torch.empty_like(pinned_in[0]).pin_memory()]

    if args.e2e_steps is None:
        args.e2e_steps = int(min(200, max(5, 4e9 // ((w.N + 2) * w.channels * w.grid * w.elem_bytes))))
    e2e_ms = pipelined_e2e(torch, dev, stream, pinned_in, nd_slot, args.e2e_steps, world, dist)
    e2e_value = whole_job_throughput(args.e2e_steps * w.channels * w.grid, world, e2e_ms)
    line = None
    if rank == 0:
        line = {
            "metric": METRIC_ND, "value": round(value, 4), "unit": UNIT_ND, "n_gpus": world, "steps": K_steps,
            "warmup": args.warmup, "ms_per_step": elapsed_ms / K_steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": nd_config(w, world),
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(achieved / peak, 4), "traffic": None, "peak_kind": peak_kind,
                         "alg_bytes_per_launch": alg_bytes, "kernel": "nd_forward_kernel",
                         "kernel_ms": round(kernel_ms, 5)},
            "e2e": {"value": round(e2e_value, 4), "unit": UNIT_ND,
                    "h2d_bytes_per_step": (w.N + 1) * w.channels * w.grid * w.elem_bytes,
                    "d2h_bytes_per_step": w.channels * w.grid * w.elem_bytes, "ms_per_step": e2e_ms / args.e2e_steps,
                    "streams": E2E_SLOTS},
            "gpu_launches": K_steps * launches_per_step,
            "clocks": clocks,
        }
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        if not args.no_cpu_baseline and world == 1:
            cb = oracle_nd_sample(w)
            line["cpu_baseline"] = {k: round(cb[k], 6) if k == "value" else cb[k]
                                    for k in ("value", "unit", "cores", "kind", "sample")}
        elif not args.no_cpu_baseline:
            line["cpu_baseline"] = None
        print(json.dumps(line))
    return 0


# ------------------------------------------------------ shared config --

def rotation(w: synth.Workload, which: str) -> tuple[int, int]:
    """(bytes of one input set, number of sets) the timed steps rotate over
    so that a set is not in L2 when it is reused: the step's algorithmic
    bytes (activations and spectra) set the size."""
    if which == "striped":
        set_bytes = 4 * w.channels * w.L * w.elem_bytes
    else:
        set_bytes = w.roofline_bytes() + (w.channels * w.L * w.elem_bytes if which == "backward" else 0)
    nsets = max(2, math.ceil(3 * L2_BYTES / set_bytes)) if set_bytes < 3 * L2_BYTES else 1
    return set_bytes, nsets


def run_config(w: synth.Workload, which: str, spec16: bool, world: int) -> dict:
    """The config dict both arms print for a workload."""
    set_bytes, nsets = rotation(w, which)
    if nsets > 1:
        l2 = (f"inputs rotated over {nsets} buffer sets of {set_bytes / 2**20:.0f} MiB "
              f"(> L2 {L2_BYTES / 2**20:.0f} MiB between reuses)")
    else:
        l2 = f"inputs of {set_bytes / 2**20:.0f} MiB per step, larger than L2 ({L2_BYTES / 2**20:.0f} MiB)"
    return {"workload": w.name, "B": w.B, "D": w.D, "L": w.L, "N": w.N, "io": w.dtype, "pass": which,
            "spectra": "f16" if spec16 else "f32", "global_batch": w.B * world,
            "parallelism": f"replicas x{world}", "l2": l2}


def filter_timings(torch, hy, tw, h, specs, w: synth.Workload, stream, reps: int = 3) -> dict:
    """CUDA-event times of hyena_filter_generate (all N filters) and of
    hyena_filter_rfft (all N spectra) on the step's stream, best of `reps`
    after one warm-up call each. They run once per weights, so they are
    reported beside the line and not counted in its value."""
    def best(fn):
        fn()
        torch.cuda.synchronize()
        out = []
        for _ in range(reps):
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize()
            out.append(a.elapsed_time(b))
        return min(out)

    gen_ms = best(lambda: hy.filter_generate(tw, w.N, w.D, w.L, w.alpha_lo, w.alpha_hi, h=h, stream=stream))
    rfft_ms = best(lambda: [hy.filter_rfft(h[n], hhat=specs[n], stream=stream) for n in range(w.N)])
    flops = filter_gen_flops(w)
    peak_tf = None
    try:
        with open(PEAKS_FILE) as f:
            peak_tf = float(json.load(f)["bf16_tflops"])
    except Exception:
        pass
    gen_tf = flops / (gen_ms * 1e-3) / 1e12
    return {"excluded_from_value": True, "generate_ms": round(gen_ms, 4), "rfft_ms": round(rfft_ms, 4),
            "generate_flops": flops, "generate_tflops": round(gen_tf, 2),
            "generate_frac_of_bf16_peak": round(gen_tf / peak_tf, 4) if peak_tf else None,
            "generate_arithmetic": "float32 SIMT (CUDA cores)",
            "rfft_bytes": w.N * w.D * w.L * 4 + w.N * w.D * (w.L + 1) * 8}


def filter_gen_flops(w: synth.Workload) -> int:
    """Multiply-add flops of the implicit-filter FFN over all L taps: two
    hidden layers of width `width` and the output layer of N*D."""
    e = 1 + 2 * w.n_bands
    return 2 * w.L * (e * w.width + w.width * w.width + w.width * w.N * w.D)


# ---------------------------------------------------------------- main --

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: enough for about 20 s of timed work, 20 to 20000)")
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--config", type=int, default=4,
                    help="workload index (default 4: the largest one-GPU workload, B=1 D=256 L=2^20 N=2 bf16)")
    ap.add_argument("--e2e-steps", type=int, default=None,
                    help="end-to-end steps (default: enough for about 4 GB of host copies, 5 to 200)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--pass", dest="which", choices=["forward", "backward", "striped", "nd"], default="forward")
    ap.add_argument("--nd-config", type=int, default=1, help="HyenaND workload index for --pass nd")
    ap.add_argument("--shape", default=None,
                    help="N,dtype,B,D,L: a custom shape instead of --config (small ncu captures)")
    ap.add_argument("--spectrum", choices=["f32", "f16"], default="f32",
                    help="forward pass: cached filter spectra as float32 (default) or f16 blocks")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.which == "nd":
        return run_nd(args)
    bwd = args.which == "backward"
    striped = args.which == "striped"
    metric = METRIC_BWD if bwd else (METRIC_STRIPED if striped else METRIC)
    if args.warmup < 3:
        args.warmup = 3

    if args.shape:
        n_, dt_, b_, d_, l_ = args.shape.split(",")
        w = synth.custom(int(n_), dt_, int(b_), int(d_), int(l_))
    else:
        w = synth.workload(args.config)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    spec16 = args.spectrum == "f16" and args.which == "forward"
    if args.impl == "reference" and args.steps is None:
        args.steps = 20
    if args.impl == "reference":
        if rank != 0:
            return 0
        times, nrows, cores = oracle_passes(w, args.steps, args.warmup, backward=bwd, striped=striped)
        mean_s = statistics.mean(times)
        value = nrows * w.L / mean_s / 1e9
        what = ("StripedHyena-SE (lf=%d, lg=%d), direct FIR sums" % (STRIPED_LF, STRIPED_LG) if striped else
                ("backward (forward again, then gradients)" if bwd else "forward") + f", all N={w.N} stages, " +
                ("direct O(L^2)" if w.L <= 8192 else "radix-2 FFT") + " causal sums, filters precomputed")
        sample = (f"each of the {args.steps} timed steps (after {args.warmup} warm-up steps) is one oracle pass "
                  f"over the same {nrows} of {w.channels} (b,c) rows of {w.name}: {what}")
        line = {"impl": "reference", "metric": metric, "value": value, "unit": UNIT, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": mean_s * 1e3,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic", "config": run_config(w, args.which, spec16, world),
                "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
                "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return 0

    import torch
    import torch.distributed as dist
    import fft_long_convolution_implicit_b200 as hy
    from fft_long_convolution_implicit_b200 import build as hybuild

    if world > 1:
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    else:
        torch.cuda.set_device(0)
    if rank == 0:
        hybuild.build()
    if world > 1:
        dist.barrier()
    hy.load()
    dev = torch.device("cuda", local_rank if world > 1 else 0)
    stream = torch.cuda.current_stream(dev)
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16

    # inputs of this rank (seeded per rank), weights and cached spectra
    wr = rank_workload(w, rank)
    if striped and w.N < 2:
        wr = synth.Workload(**{**wr.__dict__, "N": 2})
    v_np, xs_np = synth.inputs(wr)
    wt = synth.filter_weights(wr)
    tw = {k: torch.from_numpy(np.ascontiguousarray(a)).to(dev) for k, a in wt.items()}
    h = hy.filter_generate(tw, w.N, w.D, w.L, w.alpha_lo, w.alpha_hi)
    base_v = torch.from_numpy(v_np).view(w.B, w.D, w.L).to(dev).to(dt)
    base_x = [torch.from_numpy(x).view(w.B, w.D, w.L).to(dev).to(dt) for x in xs_np]
    base_h = [hy.filter_rfft(h[n]) for n in range(w.N)]
    # filter generation and the spectrum (once per weights): timed on their own, outside the line's value
    filters = filter_timings(torch, hy, tw, h, base_h, w, stream)
    if spec16:
        base_h = [hy.spectrum_to_f16(t, w.D, w.L) for t in base_h]
    del h
    base_dy = (torch.from_numpy(synth.dy_rows(wr)).view(w.B, w.D, w.L).to(dev).to(dt) if bwd else None)
    set_bytes, nsets = rotation(w, args.which)
    shared_out = None
    if bwd:
        # one set of outputs and one workspace, shared by every input set
        first = hy.PreparedBackward(base_v, base_x, base_h, base_dy, stream=stream)
        shared_out = (first.dv, first.dxs, first.dh, first._keep[4])

    if striped:
        sf = [torch.from_numpy(np.ascontiguousarray(a)).to(dev)
              for a in synth.striped_filters(wr, STRIPED_LF, STRIPED_LG)]

    def prepared(v_s, x_s, h_s, dy_s, st):
        if striped:
            return hy.PreparedStriped(x_s[0], x_s[1], v_s, *sf, stream=st)
        if bwd:
            dv_, dxs_, dh_, ws_ = shared_out
            return hy.PreparedBackward(v_s, x_s, h_s, dy_s, dv=dv_, dxs=dxs_, dh=dh_, workspace=ws_, stream=st)
        return hy.PreparedForward(v_s, x_s, h_s, stream=st, f16_spectra=spec16)

    sets = []
    for s in range(nsets):
        if s == 0:
            v_s, x_s, h_s, dy_s = base_v, base_x, base_h, base_dy
        else:
            v_s, x_s, h_s = base_v.clone(), [x.clone() for x in base_x], [t.clone() for t in base_h]
            dy_s = base_dy.clone() if bwd else None
        sets.append(prepared(v_s, x_s, h_s, dy_s, stream))
    torch.cuda.synchronize()
    launches_per_step = count_kernel_nodes(lambda st: prepared(base_v, base_x, base_h, base_dy, st))

    # warm-up
    for i in range(args.warmup):
        sets[i % nsets]()
    torch.cuda.synchronize()
    if args.steps is None:
        args.steps = default_steps(torch, lambda i: sets[i % nsets](), stream)

    sampler = ClockSampler(local_rank if world > 1 else 0)
    sampler.start()
    time.sleep(0.2)
    K = args.steps
    ev_pre = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    ev_post = [torch.cuda.Event(enable_timing=True) for _ in range(K)]
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    start.record(stream)
    for i in range(K):
        ev_pre[i].record(stream)
        sets[i % nsets]()
        ev_post[i].record(stream)
    end.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    elapsed_ms = start.elapsed_time(end)
    step_ms = [a.elapsed_time(b) for a, b in zip(ev_pre, ev_post)]
    elapsed_ms = max_over_ranks(elapsed_ms, dist if world > 1 else None, dev)
    value = whole_job_throughput(K * w.channels * w.L, world, elapsed_ms)
    kernel_ms = statistics.mean(step_ms)
    peak, peak_kind = hbm_peak()
    if bwd:
        alg_bytes = backward_bytes(w)
    elif striped:
        alg_bytes = 4 * w.channels * w.L * w.elem_bytes + 4 * w.D * (3 * STRIPED_LF + STRIPED_LG)
    else:
        alg_bytes = w.roofline_bytes()
        if spec16:
            # the spectra are read as 4-byte f16 pairs instead of 8-byte float2
            alg_bytes -= 4 * w.N * w.D * (w.L + 1)
    achieved = alg_bytes / (kernel_ms * 1e-3) / 1e9

    # end to end through the public API: pinned host inputs in, result out
    if args.e2e_steps is None:
        copy_bytes = (w.N + 2 + (2 * w.N + 2 if bwd else 0)) * w.channels * w.L * w.elem_bytes
        args.e2e_steps = int(min(200, max(5, 4e9 // copy_bytes)))
    pin_v = base_v.cpu().pin_memory()
    pin_x = [x.cpu().pin_memory() for x in base_x]
    dv = torch.empty_like(base_v)
    dxs = [torch.empty_like(x) for x in base_x]
    if bwd:
        pin_dy = base_dy.cpu().pin_memory()
        ddy = torch.empty_like(base_dy)
        dv_s, dxs_s, dh_s, ws_s = shared_out
        pin_out = [torch.empty_like(dv_s, device="cpu").pin_memory()] + \
                  [torch.empty_like(t, device="cpu").pin_memory() for t in dxs_s] + \
                  [torch.empty_like(dh_s, device="cpu").pin_memory()]
        e2e_call = hy.PreparedBackward(dv, dxs, sets[0]._keep[2], ddy, dv=dv_s, dxs=dxs_s, dh=dh_s,
                                       workspace=ws_s, stream=stream)
        h2d = (w.N + 2) * w.channels * w.L * w.elem_bytes
        d2h = (w.N + 1) * w.channels * w.L * w.elem_bytes + 4 * w.N * w.D * w.L
    elif striped:
        h2d = 3 * w.channels * w.L * w.elem_bytes
        d2h = w.channels * w.L * w.elem_bytes
    else:
        h2d = (w.N + 1) * w.channels * w.L * w.elem_bytes
        d2h = w.channels * w.L * w.elem_bytes

    def slot(st):
        sv = torch.empty_like(base_v)
        sxs = [torch.empty_like(x) for x in base_x]
        if striped:
            call = hy.PreparedStriped(sxs[0], sxs[1], sv, *sf, stream=st)
        else:
            call = hy.PreparedForward(sv, sxs, sets[0]._keep[2], stream=st, f16_spectra=spec16)
        return [sv, *sxs], lambda: [call()], [torch.empty_like(pin_v).pin_memory()]

    def e2e_step():
        dv.copy_(pin_v, non_blocking=True)
        for d, p in zip(dxs, pin_x):
            d.copy_(p, non_blocking=True)
        ddy.copy_(pin_dy, non_blocking=True)
        gdv, gdxs, gdh = e2e_call()
        for p, t in zip(pin_out, [gdv, *gdxs, gdh]):
            p.copy_(t, non_blocking=True)

    if bwd:
        # one workspace and one set of outputs: the steps run back to back on one stream
        for _ in range(3):
            e2e_step()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), dist if world > 1 else None, dev)
    else:
        e2e_ms = pipelined_e2e(torch, dev, stream, [pin_v, *pin_x], slot, args.e2e_steps, world, dist)
    e2e_value = whole_job_throughput(args.e2e_steps * w.channels * w.L, world, e2e_ms)

    line = None
    if rank == 0:
        line = {
            "metric": metric, "value": round(value, 4), "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": elapsed_ms / K, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": run_config(w, args.which, spec16, world),
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(achieved / peak, 4),
                         "traffic": None if (bwd or striped or spec16) else measured_traffic(w.name),
                         "peak_kind": peak_kind, "alg_bytes_per_launch": alg_bytes,
                         "kernel": ("whole backward step (all its launches)" if bwd else
                                    ("striped_kernel (fused FIR)" if striped else dominant_kernel(w, spec16)[0])),
                         "kernel_ms": round(kernel_ms, 5)},
            "e2e": {"value": round(e2e_value, 4), "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / args.e2e_steps,
                    "streams": 1 if bwd else E2E_SLOTS},
            "gpu_launches": K * launches_per_step,
            "clocks": clocks,
        }
        if not striped:
            line["filters"] = filters
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        if not args.no_cpu_baseline and world == 1:
            cb = oracle_striped_sample(w) if striped else oracle_sample(w, backward=bwd)
            line["cpu_baseline"] = {k: round(cb[k], 6) if k == "value" else cb[k]
                                    for k in ("value", "unit", "cores", "kind", "sample")}
        elif not args.no_cpu_baseline:
            line["cpu_baseline"] = None
        print(json.dumps(line))
    return 0


if __name__ == "__main__":
    sys.exit(main())

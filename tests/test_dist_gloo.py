"""Multi-rank (replica) logic of bench.py on CPU with gloo, world size 2.

Every (b, c) channel is independent, so N GPUs run N replicas on their own
batches with no collective on the data path; the only collectives are the
barrier and the max over ranks of the elapsed time."""
import json
import os
import socket
import subprocess
import sys
from datetime import timedelta

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    import synth
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        elapsed = 10.0 + 5.0 * rank                     # rank 1 is the slow one
        mx = bench.max_over_ranks(elapsed, dist, torch.device("cpu"))
        w = bench.rank_workload(synth.workload(1), rank)
        v, _ = synth.inputs(w, rows=[0])
        value = bench.whole_job_throughput(100 * w.channels * w.L, world, mx)
        dist.barrier()
        q.put((rank, mx, w.seed, float(v[0, 0]), value))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_per_rank_inputs():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    (r0, mx0, seed0, v0, val0), (r1, mx1, seed1, v1, val1) = res
    assert mx0 == mx1 == 15.0                          # the max over ranks, on every rank
    assert seed0 != seed1 and v0 != v1                 # each rank has its own batch
    import synth
    w = synth.workload(1)
    assert val0 == val1 == pytest.approx(100 * w.channels * w.L * 2 / 15e-3 / 1e9)


def test_single_process_helpers_without_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, None, None) == 3.5
    assert bench.whole_job_throughput(2e9, 4, 1000.0) == pytest.approx(8.0)


def test_reference_arm_under_torchrun_two_ranks():
    """Rank 0 alone times the oracle and prints the line; rank 1 exits 0."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl", "reference",
           "--gpus", "2", "--steps", "3", "--warmup", "3"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["e2e"]["h2d_bytes_per_step"] == 0

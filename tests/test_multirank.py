"""The multi-rank (replicas only) path of bench.py, on CPU with two gloo ranks.

Attention heads and batches are independent, so N GPUs run N replicas of the
workload with no collective on the data path; the only collectives are the
barrier and the max-over-ranks of the step time.  These tests run that host
logic with world size 2 over gloo, and launch the reference arm under torchrun.
"""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        sys.path.insert(0, ROOT)
        import attn_inputs
        import bench
        w = attn_inputs.WORKLOADS["c1"]
        # each rank draws its own replica, deterministically
        q = attn_inputs.draw(w.B, w.N, w.H, w.d, w.dtype, bench.replica_seed(w, rank), 1)[0]
        q2 = attn_inputs.draw(w.B, w.N, w.H, w.d, w.dtype, bench.replica_seed(w, rank), 1)[0]
        assert torch.equal(q, q2)
        digest = float(q.float().sum())
        # the step time reported by every rank is the slowest rank's
        local_ms = 1.0 + 2.5 * rank
        got = bench.max_over_ranks(local_ms, dist, "cpu")
        sums = [torch.zeros(1) for _ in range(world)]
        dist.all_gather(sums, torch.tensor([digest]))
        out[rank] = (got, [float(x) for x in sums])
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_replicas_and_max_timing():
    world = 2
    mgr = mp.get_context("spawn").Manager()  # no fork after the oracle started threads
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    for r in range(world):
        got, digests = out[r]
        assert got == 1.0 + 2.5 * (world - 1)
        assert digests[0] != digests[1]  # replicas hold different batches


def test_job_throughput_counts_every_rank():
    import bench
    assert bench.job_tflops(1e12, 1000.0, 1) == pytest.approx(1.0)
    assert bench.job_tflops(1e12, 1000.0, 4) == pytest.approx(4.0)


def test_reference_arm_under_torchrun_prints_one_line():
    import oracle
    oracle.build()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py",
           "--impl", "reference", "--gpus", "2", "--workload", "c1", "--steps", "1",
           "--warmup", "3"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["cpu_baseline"]["kind"] == "oracle"
    assert line["unit"] == "TFLOP/s" and line["e2e"]["h2d_bytes_per_step"] == 0
    assert np.isfinite(line["value"]) and line["value"] > 0

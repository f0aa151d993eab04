"""The N > 1 host logic of bench.py on CPU ranks (gloo, world size 2).

The path has no exchange step, so N GPUs run N independent replicas; what the
ranks share is the timing: a barrier around the timed region and the slowest
rank's time.  These tests run that logic on CPU ranks, and launch the reference
arm under torchrun to check that only rank 0 prints and every rank exits 0.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        sys.path.insert(0, ROOT)
        import bench
        dist.barrier()
        elapsed = [3.5, 7.25][rank]                    # each rank's own device time
        results[rank] = bench._max_over_ranks(elapsed, True, torch.device("cpu"))
    finally:
        dist.destroy_process_group()


def test_slowest_rank_time_is_reported_on_every_rank():
    port = _free_port()
    with mp.Manager() as m:
        results = m.dict()
        mp.spawn(_rank_main, args=(2, port, results), nprocs=2, join=True)
        assert dict(results) == {0: 7.25, 1: 7.25}


def test_single_rank_needs_no_process_group():
    import bench
    assert bench._max_over_ranks(1.25, False, torch.device("cpu")) == 1.25


@pytest.mark.slow
def test_reference_arm_under_torchrun_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py",
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3",
           "--cpu-seconds", "0.2", "--reference-budget", "1"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["unit"] == "tokens/s"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["value"] > 0
    assert d["e2e"]["h2d_bytes_per_step"] == 0

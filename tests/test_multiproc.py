"""Multi-rank host logic of the bench on CPU (gloo, world size 2).

The attention path shards by independent batches (no data-path collective); what crosses
ranks is the timing: every rank measures its own step time, the job time is the slowest
rank's, and the whole-job rate counts every rank's work.  The reference arm runs on
rank 0 only.
"""
import os
import socket
import sys

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
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        local_ms = [12.5, 14.0][rank]
        job_ms = bench.max_over_ranks(local_ms, "cpu")
        rate = bench.job_rate_tflops(12.8737e12, world, job_ms)

        class Args:
            steps, warmup, gpus = 1, 3, world
        ref = bench.run_reference(Args, rank) if rank != 0 else "skipped"
        out[rank] = (job_ms, rate, ref)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_rate_gloo():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
    for rank in range(world):
        job_ms, rate, ref = out[rank]
        assert job_ms == 14.0                                  # slowest rank sets the time
        assert rate == pytest.approx(2 * 12.8737e12 / 14.0e-3 / 1e12)
    assert out[1][2] is None                                   # reference arm: rank 0 only


def test_single_process_helpers():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, "cpu") == 3.5
    assert bench.job_rate_tflops(1e12, 1, 1.0) == pytest.approx(1000.0)
    assert bench.NCU_TRAFFIC_BYTES is None or bench.NCU_TRAFFIC_BYTES > 0

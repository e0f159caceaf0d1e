"""Host-side logic of the multi-rank benchmark, on CPU with the gloo backend:
the job's time is the slowest rank's, its throughput sums the ranks' batches,
and the reference arm runs on rank 0 only."""
import os
import socket
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


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import datetime

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        per_rank_ms = [3.0, 7.5, 5.0, 1.0][rank]
        ms = bench.reduce_max(per_rank_ms, torch.device("cpu"))
        value = bench.job_tflops(world, 2.0e12, ms)

        class A:
            warmup, steps = 0, 1
        ref = bench.run_reference(A, rank, world) if rank != 0 else "skipped"
        out[rank] = (ms, value, ref)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_max_over_ranks_and_job_value(world):
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
        res = dict(out)
    slowest = max([3.0, 7.5, 5.0, 1.0][:world])
    for r in range(world):
        ms, value, ref = res[r]
        assert ms == slowest
        assert value == pytest.approx(world * 2.0e12 / (slowest * 1e-3) / 1e12)
        if r != 0:
            assert ref is None  # only rank 0 runs and prints the reference arm


def test_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert not dist.is_initialized()
    assert bench.reduce_max(4.25, torch.device("cpu")) == 4.25
    assert bench.job_tflops(1, 1e12, 1000.0) == pytest.approx(1.0)

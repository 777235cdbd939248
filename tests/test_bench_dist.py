"""bench.py's multi-rank host logic on CPU: two gloo ranks, the job time is the max over
ranks and the value counts every rank's tokens (weak scaling)."""
import os
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    local = [12.5, 30.0][rank]
    t = bench.job_time_ms(local, "cpu")
    dist.barrier()
    out[rank] = (t, bench.job_value(16, 10, world, t))
    dist.destroy_process_group()


def test_job_time_is_max_over_ranks_and_value_counts_all_ranks():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    mp.start_processes(_rank, args=(2, port, out), nprocs=2, join=True, start_method="spawn")
    assert out[0][0] == out[1][0] == 30.0
    assert out[0][1] == pytest.approx(2 * 16 * 10 / 0.030)

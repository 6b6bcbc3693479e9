"""bench.py's multi-rank logic on CPU: two gloo ranks (world size 2).

Every rank times its own replica; the job time is the max over ranks and the
job throughput counts every rank's bytes against that time."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 2.0 + rank          # rank 1 is the slow one
        ms = bench.max_over_ranks(local_ms, world, device="cpu")
        out[rank] = (ms, bench.job_throughput(1_000_000_000, world, ms))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True,
                       start_method="spawn")
    assert out[0] == out[1]
    ms, gbs = out[0]
    assert ms == 3.0
    assert gbs == pytest.approx(2 * 1.0 / 3.0e-3)


def test_single_rank_is_identity():
    assert bench.max_over_ranks(1.25, 1) == 1.25
    assert bench.job_throughput(537_000_000, 1, 1.0) == pytest.approx(537.0)

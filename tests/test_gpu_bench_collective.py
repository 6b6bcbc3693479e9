"""bench.py's --collective environment on the GPU: `CudaCollectiveEnv` (inputs
drawn on the device, the expected output from the one-GPU fused kernel, the
real `QuantizedAllReduce` with IPC-mapped arenas, CUDA-event timing) driven by
`collective_sweep` with two gloo ranks sharing cuda:0.  Only what needs one GPU
per rank is replaced: NCCL's fp16 all-reduce (here a gloo all-reduce of a host
copy, a stand-in whose time means nothing).  The environment's own barriers,
flags and max-over-ranks already run on its gloo group.  The one-kernel form is
left out by the environment itself, since the ranks share a GPU; the
host-barrier form may."""
import datetime
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench

pytestmark = pytest.mark.gpu


class SharedGpuEnv(bench.CudaCollectiveEnv):
    def baseline_buffer(self, x):
        return x.float().cpu()

    def baseline(self, buf):
        dist.all_reduce(buf)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, points, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        env = SharedGpuEnv(rank, world, 0)
        rows = []
        bench.collective_sweep(env, points, steps=3, warmup=1, emit=rows.append)
        out[rank] = (sorted(env.forms), rows)
    finally:
        dist.destroy_process_group()


def test_sweep_on_two_ranks_sharing_one_gpu():
    world = 2
    points = [(8, 2 * 8192), (4, 2 * 8192 * 8), (8, 2 * 8192 * 64)]
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), points, out), nprocs=world, start_method="spawn")
    forms0, rows = out[0]
    assert forms0 == ["host_barrier"] and out[1][0] == forms0   # ranks share cuda:0: no one-kernel form
    assert out[1][1] == []
    assert len(rows) == len(points)
    for (bits, n), row in zip(points, rows):
        assert row["P"] == world and row["bits"] == bits and row["elements_per_rank"] == n
        assert row["bit_exact_vs_fused"] == {"host_barrier": True}, row
        assert row["wait_status"] == {"host_barrier": 0}
        assert row["us"]["host_barrier"] > 0
        assert row["wire_bytes_per_rank"] == bench.wire_bytes_per_rank(world, n, bits, 128)


def _rank_in_line(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        bench.CudaCollectiveEnv = SharedGpuEnv

        class Args:
            steps, warmup = 2, 1

        out[rank] = bench.collective_in_line(Args, world, rank, 0)
    finally:
        dist.destroy_process_group()


def test_collective_object_of_the_multi_gpu_line_at_its_message_sizes():
    """The N > 1 line's collective object at its own points (the decode-shaped and the
    prefill-shaped message), both ranks on cuda:0: every point bit-exact."""
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_in_line, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
    assert out[1] is None
    obj = out[0]
    assert obj["error"] is None, obj["error"]
    assert [(p["bits"], p["elements_per_rank"]) for p in obj["points"]] == bench.LINE_COLLECTIVE_POINTS
    for p in obj["points"]:
        assert p["bit_exact_vs_fused"] == {"host_barrier": True} and p["wait_status"] == {"host_barrier": 0}

"""bench.py's --collective sweep on CPU: its point list, its wire-byte
accounting and its JSON contract, driven by two gloo ranks whose quantized
all-reduce runs the real host schedule (`collective.QuantizedAllReduce`) on
shared-memory arenas with the oracle's steps, and whose baseline is gloo's
all-reduce of the fp16 message.  The GPU form (NCCL, CUDA events, one GPU
per rank) runs the same `collective_sweep` function."""
import os
import socket
import time

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import oracle
from bit_quantized_all_block_b200 import synth
from bit_quantized_all_block_b200.collective import QuantizedAllReduce


def test_points_cover_16kb_to_1gb_per_rank_in_whole_chunks():
    pts = bench.collective_points(8)
    assert [b for b, _ in pts] == [8] * 17 + [4] * 17
    ns = [n for _, n in pts[:17]]
    assert ns[0] * 2 == 16 << 10 and ns[-1] * 2 == 1 << 30
    assert all(b == 2 * a for a, b in zip(ns, ns[1:]))
    for P in (2, 3, 4, 5, 8):
        for bits, n in bench.collective_points(P):
            assert n % (P * 128) == 0 and n > 0
            assert (16 << 10) // 2 - P * 128 < n <= (1 << 30) // 2


def test_wire_bytes_by_hand():
    # P=2, 2048 elements per rank, INT8, blocks of 128: a payload is 2048 code
    # bytes + 16 blocks * 5 bytes = 2128; each rank pulls half of one in the
    # reduce-scatter and half in the all-gather
    assert bench.wire_bytes_per_rank(2, 2048, 8, 128) == {"quantized": 2128, "nccl_fp16_ring": 4096}
    # P=4, INT4: 65536/2 + 512*5 = 35328 per payload, 2 * 3/4 of it
    assert bench.wire_bytes_per_rank(4, 65536, 4, 128) == {"quantized": 52992, "nccl_fp16_ring": 196608}


class CpuEnv:
    """The sweep's environment on CPU (see bench.collective_sweep)."""

    timing_note = "host wall clock (CPU stand-in for the device timing)"

    def __init__(self, rank, world, dtype):
        from tests.collective_cpu_ops import OracleOps
        self.OracleOps = OracleOps
        self.rank, self.world, self.dtype = rank, world, dtype
        self.forms = {"host_barrier": False}
        self.calls = []

    def _all(self, n):
        H = 128
        return synth.partials(self.world, n // H, H, self.dtype, 0.05, 20.0, seed=n)

    def partial(self, n):
        return self._all(n)[self.rank]

    def expected(self, n, bits, block):
        return oracle.allreduce(list(self._all(n)), self.dtype, bits, block)[0]

    def allreduce(self, n, bits, block, one_kernel):
        assert not one_kernel
        self.calls.append((n, bits, block))
        return QuantizedAllReduce(n, bits, block, ops=self.OracleOps(self.dtype), timeout=30.0)

    def new_output(self, x):
        return np.empty(x.shape[0], np.uint16)

    def equal(self, a, b):
        return bool(np.array_equal(a, b))

    def baseline_buffer(self, x):
        return torch.from_numpy(x.view(np.int16).copy()).view(torch.float16)

    def baseline(self, buf):
        dist.all_reduce(buf)

    def sync(self):
        pass

    def barrier(self):
        dist.barrier()

    def timed(self, fn):
        t0 = time.perf_counter()
        fn()
        return (time.perf_counter() - t0) * 1e3

    def all_true(self, flag):
        t = torch.tensor([1 if flag else 0], dtype=torch.int32)
        dist.all_reduce(t, op=dist.ReduceOp.MIN)
        return bool(t.item())

    def max_over_ranks(self, v):
        t = torch.tensor([v], dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, points, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        env = CpuEnv(rank, world, oracle.FP16)
        rows = []
        bench.collective_sweep(env, points, steps=2, warmup=1, emit=rows.append)
        out[rank] = (rows, env.calls)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_sweep_lines_on_gloo_ranks(world):
    # the oracle's RS step (the CPU stand-in) wants whole P-block groups per chunk
    points = [(8, world * world * 128 * 2), (4, world * world * 128 * 3)]
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), points, out), nprocs=world, start_method="spawn")
    rows0, calls0 = out[0]
    assert len(rows0) == len(points)
    for r in range(1, world):
        rows, calls = out[r]
        assert rows == []                        # rank 0 alone emits
        assert calls == calls0                   # every rank made the same collective calls in the same order
    assert calls0 == [(n, bits, 128) for bits, n in points]
    for (bits, n), row in zip(points, rows0):
        assert row["mode"] == "collective" and row["P"] == world
        assert row["bits"] == bits and row["elements_per_rank"] == n and row["bytes_per_rank"] == 2 * n
        assert set(row["us"]) == {"host_barrier", "nccl_fp16"} and all(v > 0 for v in row["us"].values())
        assert row["speedup_vs_nccl_fp16"]["host_barrier"] == pytest.approx(
            row["us"]["nccl_fp16"] / row["us"]["host_barrier"], rel=0.02)
        assert row["wire_bytes_per_rank"] == bench.wire_bytes_per_rank(world, n, bits, 128)
        assert row["bit_exact_vs_fused"] == {"host_barrier": True}
        assert row["wait_status"] == {"host_barrier": 0}
        assert row["steps"] == 2 and row["warmup"] == 1 and row["timing"]


def test_one_rank_prints_the_unavailable_line():
    """Without torchrun (one rank) the mode says it needs two or more GPUs and exits 0,
    before any CUDA call."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--collective"], capture_output=True,
                       text=True, cwd=root, env=env, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    (line,) = [l for l in r.stdout.splitlines() if l.startswith("{")]
    d = json.loads(line)
    assert d["mode"] == "collective" and "2 or more GPUs" in d["unavailable"]


class _GivesUpOnRank1:
    """A one-kernel form whose first call reports a bounded wait that gave up, on rank 1 only."""

    def __init__(self, inner, rank, calls):
        self.inner, self.rank, self.calls = inner, rank, calls

    def __call__(self, x, y):
        self.calls.append("one_kernel call")
        return self.inner(x, y)

    def last_status(self):
        return 1 if self.rank == 1 else 0

    def close(self):
        self.inner.close()


class _EnvWithFailingForm(CpuEnv):
    def __init__(self, rank, world, dtype):
        super().__init__(rank, world, dtype)
        self.forms = {"host_barrier": False, "one_kernel": True}

    def allreduce(self, n, bits, block, one_kernel):
        inner = super().allreduce(n, bits, block, False)
        return _GivesUpOnRank1(inner, self.rank, self.calls) if one_kernel else inner


def _rank_failing(rank, world, port, points, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        env = _EnvWithFailingForm(rank, world, oracle.FP16)
        rows = []
        bench.collective_sweep(env, points, steps=3, warmup=2, emit=rows.append)
        out[rank] = (rows, env.calls)
    finally:
        dist.destroy_process_group()


def test_a_form_whose_first_call_gave_up_is_not_timed():
    """A give-up on any rank is seen by every rank (max over ranks), so no rank times
    that form: its later calls would give up too, each after the wait limit."""
    world, n = 2, 2 * 2 * 128 * 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_failing, args=(world, _free_port(), [(8, n)], out), nprocs=world,
                       start_method="spawn")
    (row,), calls0 = out[0]
    assert out[1][0] == []
    for r in range(world):
        assert out[r][1].count("one_kernel call") == 1      # the checked call only: no warm-up, no timing
    assert row["wait_status"] == {"host_barrier": 0, "one_kernel": 1}
    assert row["us"]["one_kernel"] is None and row["us"]["host_barrier"] > 0
    assert set(row["speedup_vs_nccl_fp16"]) == {"host_barrier"}


def _rank_in_line(rank, world, port, fail, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        def make_env(rank_, world_, local):
            if fail:
                raise RuntimeError("no peer access")
            return CpuEnv(rank_, world_, oracle.FP16)

        bench.CudaCollectiveEnv = make_env
        bench.LINE_COLLECTIVE_POINTS = [(8, world * world * 128), (4, world * world * 128 * 2)]

        class Args:
            steps, warmup = 2, 1

        out[rank] = bench.collective_in_line(Args, world, rank, 0)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("fail", [False, True], ids=["runs", "env_fails"])
def test_collective_object_of_the_multi_gpu_line(fail):
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_in_line, args=(world, _free_port(), fail, out), nprocs=world, start_method="spawn")
    assert out[1] is None                                   # rank 0 alone carries it
    obj = out[0]
    assert "P = 2" in obj["what"]
    if fail:
        assert obj["points"] == [] and "no peer access" in obj["error"]
    else:
        assert obj["error"] is None and len(obj["points"]) == 2
        assert [(p["bits"], p["elements_per_rank"]) for p in obj["points"]] == [(8, 512), (4, 1024)]
        assert all(p["bit_exact_vs_fused"] == {"host_barrier": True} for p in obj["points"])


class _FailsOnRank1AtSecondPoint(CpuEnv):
    def allreduce(self, n, bits, block, one_kernel):
        if self.rank == 1 and len(self.calls) == 1:
            raise RuntimeError("peer mapping lost")
        return super().allreduce(n, bits, block, one_kernel)


def _rank_asymmetric(rank, world, port, out):
    import datetime
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=30))
    t0 = time.monotonic()
    try:
        bench.CudaCollectiveEnv = lambda r, w, local: _FailsOnRank1AtSecondPoint(r, w, oracle.FP16)
        bench.LINE_COLLECTIVE_POINTS = [(8, world * world * 128), (4, world * world * 128 * 2)]

        class Args:
            steps, warmup = 2, 1

        obj = bench.collective_in_line(Args, world, rank, 0)
        out[rank] = (obj, time.monotonic() - t0)
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(240)
def test_a_failure_on_one_rank_ends_every_rank_with_an_error_report():
    """Rank 1 raises inside the sweep, rank 0 does not: rank 1 leaves, rank 0's next
    step on the gloo group fails instead of waiting for good, and rank 0 still gets
    its object, with the first point and the error."""
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_asymmetric, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
    obj, seconds = out[0]
    assert out[1][0] is None
    assert obj["error"] and len(obj["points"]) == 1
    assert seconds < 120


def test_line_points_fit_every_rank_count():
    """The multi-GPU line's fixed message sizes divide into whole chunks of blocks at
    every world size of a scaling run (2, 4 and 8 processes).  (Other world sizes get
    an error in the object: the collective's layout refuses such a message.)"""
    for P in (2, 4, 8):
        for bits, n in bench.LINE_COLLECTIVE_POINTS:
            assert bits in (4, 8)
            assert n % (P * bench.COLLECTIVE_BLOCK) == 0, (P, n)

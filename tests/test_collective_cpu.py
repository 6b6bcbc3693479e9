"""The P-rank quantized all-reduce's host logic on CPU (no GPU): arena layout,
the per-rank schedule, and the whole three-step exchange run by 2 and 4 gloo
ranks (one process each) whose arenas are shared memory and whose steps are
the oracle's -- the result must be the oracle's one-process all-reduce, bit
for bit, on every rank, over two consecutive calls on the same arenas."""
import os
import socket

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from bit_quantized_all_block_b200 import synth
from bit_quantized_all_block_b200.collective import ALIGN, Layout, QuantizedAllReduce, schedule


@pytest.mark.parametrize("n,P,bits,block", [(4096, 2, 8, 128), (4096, 4, 4, 32), (65536, 8, 4, 4096),
                                            (3 * 8 * 512, 8, 8, 512)])
def test_layout_parts_are_aligned_sized_and_disjoint(n, P, bits, block):
    L = Layout(n, P, bits, block)
    m = n // P
    parts = []
    for ref in [L.step1(0, c) for c in range(P)] + [L.step2(0)]:
        assert ref.n == m
        parts += [(ref.codes, m * bits // 8), (ref.scales, 4 * (m // block)), (ref.zps, m // block)]
    for off, size in parts:
        assert off % ALIGN == 0 and off + size <= L.nbytes
    parts.sort()
    for (o1, s1), (o2, _) in zip(parts, parts[1:]):
        assert o1 + s1 <= o2


def test_layout_rejects_chunks_that_are_not_whole_blocks():
    with pytest.raises(ValueError):
        Layout(4096 + 128, 2, 8, 128)


def test_schedule_reads_the_owned_chunk_from_every_rank():
    L = Layout(8192, 4, 8, 128)
    for rank in range(4):
        quantize, (ins, out), ag = schedule(rank, L)
        assert [q.holder for q in quantize] == [rank] * 4
        assert quantize == [L.step1(rank, c) for c in range(4)]
        assert ins == [L.step1(r, rank) for r in range(4)]       # chunk `rank` of every holder
        assert out == L.step2(rank)
        assert [a.holder for a in ag] == [0, 1, 2, 3]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, case, out):
    from tests.collective_cpu_ops import OracleOps
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        n, dtype, bits, block, seeds = case
        ar = QuantizedAllReduce(n, bits, block, ops=OracleOps(dtype))
        ys = []
        for seed in seeds:
            xs = synth.partials(world, n // block, block, dtype, 0.05, 20.0, seed=seed)
            ys.append(ar(xs[rank]).copy())
        ar.close()
        out[rank] = ys
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,bits,block,dtype", [(2, 8, 128, oracle.FP16), (4, 4, 64, oracle.BF16)])
def test_ranks_reproduce_the_one_process_allreduce(world, bits, block, dtype):
    n = world * world * block * 3     # the oracle's RS step wants whole P-block groups per chunk
    seeds = (11, 12)
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), (n, dtype, bits, block, seeds), out),
                       nprocs=world, join=True, start_method="spawn")
    for k, seed in enumerate(seeds):
        xs = synth.partials(world, n // block, block, dtype, 0.05, 20.0, seed=seed)
        y_ref, _, _ = oracle.allreduce(list(xs), dtype, bits, block)
        for r in range(world):
            assert np.array_equal(out[r][k], y_ref), f"rank {r}, call {k}"


def test_one_kernel_mode_refuses_ranks_on_one_device():
    from bit_quantized_all_block_b200.collective import ranks_share_a_device
    assert ranks_share_a_device(["GPU-a", "GPU-a"])
    assert ranks_share_a_device(["GPU-a", "GPU-b", "GPU-a", "GPU-c"])
    assert not ranks_share_a_device(["GPU-a", "GPU-b", "GPU-c", "GPU-d"])


def test_layout_reserves_aligned_counters():
    L = Layout(8192, 4, 8, 128)
    assert L.counters % ALIGN == 0 and L.counters + 8 <= L.nbytes
    last = L.step2(0)
    assert L.counters >= last.zps + 2048 // 128


def _leaving_rank_main(rank, world, port, out, stall=0.0):
    """Every rank makes one call; the last rank then leaves (after `stall`
    seconds alive without taking part), the others call again."""
    import time
    from tests.collective_cpu_ops import OracleOps
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    n, dtype, bits, block = world * world * 128 * 2, oracle.FP16, 8, 128
    ops = OracleOps(dtype)
    try:
        ar = QuantizedAllReduce(n, bits, block, ops=ops, timeout=3.0)
        xs = synth.partials(world, n // block, block, dtype, 0.0, 1.0, seed=5)
        ar(xs[rank])
        if rank == world - 1:
            time.sleep(stall)
            out[rank] = "left"
            return
        t0 = time.time()
        try:
            ar(xs[rank])
            out[rank] = "no error"
        except RuntimeError as e:
            out[rank] = ("error", time.time() - t0, str(e)[:200])
    finally:
        ops.close()          # this rank's arena and its views of the others' (no collective step)
        dist.destroy_process_group()


@pytest.mark.parametrize("stall", [0.0, 8.0], ids=["exits", "stalls"])
def test_a_rank_that_leaves_ends_the_others_call_with_an_error(stall):
    """Failure detection on the host: after one call the last rank leaves --
    at once (its connections close) or after staying alive 8 s without taking
    part; the others' next call must end with an error, at the latest after
    the collective's 3 s timeout, never waiting for the missing rank."""
    world = 3
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_leaving_rank_main, args=(world, _free_port(), out, stall), nprocs=world, join=True,
                       start_method="spawn")
    assert out[world - 1] == "left"
    for r in range(world - 1):
        res = out[r]
        assert res[0] == "error", f"rank {r}: {res}"
        assert res[1] < (6.0 if stall else 30.0), f"rank {r} waited {res[1]:.1f} s"
    if stall:
        assert any(2.5 < out[r][1] for r in range(world - 1)), "the timeout path was not taken"


class _AddressOps:
    """The one-kernel mode's device side reduced to addresses: each rank's arena
    sits at a made-up base address (never dereferenced: the kernel call is
    replaced by a recorder), one made-up device per rank."""

    def __init__(self, rank):
        import torch
        self.torch, self.device, self.rank, self.base = torch, torch.device("cpu"), rank, {}

    def alloc(self, nbytes):
        pass

    def export(self):
        return 0x10000000 * (self.rank + 1)

    def device_id(self):
        return f"fake-gpu-{self.rank}"

    def attach(self, rank, exported):
        self.base = dict(enumerate(exported))

    def qbuf(self, ref, bits, block):
        from bit_quantized_all_block_b200 import PeerQBuf
        b = self.base[ref.holder]
        return PeerQBuf(b + ref.codes, b + ref.scales, b + ref.zps, ref.n, bits, block)

    def new_output(self, x):
        return x.new_empty(x.shape[0])

    def sync(self):
        pass

    def close(self):
        pass


def _one_kernel_rank(rank, world, port, n, out):
    import torch

    from bit_quantized_all_block_b200 import collective
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        calls = []

        def record(rank_, x, y, bits, block, s1, s2, ctr1, ctr2, epoch, status, tables=None):
            a1, a2, c1, c2 = tables.args
            calls.append((rank_, epoch, id(tables), [(q.codes, q.scales, q.zps) for q in a1],
                          [(q.codes, q.scales, q.zps) for q in a2], [c or 0 for c in c1], [c or 0 for c in c2]))

        collective.fc_p2p_allreduce = record
        ar = collective.QuantizedAllReduce(n, 8, 128, ops=_AddressOps(rank), one_kernel=True, timeout=30.0)
        x = torch.zeros(n, dtype=torch.float16)
        for _ in range(3):
            ar(x)
        out[rank] = calls
    finally:
        dist.destroy_process_group()


def test_one_kernel_calls_pass_the_arena_tables_built_once():
    """Every call hands the kernel the same tables, built at construction: rank p's
    step-1 payload of chunk c and owner c's step-2 payload at their layout offsets
    in the holder's arena, the counters at the arena's counter words; the epoch
    is 0 on every call (the kernel derives it from the counters, so a captured
    call can be replayed)."""
    world, n = 2, 2 * 128 * 16
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_one_kernel_rank, args=(world, _free_port(), n, out), nprocs=world, start_method="spawn")
    L = Layout(n, world, 8, 128)
    base = [0x10000000 * (r + 1) for r in range(world)]
    want_s1 = [(base[p] + L.step1(p, c).codes, base[p] + L.step1(p, c).scales, base[p] + L.step1(p, c).zps)
               for p in range(world) for c in range(world)]
    want_s2 = [(base[c] + L.step2(c).codes, base[c] + L.step2(c).scales, base[c] + L.step2(c).zps)
               for c in range(world)]
    for r in range(world):
        calls = out[r]
        assert [c[1] for c in calls] == [0, 0, 0] and all(c[0] == r for c in calls)   # epochs derived on the device
        assert len({c[2] for c in calls}) == 1                   # one tables object for every call
        for _, _, _, s1, s2, c1, c2 in calls:
            assert s1 == want_s1 and s2 == want_s2
            assert c1 == [b + L.counters for b in base] and c2 == [b + L.counters + 4 for b in base]

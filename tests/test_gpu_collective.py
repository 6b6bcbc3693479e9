"""The P-rank quantized all-reduce on the GPU: P processes (gloo group), each
with its own arena in device memory, the peers' arenas mapped through the
library's IPC calls, the three steps run by the library's kernels reading the
peers' payloads directly.  Here all ranks share cuda:0 (no kernel waits on
another rank, so that is valid); on a multi-GPU node the same loads cross
NVLink.  Every rank's output must equal the CPU oracle's one-process
all-reduce bit for bit, over two consecutive calls."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from bit_quantized_all_block_b200 import synth

pytestmark = pytest.mark.gpu


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, case, out):
    from bit_quantized_all_block_b200.collective import QuantizedAllReduce
    from tests.gpu_util import tdtype
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        n, dtype, bits, block, seeds = case
        ar = QuantizedAllReduce(n, bits, block)
        ys = []
        for seed in seeds:
            xs = synth.partials(world, n // block, block, dtype, 0.05, 20.0, seed=seed)
            x = torch.from_numpy(xs[rank].view(np.int16).copy()).view(tdtype(dtype)).cuda()
            y = ar(x)
            torch.cuda.synchronize()
            ys.append(y.view(torch.int16).cpu().numpy().view(np.uint16))
        ar.close()
        out[rank] = ys
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,bits,block,dtype,rows", [
    (2, 8, 128, oracle.FP16, 48),        # several tiles per chunk, ragged
    (4, 4, 128, oracle.BF16, 3),         # chunks of 3 blocks: not a multiple of P blocks
    (4, 8, 1024, oracle.FP16, 12),       # blocks that span warps
    (8, 4, 32, oracle.BF16, 8),
])
def test_ranks_match_the_oracle(world, bits, block, dtype, rows):
    n = rows * world * block
    seeds = (21, 22)
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), (n, dtype, bits, block, seeds), out),
                       nprocs=world, join=True, start_method="spawn")
    for k, seed in enumerate(seeds):
        xs = synth.partials(world, n // block, block, dtype, 0.05, 20.0, seed=seed)
        y_ref, _, _ = oracle.allreduce(list(xs), dtype, bits, block)
        for r in range(world):
            got = out[r][k]
            bad = np.nonzero(got != y_ref)[0]
            assert bad.size == 0, f"rank {r}, call {k}: {bad.size} outputs differ, first at {bad[:8]}"


def _rank_one_kernel(rank, world, port, out):
    from bit_quantized_all_block_b200.collective import QuantizedAllReduce
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        try:
            QuantizedAllReduce(2 * 128 * 4, 8, 128, one_kernel=True)
            out[rank] = "built"
        except ValueError:
            out[rank] = "refused"
    finally:
        dist.destroy_process_group()


def test_one_kernel_mode_refuses_ranks_that_share_a_gpu():
    """The one-kernel mode's kernels wait on each other; on a shared GPU that
    could never be guaranteed to progress, so construction is refused (before
    any launch)."""
    out = mp.get_context("spawn").Manager().dict()
    mp.start_processes(_rank_one_kernel, args=(2, _free_port(), out), nprocs=2, join=True, start_method="spawn")
    assert out[0] == "refused" and out[1] == "refused"

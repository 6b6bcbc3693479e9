"""The one-kernel P-GPU all-reduce, run in its emulated form: one cooperative
launch on one GPU whose CTAs play all P ranks, every rank's buffers in that
GPU's memory, the ranks synchronised only by the kernel's counters.  Every
rank's output, every step-1 chunk payload and every owner's step-2 payload
must equal the CPU oracle's, over consecutive calls on the same counters; a
wait that nothing satisfies must give up, report it, and leave the context
usable."""
import numpy as np
import pytest
import torch

import bit_quantized_all_block_b200 as fc
import oracle
from bit_quantized_all_block_b200 import synth
from tests.gpu_util import tdtype, to_dev

pytestmark = pytest.mark.gpu


class Ranks:
    """Buffers of P emulated ranks for n elements."""

    def __init__(self, P, n, dtype, bits, block):
        self.P, self.n, self.bits, self.block = P, n, bits, block
        self.m = n // P
        self.s1 = [fc.QBuf.empty(self.m, bits, block) for _ in range(P * P)]      # s1[p*P + c]
        self.s2 = [fc.QBuf.empty(self.m, bits, block) for _ in range(P)]
        self.ctr = torch.zeros(2 * P, dtype=torch.int32, device="cuda")
        base = self.ctr.data_ptr()
        self.ctr1 = [base + 4 * p for p in range(P)]
        self.ctr2 = [base + 4 * (P + p) for p in range(P)]
        self.status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        self.ys = [torch.empty(n, dtype=tdtype(dtype), device="cuda") for _ in range(P)]

    def run(self, xs_dev, epoch, ctas_per_rank=0):
        fc.fc_p2p_allreduce_emulated(xs_dev, self.ys, self.bits, self.block, self.s1, self.s2, self.ctr1,
                                     self.ctr2, epoch, self.status, ctas_per_rank)
        torch.cuda.synchronize()
        return int(self.status.item())


def _check(R, xs, dtype):
    P, m, bits, block = R.P, R.m, R.bits, R.block
    y_ref, p1_ref, p2_ref = oracle.allreduce(list(xs), dtype, bits, block)
    for p in range(P):
        got = R.ys[p].view(torch.int16).cpu().numpy().view(np.uint16)
        assert np.array_equal(got, y_ref), f"rank {p}: output differs"
    cb, nb = m * bits // 8, m // block
    for p in range(P):
        for c in range(P):
            q = R.s1[p * P + c]
            assert np.array_equal(q.codes.cpu().numpy(), p1_ref[p].codes[c * cb:(c + 1) * cb])
            assert np.array_equal(q.scales.cpu().numpy().view(np.uint32),
                                  p1_ref[p].scales[c * nb:(c + 1) * nb].view(np.uint32))
            assert np.array_equal(q.zps.cpu().numpy(), p1_ref[p].zps[c * nb:(c + 1) * nb])
    for c in range(P):
        q = R.s2[c]
        assert np.array_equal(q.codes.cpu().numpy(), p2_ref.codes[c * cb:(c + 1) * cb])
        assert np.array_equal(q.scales.cpu().numpy().view(np.uint32), p2_ref.scales[c * nb:(c + 1) * nb].view(np.uint32))
        assert np.array_equal(q.zps.cpu().numpy(), p2_ref.zps[c * nb:(c + 1) * nb])


@pytest.mark.parametrize("P,bits,block,dtype,blocks_per_chunk", [
    (2, 8, 128, oracle.FP16, 75),        # several tiles per rank, ragged
    (4, 4, 128, oracle.BF16, 3),         # chunks of 3 blocks
    (4, 8, 32, oracle.FP16, 129),
    (8, 4, 64, oracle.BF16, 17),
    (8, 8, 1024, oracle.FP16, 2),        # blocks that span warps
    (2, 4, 4096, oracle.BF16, 3),
])
def test_emulated_ranks_match_the_oracle(P, bits, block, dtype, blocks_per_chunk):
    n = P * block * blocks_per_chunk
    R = Ranks(P, n, dtype, bits, block)
    for epoch, seed in ((1, 50), (2, 51), (3, 52)):      # the same counters, call after call
        xs = synth.partials(P, n // block, block, dtype, 0.05, 20.0, seed=seed + P + bits)
        assert R.run(to_dev(xs, dtype), epoch) == 0
        _check(R, xs, dtype)


@pytest.mark.parametrize("P,bits,block,dtype", [(2, 8, 128, oracle.FP16), (8, 4, 128, oracle.BF16)])
def test_tables_marshalled_once_serve_every_call(P, bits, block, dtype):
    """fc.P2PTables built once and passed to every call (the collective object's path):
    consecutive epochs on new inputs, every output and payload equal to the oracle's."""
    n = P * block * 9
    R = Ranks(P, n, dtype, bits, block)
    tables = fc.P2PTables(R.s1, R.s2, R.ctr1, R.ctr2)
    for epoch in (1, 2, 3):
        xs = synth.partials(P, n // block, block, dtype, 0.05, 20.0, seed=90 + epoch + P)
        fc.fc_p2p_allreduce_emulated(to_dev(xs, dtype), R.ys, bits, block, None, None, None, None, epoch,
                                     R.status, tables=tables)
        torch.cuda.synchronize()
        assert int(R.status.item()) == 0
        _check(R, xs, dtype)


@pytest.mark.parametrize("P,bits,block,dtype", [(2, 8, 128, oracle.FP16), (8, 4, 256, oracle.BF16)])
def test_epoch_derived_from_the_counters(P, bits, block, dtype):
    """epoch 0: the kernel derives each call's epoch from its rank's phase-1 counter,
    also after calls that passed explicit epochs; every call bit-exact with the oracle."""
    n = P * block * 11
    R = Ranks(P, n, dtype, bits, block)
    for epoch, seed in ((1, 60), (0, 61), (0, 62), (4, 63), (0, 64)):
        xs = synth.partials(P, n // block, block, dtype, 0.05, 20.0, seed=seed + P)
        assert R.run(to_dev(xs, dtype), epoch) == 0
        _check(R, xs, dtype)


@pytest.mark.parametrize("P,bits,block,dtype", [(4, 8, 128, oracle.FP16), (8, 4, 128, oracle.BF16)])
def test_call_captured_in_a_cuda_graph_and_replayed(P, bits, block, dtype):
    """A call with epoch 0 captured once and replayed (the decode-loop pattern): every
    replay runs the next epoch on the same counters, with the inputs rewritten in
    place between replays, and gives the oracle's result."""
    n = P * block * 13
    R = Ranks(P, n, dtype, bits, block)
    tables = fc.P2PTables(R.s1, R.s2, R.ctr1, R.ctr2)
    xs = synth.partials(P, n // block, block, dtype, 0.05, 20.0, seed=70 + P)
    xd = to_dev(xs, dtype)

    def call():
        fc.fc_p2p_allreduce_emulated(xd, R.ys, bits, block, None, None, None, None, 0, R.status, tables=tables)

    call()                                   # outside the capture: loads the module, epoch 1
    torch.cuda.synchronize()
    assert int(R.status.item()) == 0
    _check(R, xs, dtype)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        call()
    for rep in range(3):
        xs = synth.partials(P, n // block, block, dtype, 0.05, 20.0, seed=80 + rep + P)
        for d, h in zip(xd, to_dev(xs, dtype)):
            d.copy_(h)
        g.replay()
        torch.cuda.synchronize()
        assert int(R.status.item()) == 0, f"replay {rep}: a wait gave up"
        _check(R, xs, dtype)
    counts = R.ctr.cpu().tolist()        # four complete calls: every counter at 4 x CTAs per rank
    assert len(set(counts)) == 1 and counts[0] > 0 and counts[0] % 4 == 0, counts
    del g


def test_few_ctas_per_rank_loop_over_tiles():
    P, bits, block, dtype = 4, 8, 128, oracle.FP16
    n = P * 128 * 80
    R = Ranks(P, n, dtype, bits, block)
    xs = synth.partials(P, n // block, block, dtype, 0.05, 20.0, seed=60)
    assert R.run(to_dev(xs, dtype), 1, ctas_per_rank=2) == 0
    _check(R, xs, dtype)


def test_a_wait_nothing_satisfies_gives_up():
    P, bits, block, dtype = 2, 8, 128, oracle.FP16
    n = P * 128 * 8
    R = Ranks(P, n, dtype, bits, block)
    xs = to_dev(synth.partials(P, n // block, block, dtype, 0.0, 1.0, seed=61), dtype)
    # fresh counters but the third call's epoch: phase 1 counts to 1 x CTAs,
    # the wait wants 3 x CTAs -- nothing will satisfy it
    assert R.run(xs, 3) == 1
    y = fc.fc_quantized_allreduce(xs, bits, block)          # the context is still usable
    torch.cuda.synchronize()
    assert y.shape[0] == n

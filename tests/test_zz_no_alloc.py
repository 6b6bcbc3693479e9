"""The all-reduce entry point that allocates nothing.

Some callers cannot allocate device memory where they run the all-reduce: a
plugin inside a framework that owns all device memory and forbids allocation
in its execute callback, a serving loop that cannot pay for the device-wide
synchronisation of cudaFree, a process whose memory is already reserved by a
caching allocator.  fc_p2p_allreduce_emulated_noalloc serves them: it keeps the
wire payloads, the phase counters and the status word in the library's own
static device array, and the caller passes only inputs and outputs.

Checked here through the C ABI (ctypes on libfc.so): on two calls in a row on
the same scratch every rank's output equals the CPU oracle's all-reduce of the
same inputs, bit for bit, and the bits of fc_p2p_allreduce_emulated with
caller-owned scratch (stale payloads or counters from the first call would
show in the second); the largest problem that fits the array runs and one more
chunk of blocks is refused before any launch.  This file is collected last so that a run
stopping at its first failure has run every other test before it."""
import ctypes

import numpy as np
import pytest
import torch

import bit_quantized_all_block_b200 as fc
import oracle
from bit_quantized_all_block_b200 import synth
from tests.gpu_util import host_u16, tdtype, to_dev

pytestmark = pytest.mark.gpu


def _noalloc(xs, ys, bits, block, status=None):
    """One call of the new entry point through the C ABI; returns its fc_status."""
    P = len(xs)
    xp = (ctypes.c_void_p * P)(*[x.data_ptr() for x in xs])
    yp = (ctypes.c_void_p * P)(*[y.data_ptr() for y in ys])
    st = ctypes.c_void_p(status.data_ptr()) if status is not None else None
    dt = fc.FC_FP16 if xs[0].dtype == torch.float16 else fc.FC_BF16
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return fc.library().fc_p2p_allreduce_emulated_noalloc(P, dt, xs[0].numel(), bits, block, xp, yp, st, stream)


def _with_caller_scratch(xs, bits, block):
    """The existing entry point, every buffer allocated by the caller (torch)."""
    P, n = len(xs), xs[0].numel()
    m = n // P
    s1 = [fc.QBuf.empty(m, bits, block) for _ in range(P * P)]
    s2 = [fc.QBuf.empty(m, bits, block) for _ in range(P)]
    ctr = torch.zeros(2 * P, dtype=torch.int32, device="cuda")
    c1 = [ctr.data_ptr() + 4 * p for p in range(P)]
    c2 = [ctr.data_ptr() + 4 * (P + p) for p in range(P)]
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    ys = [torch.empty_like(x) for x in xs]
    fc.fc_p2p_allreduce_emulated(xs, ys, bits, block, s1, s2, c1, c2, 1, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return [host_u16(y) for y in ys]


def _check_against_oracle(xs_host, ys, dtype, bits, block, what):
    """Every rank's output equals the oracle's all-reduce of the host inputs."""
    y_ref = oracle.allreduce(list(xs_host), dtype, bits, block)[0]
    for p, y in enumerate(ys):
        got = host_u16(y)
        bad = np.nonzero(got != y_ref)[0]
        assert bad.size == 0, f"{what}, rank {p}: {bad.size} outputs differ from the oracle, first at {bad[:8]}"


def _scratch_bytes(P, n, bits, block):
    r = lambda v: (v + 255) // 256 * 256
    m = n // P
    return 256 + P * (P + 1) * (r(m * bits // 8) + r(4 * (m // block)) + r(m // block))


@pytest.mark.parametrize("P,bits,block,dtype,n", [
    (4, 8, 128, oracle.FP16, 8 * 8192),         # the decode-shaped message: 8 tokens x 8192 hidden
    (8, 4, 64, oracle.BF16, 8 * 64 * 37),       # chunks of 37 blocks, a ragged last tile
    (2, 8, 1024, oracle.FP16, 2 * 1024 * 5),    # blocks that span warps
])
def test_two_calls_in_a_row_match_the_allocating_entry_point(P, bits, block, dtype, n):
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    for seed in (70, 71):                       # the second call reuses the first call's scratch
        xh = synth.partials(P, n // block, block, dtype, 0.05, 20.0, seed=seed + P)
        xs = to_dev(xh, dtype)
        ys = [torch.full_like(x, float("nan")) for x in xs]
        assert _noalloc(xs, ys, bits, block, status) == fc.FC_OK
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        _check_against_oracle(xh, ys, dtype, bits, block, f"call with seed {seed}")
        want = _with_caller_scratch(xs, bits, block)
        for p in range(P):
            assert np.array_equal(host_u16(ys[p]), want[p]), f"call with seed {seed}, rank {p}: output differs"


def test_without_a_status_word():
    P, bits, block, dtype, n = 4, 4, 128, oracle.FP16, 4 * 128 * 9
    for seed in (72, 73):
        xh = synth.partials(P, n // block, block, dtype, 0.0, 1.0, seed=seed)
        xs = to_dev(xh, dtype)
        ys = [torch.empty_like(x) for x in xs]
        assert _noalloc(xs, ys, bits, block, None) == fc.FC_OK
        torch.cuda.synchronize()
        _check_against_oracle(xh, ys, dtype, bits, block, f"seed {seed}")
        want = _with_caller_scratch(xs, bits, block)
        for p in range(P):
            assert np.array_equal(host_u16(ys[p]), want[p])


def test_the_largest_problem_that_fits_and_one_chunk_more():
    P, bits, block, dtype = 4, 8, 128, oracle.FP16
    step = P * block
    n = step
    while _scratch_bytes(P, n + step, bits, block) <= fc.FC_NOALLOC_SCRATCH_BYTES:
        n += step
    assert _scratch_bytes(P, n, bits, block) > fc.FC_NOALLOC_SCRATCH_BYTES - 32 * 1024   # the array's far end is used
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    for seed in (74, 75):
        xh = synth.partials(P, n // block, block, dtype, 0.001, 50.0, seed=seed)
        xs = to_dev(xh, dtype)
        ys = [torch.empty_like(x) for x in xs]
        assert _noalloc(xs, ys, bits, block, status) == fc.FC_OK
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        _check_against_oracle(xh, ys, dtype, bits, block, f"seed {seed}")
        want = _with_caller_scratch(xs, bits, block)
        for p in range(P):
            assert np.array_equal(host_u16(ys[p]), want[p]), f"seed {seed}, rank {p}: output differs"
    # one more chunk of blocks does not fit: refused on the host, nothing launched
    big = [torch.empty(n + step, dtype=tdtype(dtype), device="cuda") for _ in range(P)]
    out = [torch.empty_like(x) for x in big]
    assert _noalloc(big, out, bits, block, status) == fc.FC_ERR_TOO_LARGE

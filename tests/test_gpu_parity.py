"""GPU parity: the sm_100a kernels, called through the C ABI, are bit-exact
with the CPU oracle -- codes, scale bit patterns, zero-points and outputs --
for the fused kernel (with and without payload outputs) and for the staged
pipeline, over every block size, both bit widths, both dtypes, P = 1..8,
multi-tile sizes with ragged tails, and the edge cases of the method."""
import numpy as np
import pytest
import torch

import bit_quantized_all_block_b200 as fc
import oracle
from bit_quantized_all_block_b200 import synth
from tests.gpu_util import assert_payload_equal, assert_y_equal, run_fused, run_staged, to_dev, tdtype

pytestmark = pytest.mark.gpu

BLOCKS = [32, 64, 128, 256, 512, 1024, 2048, 4096]


def check_all(xs, dtype, bits, block, staged=True):
    y_ref, p1_ref, p2_ref = oracle.allreduce(list(xs), dtype, bits, block)
    xd = to_dev(xs, dtype)
    y, s1, s2 = run_fused(xd, bits, block)
    assert_y_equal(y, y_ref, "fused y")
    for r in range(len(xs)):
        assert_payload_equal(s1[r], p1_ref[r], f"fused step1[{r}]")
    assert_payload_equal(s2, p2_ref, "fused step2")
    y_only, _, _ = run_fused(xd, bits, block, with_payloads=False)
    assert_y_equal(y_only, y_ref, "fused y (no payloads)")
    if staged:
        y_st, s1_st, s2_st = run_staged(xd, bits, block)
        for r in range(len(xs)):
            assert_payload_equal(s1_st[r], p1_ref[r], f"staged step1[{r}]")
        assert_payload_equal(s2_st, p2_ref, "staged step2")
        assert_y_equal(y_st, y_ref, "staged y")


@pytest.mark.parametrize("w", [synth.SMALL_P2, synth.DECODE_P4], ids=lambda w: w.name)
def test_small_workloads_in_full(w):
    check_all(synth.workload_partials(w), w.dtype, w.bits, w.block)


@pytest.mark.parametrize("dtype", [oracle.FP16, oracle.BF16], ids=["fp16", "bf16"])
@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("block", [2048, 4096])
@pytest.mark.parametrize("P,m", [(1, 5), (3, 3)])
def test_blocks_spanning_warps_with_a_partly_empty_last_tile(dtype, bits, block, P, m):
    """An odd number of blocks of 2048 or 4096: the staged kernels' 8192-element tiles
    leave the last one partly empty, so some threads of a CTA hold no block but still
    take part in its cross-warp reduction (the step-1 kernel issues its next loads
    before that barrier for these blocks)."""
    n = P * block * m
    assert (n // block) % 2 == 1
    xs = synth.partials(P, n // block, block, dtype, 0.05, 20.0, seed=700 + P + bits + dtype + block // 1024)
    check_all(xs, dtype, bits, block, staged=True)


@pytest.mark.parametrize("dtype", [oracle.FP16, oracle.BF16], ids=["fp16", "bf16"])
@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("block", BLOCKS)
@pytest.mark.parametrize("P", [1, 2, 3, 4, 8])
def test_sweep_ragged(dtype, bits, block, P):
    # several 4096-element tiles plus a ragged tail (n not a multiple of 4096)
    m = (3 * 4096) // (P * block) + 3
    n = P * block * m
    seed = block * 10 + P + bits + dtype
    xs = synth.partials(P, n // block, block, dtype, 0.05, 20.0, seed=seed)
    check_all(xs, dtype, bits, block, staged=(P in (1, 3, 8)))


@pytest.mark.parametrize("dtype", [oracle.FP16, oracle.BF16], ids=["fp16", "bf16"])
@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("block", [32, 64, 128, 1024, 4096])
@pytest.mark.parametrize("P", [5, 6, 7])
def test_rank_counts_between_powers_of_two(dtype, bits, block, P):
    """P = 5..7: the fused kernel gathers each lane's rank extremes by a
    reduce-scatter over 8 lane slots, three to one of them standing in for
    rank 0 -- with groups narrower than P (blocks of 32 at E = 16: every lane
    computes every rank), groups of at least 8 lanes inside a warp (64, 128)
    and blocks that span warps (1024, 4096); several tiles and a ragged tail."""
    m = (3 * 4096) // (P * block) + 2
    n = P * block * m
    xs = synth.partials(P, n // block, block, dtype, 0.05, 20.0, seed=300 + 10 * P + block + bits + dtype)
    check_all(xs, dtype, bits, block, staged=(block == 128))


@pytest.mark.parametrize("dtype", [oracle.FP16, oracle.BF16], ids=["fp16", "bf16"])
@pytest.mark.parametrize("bits", [8, 4])
def test_zeros_and_sparse(dtype, bits):
    P, block = 4, 128
    xs = synth.uniform_partials(P, P * block * 40, dtype, seed=5, zero_frac=0.9)
    xs[:, : 2 * block * P] = 0            # whole all-zero blocks in every rank
    xs[1, 5 * block: 6 * block] = 0x8000 if dtype == oracle.FP16 else 0x8000   # negative zeros
    check_all(xs, dtype, bits, block)


@pytest.mark.parametrize("bits", [8, 4])
def test_fp16_extremes(bits):
    """Largest finite, subnormal and mixed-sign values; sums that overflow fp16."""
    P, block, n = 8, 64, 8 * 64 * 9
    rng = np.random.default_rng(3)
    vals = np.array([65504.0, -65504.0, 2.0 ** -24, -(2.0 ** -24), 2.0 ** -14, 1.0, -1.0, 0.0],
                    dtype=np.float32)
    x = rng.choice(vals, size=(P, n)).astype(np.float16).view(np.uint16)
    x[:, :block] = np.float16(65504.0).view(np.uint16)           # block summing to inf
    x[:, block:2 * block] = np.float16(2.0 ** -24).view(np.uint16)   # subnormal-only block
    check_all(x, oracle.FP16, bits, block)


@pytest.mark.parametrize("bits", [8, 4])
def test_bf16_wide_and_tiny_ranges(bits):
    """bf16 blocks with ranges from 2^-90 to 2^90 (inside the documented span)."""
    P, block = 3, 256
    nb = 24
    rng = np.random.default_rng(4)
    z = rng.standard_normal((P, nb, block)).astype(np.float32)
    mag = (2.0 ** rng.integers(-90, 90, size=(1, nb, 1))).astype(np.float32)
    x32 = (z * mag).reshape(P, -1)
    xs = np.stack([torch.from_numpy(r).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
                   for r in x32])
    check_all(xs, oracle.BF16, bits, block)


def test_single_block_and_empty():
    for P in (1, 4):
        xs = synth.uniform_partials(P, P * 128, oracle.FP16, seed=P)
        check_all(xs, oracle.FP16, 8, 128)
    # n == 0: a no-op that leaves the output untouched
    e = [torch.empty(0, dtype=torch.float16, device="cuda") for _ in range(2)]
    y = torch.full((1,), 7.0, dtype=torch.float16, device="cuda")
    fc.fc_quantized_allreduce(e, 8, 128, y=y[:0])
    torch.cuda.synchronize()
    assert y.item() == 7.0


def test_staged_and_fused_calls_on_a_side_stream():
    xs = synth.uniform_partials(2, 2 * 128 * 64, oracle.FP16, seed=8)
    y_ref, _, _ = oracle.allreduce(list(xs), oracle.FP16, 8, 128)
    xd = to_dev(xs, oracle.FP16)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        y = fc.fc_quantized_allreduce(xd, 8, 128)
    s.synchronize()
    assert_y_equal(y, y_ref, "side stream")


def _at_16_mod_32(t):
    """A copy of t whose data pointer is 16-byte but not 32-byte aligned."""
    pad = 32 // t.element_size()
    buf = torch.empty(t.numel() + pad, dtype=t.dtype, device=t.device)
    v = buf[pad // 2: pad // 2 + t.numel()]
    assert v.data_ptr() % 32 == 16
    v.copy_(t)
    return v


def _qbuf_at_16_mod_32(n, bits, block):
    q = fc.QBuf.empty(n, bits, block)
    return fc.QBuf(_at_16_mod_32(q.codes), _at_16_mod_32(q.scales), _at_16_mod_32(q.zps), n, bits, block)


@pytest.mark.parametrize("dtype", [oracle.FP16, oracle.BF16], ids=["fp16", "bf16"])
@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("block", [32, 128, 1024])
@pytest.mark.parametrize("P", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("which", ["all", "y", "x_last"])
def test_buffers_aligned_to_16_but_not_32(dtype, bits, block, P, which):
    """The kernels move 32 bytes per access when every pointer allows it and
    16 bytes otherwise; both forms give the oracle's bits.  `which` names the
    buffers placed at an address that is 16 mod 32."""
    m = (2 * 4096) // (P * block) + 3
    n = P * block * m
    xs = synth.partials(P, n // block, block, dtype, 0.05, 20.0, seed=900 + block + P + bits)
    y_ref, p1_ref, p2_ref = oracle.allreduce(list(xs), dtype, bits, block)
    xd = to_dev(xs, dtype)
    if which in ("all", "x_last"):
        xd[-1] = _at_16_mod_32(xd[-1])
    if which == "all":
        xd = [_at_16_mod_32(x) for x in xd]
    y = torch.empty(n, dtype=tdtype(dtype), device="cuda")
    if which in ("all", "y"):
        y = _at_16_mod_32(y)
    mk = _qbuf_at_16_mod_32 if which == "all" else fc.QBuf.empty
    s1 = [mk(n, bits, block) for _ in range(P)]
    s2 = mk(n, bits, block)
    fc.fc_quantized_allreduce(xd, bits, block, y=y, step1=s1, step2=s2)
    torch.cuda.synchronize()
    assert_y_equal(y, y_ref, f"fused y ({which})")
    for r in range(P):
        assert_payload_equal(s1[r], p1_ref[r], f"fused step1[{r}] ({which})")
    assert_payload_equal(s2, p2_ref, f"fused step2 ({which})")
    # the all-gather step alone, reading the payload just written
    y2 = torch.empty(n, dtype=tdtype(dtype), device="cuda")
    if which in ("all", "y"):
        y2 = _at_16_mod_32(y2)
    fc.fc_ag_dequant(s2, tdtype(dtype), y=y2)
    torch.cuda.synchronize()
    assert_y_equal(y2, y_ref, f"staged y ({which})")


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("P", [2, 3, 8])
def test_reduce_scatter_on_a_block_range(bits, P):
    """Every block of the reduce-scatter depends only on the same block of the
    P inputs, so the call on any block-aligned range (pointers offset into the
    payloads, a length that need not be a multiple of P blocks -- one owner's
    chunk in a P-GPU run) gives those blocks of the whole call."""
    block, nblk, k0, k = 64, 48, 16, 5
    n = nblk * block
    xs = synth.partials(P, nblk, block, oracle.FP16, 0.05, 20.0, seed=40 + P + bits)
    p1 = [oracle.quantize(x, oracle.FP16, bits, block) for x in xs]
    p2 = oracle.rs_dequant_sum_requant(p1)
    dev = [fc.QBuf(torch.from_numpy(p.codes).cuda(), torch.from_numpy(p.scales).cuda(),
                   torch.from_numpy(p.zps).cuda(), n, bits, block) for p in p1]
    cb = block * bits // 8

    def sub(q):
        return fc.PeerQBuf(q.codes.data_ptr() + k0 * cb, q.scales.data_ptr() + 4 * k0, q.zps.data_ptr() + k0,
                           k * block, bits, block)
    out = fc.QBuf.empty(k * block, bits, block)
    fc.fc_rs_dequant_sum_requant([sub(q) for q in dev], bits, block, out=out)
    torch.cuda.synchronize()
    assert np.array_equal(out.codes.cpu().numpy(), p2.codes[k0 * cb:(k0 + k) * cb])
    assert np.array_equal(out.scales.cpu().numpy().view(np.uint32), p2.scales[k0:k0 + k].view(np.uint32))
    assert np.array_equal(out.zps.cpu().numpy(), p2.zps[k0:k0 + k])

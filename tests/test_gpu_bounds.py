"""Every entry point writes its outputs and nothing else.  With no memory
checker available for the GPU, each output buffer is placed between two 4 KB
guard regions filled with a byte pattern (optionally 16 bytes off a 32-byte
boundary, the alignment the ABI allows), and after each call the guards must
still hold the pattern and the inputs must be unchanged.  Covered: the fused
all-reduce in both launch shapes (decode-sized messages and the persistent
bandwidth shape) with and without payloads, per-step widths, the three staged
steps, the one-kernel P-rank all-reduce run emulated, its allocation-free
form, and the tensor-core GEMM with the quantizer in its epilogue; sizes that
leave a ragged last tile.  (Reads outside the inputs would show up as wrong
outputs, which the parity tests compare element by element.)"""
import math

import pytest
import torch

import bit_quantized_all_block_b200 as fc

pytestmark = pytest.mark.gpu

G = 4096          # guard bytes on each side
PAT = 0xA5


class Guarded:
    """nbytes of device memory between two guard regions; `off` extra guard
    bytes in front shift the buffer's alignment."""

    def __init__(self, nbytes, off=0, fill=None, device="cuda"):
        self.raw = torch.full((G + off + nbytes + G,), PAT, dtype=torch.uint8, device=device)
        self.lo, self.n = G + off, nbytes
        self.view = self.raw[self.lo:self.lo + nbytes]
        if fill is not None:
            self.view.fill_(fill)

    def as_(self, dtype):
        return self.view.view(dtype)

    def intact(self):
        return bool((self.raw[:self.lo] == PAT).all()) and bool((self.raw[self.lo + self.n:] == PAT).all())


def guarded_payload(n, bits, block, off, keep):
    cb, nb = fc.fc_payload_sizes(n, bits, block)
    c, s, z = Guarded(cb, off), Guarded(4 * nb, off), Guarded(nb, off)
    keep += [c, s, z]
    return fc.QBuf(c.view, s.as_(torch.float32), z.view, n, bits, block)


def partials(P, n, dtype, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    return [(torch.randn(n, device="cuda", generator=g) * 3).to(dtype) for _ in range(P)]


def rounded(total, unit):
    return unit * math.ceil(total / unit)


def check(keep, xs, xs_before):
    torch.cuda.synchronize()
    for i, gbuf in enumerate(keep):
        assert gbuf.intact(), f"guard region of output buffer {i} overwritten"
    for x, x0 in zip(xs, xs_before):
        assert torch.equal(x.view(torch.int16), x0.view(torch.int16)), "an input was modified"


SHAPES = {"decode": 30000, "bandwidth": 300000}   # elements per rank, before rounding


@pytest.mark.parametrize("off", [0, 16])
@pytest.mark.parametrize("shape", sorted(SHAPES))
@pytest.mark.parametrize("P,bits,block,dtype", [
    (2, 8, 128, torch.float16), (4, 4, 64, torch.bfloat16), (8, 4, 1024, torch.float16),
    (4, 8, 256, torch.bfloat16), (8, 8, 32, torch.bfloat16), (3, 4, 128, torch.float16),
])
def test_fused_writes_only_its_outputs(P, bits, block, dtype, shape, off):
    base = SHAPES[shape] * (2 if P == 2 else 1)
    n = rounded(base, P * block)
    xs = partials(P, n, dtype, 7 * P + bits)
    xs0 = [x.clone() for x in xs]
    keep = []
    y = Guarded(2 * n, off)
    keep.append(y)
    s1 = [guarded_payload(n, bits, block, off, keep) for _ in range(P)]
    s2 = guarded_payload(n, bits, block, off, keep)
    fc.fc_quantized_allreduce(xs, bits, block, y=y.as_(dtype), step1=s1, step2=s2)
    y2 = Guarded(2 * n, off)
    keep.append(y2)
    fc.fc_quantized_allreduce(xs, bits, block, y=y2.as_(dtype))
    check(keep, xs, xs0)
    assert torch.equal(y.as_(torch.int16), y2.as_(torch.int16))


@pytest.mark.parametrize("bits_rs,bits_ag", [(8, 4), (4, 8), (16, 8), (4, 16), (16, 16)])
@pytest.mark.parametrize("off", [0, 16])
def test_per_step_widths_write_only_their_outputs(bits_rs, bits_ag, off):
    P, block, dtype = 4, 128, torch.float16
    n = rounded(SHAPES["bandwidth"], P * block)
    xs = partials(P, n, dtype, 40 + bits_rs + bits_ag)
    xs0 = [x.clone() for x in xs]
    keep = []
    y = Guarded(2 * n, off)
    keep.append(y)
    s1 = [guarded_payload(n, bits_rs, block, off, keep) for _ in range(P)] if bits_rs != 16 else None
    s2 = guarded_payload(n, bits_ag, block, off, keep) if bits_ag != 16 else None
    fc.fc_quantized_allreduce_ex(xs, bits_rs, bits_ag, block, y=y.as_(dtype), step1=s1, step2=s2)
    check(keep, xs, xs0)


@pytest.mark.parametrize("P,bits,block,dtype", [(4, 8, 128, torch.float16), (8, 4, 4096, torch.bfloat16),
                                                (2, 4, 32, torch.bfloat16)])
@pytest.mark.parametrize("off", [0, 16])
def test_staged_steps_write_only_their_outputs(P, bits, block, dtype, off):
    n = rounded(SHAPES["bandwidth"], P * block)
    xs = partials(P, n, dtype, 60 + P)
    xs0 = [x.clone() for x in xs]
    keep = []
    s1 = [guarded_payload(n, bits, block, off, keep) for _ in range(P)]
    for x, q in zip(xs, s1):
        fc.fc_quantize(x, bits, block, out=q)
    torch.cuda.synchronize()
    s1_0 = [(q.codes.clone(), q.scales.clone(), q.zps.clone()) for q in s1]
    s2 = guarded_payload(n, bits, block, off, keep)
    fc.fc_rs_dequant_sum_requant(s1, bits, block, out=s2)
    y = Guarded(2 * n, off)
    keep.append(y)
    fc.fc_ag_dequant(s2, dtype, y=y.as_(dtype))
    check(keep, xs, xs0)
    for q, (c, s, z) in zip(s1, s1_0):      # the reduce-scatter's inputs are untouched
        assert torch.equal(q.codes, c) and torch.equal(q.zps, z)
        assert torch.equal(q.scales.view(torch.int32), s.view(torch.int32))


@pytest.mark.parametrize("P,bits,block", [(2, 8, 128), (4, 4, 64), (8, 8, 1024)])
def test_one_kernel_all_reduce_writes_only_its_buffers(P, bits, block):
    dtype = torch.float16
    n = rounded(SHAPES["bandwidth"], P * block)
    m = n // P
    xs = partials(P, n, dtype, 80 + P)
    xs0 = [x.clone() for x in xs]
    keep = []
    ys = [Guarded(2 * n, 16) for _ in range(P)]
    keep += ys
    s1 = [guarded_payload(m, bits, block, 0, keep) for _ in range(P * P)]
    s2 = [guarded_payload(m, bits, block, 16, keep) for _ in range(P)]
    ctr = Guarded(8 * P, 0, fill=0)
    status = Guarded(4, 0, fill=0)
    keep += [ctr, status]
    base = ctr.view.data_ptr()
    fc.fc_p2p_allreduce_emulated(xs, [g.as_(dtype) for g in ys], bits, block, s1, s2,
                                 [base + 4 * p for p in range(P)], [base + 4 * (P + p) for p in range(P)],
                                 1, status.as_(torch.int32))
    check(keep, xs, xs0)
    assert int(status.as_(torch.int32).item()) == 0

    ys2 = [Guarded(2 * n, 0) for _ in range(P)]
    st2 = Guarded(4, 0, fill=0)
    fc.fc_p2p_allreduce_emulated_noalloc(xs, [g.as_(dtype) for g in ys2], bits, block, status=st2.as_(torch.int32))
    check(ys2 + [st2], xs, xs0)
    assert int(st2.as_(torch.int32).item()) == 0
    for a, b in zip(ys, ys2):
        assert torch.equal(a.as_(torch.int16), b.as_(torch.int16))


@pytest.mark.parametrize("M,N,K,bits,block", [(256, 512, 128, 8, 128), (128, 256, 64, 4, 32)])
def test_gemm_writes_only_its_outputs(M, N, K, bits, block):
    dtype = torch.bfloat16
    g = torch.Generator(device="cuda").manual_seed(M + N + K)
    a = torch.randn(M, K, device="cuda", generator=g).to(dtype)
    w = torch.randn(N, K, device="cuda", generator=g).to(dtype)
    a0, w0 = a.clone(), w.clone()
    keep = []
    part = Guarded(2 * M * N, 16)
    keep.append(part)
    out = guarded_payload(M * N, bits, block, 16, keep)
    status = Guarded(16, 0, fill=0)
    keep.append(status)
    fc.fc_gemm_quantize(a, w, bits, block, out=out, partial=part.as_(dtype).view(M, N),
                        status=status.as_(torch.int32))
    check(keep, [a, w], [a0, w0])
    assert int(status.as_(torch.int32)[0].item()) == 0

"""Randomized GPU parity: seeded random configurations -- P from 1 to 8, every
block size from 32 to 4096, INT8/INT4, fp16/bf16, chunk lengths from one block
up, so both launch shapes of the fused kernel and ragged tiles occur -- with
inputs that mix, block by block, values across each format's range, all-zero
and constant blocks, one-signed blocks, fp16 subnormals and outliers.  The
fused all-reduce (with both payloads, output buffer at a random 16- or
32-byte alignment), the staged pipeline and a random per-step-width call must
equal the CPU oracle bit for bit."""
import numpy as np
import pytest
import torch

import bit_quantized_all_block_b200 as fc
import oracle
from tests.gpu_util import assert_payload_equal, assert_y_equal, tdtype

pytestmark = pytest.mark.gpu

BLOCKS = [32, 64, 128, 256, 512, 1024, 2048, 4096]


def random_blocks(rng, n, block, dtype):
    """n values (fp16/bf16 bit patterns) built block by block from a random kind."""
    lo, hi = (-8, 4) if dtype == oracle.FP16 else (-40, 40)
    v = np.empty(n, dtype=np.float32)
    for k in range(n // block):
        scale = np.float32(2.0 ** rng.integers(lo, hi + 1))
        kind = rng.integers(0, 8)
        x = rng.standard_normal(block).astype(np.float32) * scale
        if kind == 1:
            x[:] = 0
        elif kind == 2:
            x[:] = x[0]
        elif kind == 3:
            x = np.abs(x)
        elif kind == 4:
            x = -np.abs(x)
        elif kind == 5 and dtype == oracle.FP16:
            x = (rng.integers(-1023, 1024, block) * 2.0 ** -24).astype(np.float32)    # subnormals
        elif kind == 6:
            x[rng.integers(0, block)] *= 32
        v[k * block:(k + 1) * block] = x
    t = torch.from_numpy(v).to(torch.float16 if dtype == oracle.FP16 else torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def offset_output(n, dt, off_bytes):
    """An n-element output at `off_bytes` past a 256-byte boundary."""
    raw = torch.empty(n + 16, dtype=dt, device="cuda")
    return raw[off_bytes // 2:off_bytes // 2 + n]


@pytest.mark.parametrize("seed", range(40))
def test_random_configuration(seed):
    rng = np.random.default_rng(1000 + seed)
    P = int(rng.integers(1, 9))
    bits = int(rng.choice([4, 8]))
    block = int(rng.choice(BLOCKS))
    dtype = int(rng.choice([oracle.FP16, oracle.BF16]))
    k = int(rng.choice([1, 2, 3, 5, 8, 13, 40]))
    n = P * block * k
    xs = np.stack([random_blocks(rng, n, block, dtype) for _ in range(P)])
    dt = tdtype(dtype)
    xd = [torch.from_numpy(x.view(np.int16).copy()).view(dt).cuda() for x in xs]

    y_ref, p1_ref, p2_ref = oracle.allreduce(list(xs), dtype, bits, block)
    y = offset_output(n, dt, int(rng.choice([0, 16])))
    s1 = [fc.QBuf.empty(n, bits, block) for _ in range(P)]
    s2 = fc.QBuf.empty(n, bits, block)
    fc.fc_quantized_allreduce(xd, bits, block, y=y, step1=s1, step2=s2)
    q1 = [fc.fc_quantize(x, bits, block) for x in xd]
    q2 = fc.fc_rs_dequant_sum_requant(q1, bits, block)
    y_st = fc.fc_ag_dequant(q2, dt)
    torch.cuda.synchronize()
    what = f"P={P} bits={bits} block={block} dtype={dtype} n={n}"
    assert_y_equal(y, y_ref, "fused " + what)
    assert_y_equal(y_st, y_ref, "staged " + what)
    for r in range(P):
        assert_payload_equal(s1[r], p1_ref[r], f"fused step1[{r}] " + what)
        assert_payload_equal(q1[r], p1_ref[r], f"staged step1[{r}] " + what)
    assert_payload_equal(s2, p2_ref, "fused step2 " + what)
    assert_payload_equal(q2, p2_ref, "staged step2 " + what)

    b_rs, b_ag = (int(b) for b in rng.choice([4, 8, 16], size=2))
    if (b_rs != b_ag or b_rs == 16) and P not in (2, 4, 8):
        return                     # provided for P in {2, 4, 8} only (equal quantized widths: every P)
    y_ex_ref, _, _ = oracle.allreduce_ex(list(xs), dtype, b_rs, b_ag, block)
    y_ex = fc.fc_quantized_allreduce_ex(xd, b_rs, b_ag, block)
    torch.cuda.synchronize()
    assert_y_equal(y_ex, y_ex_ref, f"widths ({b_rs}, {b_ag}) " + what)

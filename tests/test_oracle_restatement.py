"""C oracle == numpy restatement, bit for bit, on seeded synthetic partials."""
import numpy as np
import pytest
import torch

import oracle
from bit_quantized_all_block_b200 import synth
from tests import np_restatement as npr


def narrow_lib(v, dtype):
    if dtype == oracle.FP16:
        return v.astype(np.float16).view(np.uint16)
    return torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


CASES = [
    (synth.SMALL_P2, None),
    (synth.DECODE_P4, None),
    (synth.PREFILL_70B_INT8, 2),
    (synth.PREFILL_70B_INT4, 2),
] + [(w, 8) for w in synth.BLOCK_SWEEP_8B]


@pytest.mark.parametrize("w,rows", CASES, ids=[c[0].name for c in CASES])
def test_oracle_matches_restatement(w, rows):
    xs = synth.workload_partials(w, rows=rows)
    y, p1, p2 = oracle.allreduce(list(xs), w.dtype, w.bits, w.block)
    v = [oracle.widen(x, w.dtype) for x in xs]
    q1s, s1s, z1s, q2, s2, z2, xh2 = npr.allreduce(v, w.bits, w.block)
    for r in range(w.P):
        assert np.array_equal(p1[r].codes, npr.pack(q1s[r], w.bits))
        assert np.array_equal(p1[r].scales.view(np.uint32), s1s[r].view(np.uint32))
        assert np.array_equal(p1[r].zps, z1s[r].astype(np.uint8))
    assert np.array_equal(p2.codes, npr.pack(q2, w.bits))
    assert np.array_equal(p2.scales.view(np.uint32), s2.view(np.uint32))
    assert np.array_equal(y, narrow_lib(xh2, w.dtype))


@pytest.mark.parametrize("block", [2, 6, 32, 96, 4096])
@pytest.mark.parametrize("bits", [8, 4])
def test_odd_shapes(block, bits):
    P = 3
    xs = synth.uniform_partials(P, P * block * 2, oracle.BF16, seed=block, zero_frac=0.2)
    y, p1, p2 = oracle.allreduce(list(xs), oracle.BF16, bits, block)
    v = [oracle.widen(x, oracle.BF16) for x in xs]
    *_, q2, s2, z2, xh2 = npr.allreduce(v, bits, block)
    assert np.array_equal(p2.codes, npr.pack(q2, bits))
    assert np.array_equal(y, narrow_lib(xh2, oracle.BF16))

"""Full-size GPU parity: the fused all-reduce runs on the whole workload (the
launch bench.py times, payloads written) and its whole output and every
payload are checked bit for bit against the CPU oracle run over every token
row (on all host cores: every block depends only on the same block of every
rank, so row slices are independent all-reduces).  The staged pipeline is
compared with the fused kernel on the whole output."""
import functools

import numpy as np
import pytest
import torch

import bit_quantized_all_block_b200 as fc
from bit_quantized_all_block_b200 import synth
from tests.gpu_util import to_dev
from tests.oracle_rows import allreduce_all_rows

pytestmark = pytest.mark.gpu

FULL = [synth.PREFILL_70B_INT8, synth.PREFILL_70B_INT4, *synth.BLOCK_SWEEP_8B]


@functools.lru_cache(maxsize=1)
def inputs(P, T, H, dtype, frac, factor, seed):
    return synth.partials(P, T, H, dtype, frac, factor, seed)


@pytest.mark.parametrize("w", FULL, ids=lambda w: w.name)
def test_full_size_every_output(w):
    xs = inputs(w.P, w.T, w.H, w.dtype, w.outlier_frac, w.outlier_factor, w.seed)
    xd = to_dev(xs, w.dtype)
    s1 = [fc.QBuf.empty(w.n, w.bits, w.block) for _ in range(w.P)]
    s2 = fc.QBuf.empty(w.n, w.bits, w.block)
    y = fc.fc_quantized_allreduce(xd, w.bits, w.block, step1=s1, step2=s2)
    torch.cuda.synchronize()

    y_ref, p1_ref, p2_ref = allreduce_all_rows(xs, w.T, w.H, w.dtype, w.bits, w.block)
    got = y.view(torch.int16).cpu().numpy().view(np.uint16)
    bad = np.nonzero(got != y_ref)[0]
    assert bad.size == 0, f"{bad.size} of {got.size} outputs differ, first at {bad[:8]}"
    for q, (codes, scales, zps) in zip(s1 + [s2], p1_ref + [p2_ref]):
        assert np.array_equal(q.codes.cpu().numpy(), codes)
        assert np.array_equal(q.scales.cpu().numpy().view(np.uint32), scales.view(np.uint32))
        assert np.array_equal(q.zps.cpu().numpy(), zps)

    # staged pipeline == fused kernel on the whole tensor
    q1 = [fc.fc_quantize(x, w.bits, w.block) for x in xd]
    q2 = fc.fc_rs_dequant_sum_requant(q1, w.bits, w.block)
    y_st = fc.fc_ag_dequant(q2, xd[0].dtype)
    torch.cuda.synchronize()
    assert torch.equal(y_st.view(torch.int16), y.view(torch.int16))
    assert torch.equal(q2.codes, s2.codes) and torch.equal(q2.zps, s2.zps)
    assert torch.equal(q2.scales.view(torch.int32), s2.scales.view(torch.int32))
    for a, b in zip(q1, s1):
        assert torch.equal(a.codes, b.codes)


@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("lg", [13, 16, 20, 24])
def test_message_sweep_points(bits, lg):
    """Message sizes of the sweep (2^lg fp16 elements per rank, P=4) in full."""
    w = [v for v in synth.message_sweep(bits) if v.n == 1 << lg][0]
    xs = synth.workload_partials(w)
    xd = to_dev(xs, w.dtype)
    y = fc.fc_quantized_allreduce(xd, w.bits, w.block)
    torch.cuda.synchronize()
    y_ref, _, _ = allreduce_all_rows(xs, w.T, w.H, w.dtype, w.bits, w.block)
    assert np.array_equal(y.view(torch.int16).cpu().numpy().view(np.uint16), y_ref)

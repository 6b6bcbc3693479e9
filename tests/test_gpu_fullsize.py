"""Full-size GPU parity: the fused all-reduce runs on the whole workload (the
launch bench.py times, payloads written), then sampled token rows -- first,
last and seeded random rows -- are checked bit for bit against the oracle run
on exactly those rows (every block depends only on the same block of every
rank, so a row sample is an independent all-reduce).  The staged pipeline is
compared with the fused kernel on the whole output."""
import functools

import numpy as np
import pytest
import torch

import bit_quantized_all_block_b200 as fc
import oracle
from bit_quantized_all_block_b200 import synth
from tests.gpu_util import to_dev

pytestmark = pytest.mark.gpu

FULL = [synth.PREFILL_70B_INT8, synth.PREFILL_70B_INT4, *synth.BLOCK_SWEEP_8B]


@functools.lru_cache(maxsize=1)
def inputs(P, T, H, dtype, frac, factor, seed):
    return synth.partials(P, T, H, dtype, frac, factor, seed)


def sample_rows(T, k=16, seed=0):
    rng = np.random.default_rng(seed)
    mid = rng.choice(np.arange(8, T - 8), size=k, replace=False)
    return np.sort(np.concatenate([np.arange(8), mid, np.arange(T - 8, T)]))


def rows_of(a, rows, width):
    return a.reshape(-1, width)[rows].ravel()


@pytest.mark.parametrize("w", FULL, ids=lambda w: w.name)
def test_full_size_sampled_rows(w):
    xs = inputs(w.P, w.T, w.H, w.dtype, w.outlier_frac, w.outlier_factor, w.seed)
    xd = to_dev(xs, w.dtype)
    s1 = [fc.QBuf.empty(w.n, w.bits, w.block) for _ in range(w.P)]
    s2 = fc.QBuf.empty(w.n, w.bits, w.block)
    y = fc.fc_quantized_allreduce(xd, w.bits, w.block, step1=s1, step2=s2)
    torch.cuda.synchronize()

    rows = sample_rows(w.T, seed=w.block)
    sub = [rows_of(x, rows, w.H) for x in xs]
    y_ref, p1_ref, p2_ref = oracle.allreduce(sub, w.dtype, w.bits, w.block)
    idx = torch.from_numpy(rows).cuda()
    y_rows = y.view(w.T, w.H)[idx].contiguous().view(torch.int16).cpu().numpy().view(np.uint16).ravel()
    assert np.array_equal(y_rows, y_ref)

    cb_row = w.H * w.bits // 8            # code bytes per token row
    nb_row = w.H // w.block               # blocks per token row
    for q, p in zip(s1 + [s2], p1_ref + [p2_ref]):
        assert np.array_equal(q.codes.view(w.T, cb_row)[idx].cpu().numpy().ravel(), p.codes)
        assert np.array_equal(q.scales.view(w.T, nb_row)[idx].cpu().numpy().ravel().view(np.uint32),
                              p.scales.view(np.uint32))
        assert np.array_equal(q.zps.view(w.T, nb_row)[idx].cpu().numpy().ravel(), p.zps)

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
    """Decode-regime message sizes (2^lg fp16 elements per rank, P=4) in full."""
    w = [v for v in synth.message_sweep(bits) if v.n == 1 << lg][0]
    xs = synth.workload_partials(w)
    rows = np.arange(w.T) if w.T <= 64 else sample_rows(w.T, seed=lg)
    xd = to_dev(xs, w.dtype)
    y = fc.fc_quantized_allreduce(xd, w.bits, w.block)
    torch.cuda.synchronize()
    sub = [rows_of(x, rows, w.H) for x in xs]
    y_ref, _, _ = oracle.allreduce(sub, w.dtype, w.bits, w.block)
    idx = torch.from_numpy(rows).cuda()
    y_rows = y.view(w.T, w.H)[idx].contiguous().view(torch.int16).cpu().numpy().view(np.uint16).ravel()
    assert np.array_equal(y_rows, y_ref)

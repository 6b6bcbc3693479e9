"""Per-step precision (Flash Communication, Fig. 5 right: quantization error
before Reduce-Scatter vs before All-Gather): the oracle's fco_allreduce_ex.

Each combination reduces to pinned pieces:
  (b, b)   == the two-step all-reduce already pinned (fco_allreduce);
  (16, 16) == library rounding of the fp32 sequential sum (numpy / torch);
  (16, b)  == quantize-dequantize of that fp32 sum;
  (b, 16)  == library rounding of the sum of the dequantized step-1 values;
  mixed    == step 1 at one width, step 2 at the other.
Plus the error bound with only the quantized steps' s/2 terms, and the MSE
ordering the figure is about (each quantized step adds error)."""
import numpy as np
import pytest
import torch

import oracle
from bit_quantized_all_block_b200 import synth

WIDTHS = [4, 8, 16]


def lib_narrow(v32, dtype):
    if dtype == oracle.FP16:
        return np.asarray(v32, np.float32).astype(np.float16).view(np.uint16)
    return torch.from_numpy(np.asarray(v32, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def seq_sum(vs):
    acc = vs[0].astype(np.float32).copy()
    for v in vs[1:]:
        acc = (acc + v.astype(np.float32)).astype(np.float32)
    return acc


def case(dtype, P=3, block=64, rows=24, seed=7):
    return list(synth.partials(P, rows, 4 * block, dtype, 0.05, 20.0, seed=seed))


@pytest.mark.parametrize("dtype", [oracle.FP16, oracle.BF16])
@pytest.mark.parametrize("b1", WIDTHS)
@pytest.mark.parametrize("b2", WIDTHS)
def test_reduces_to_pinned_pieces(dtype, b1, b2):
    block = 64
    xs = case(dtype, block=block)
    y, p1, p2 = oracle.allreduce_ex(xs, dtype, b1, b2, block)
    assert (p1 is None) == (b1 == 16) and (p2 is None) == (b2 == 16)
    if b1 == 16:
        contrib = [oracle.widen(x, dtype) for x in xs]
    else:
        q = [oracle.quantize(x, dtype, b1, block) for x in xs]
        for a, b in zip(q, p1):
            assert np.array_equal(a.codes, b.codes) and np.array_equal(a.zps, b.zps)
        contrib = [oracle.dequantize(p) for p in q]
    S = seq_sum(contrib)
    if b2 == 16:
        assert np.array_equal(y, lib_narrow(S, dtype))
    else:
        q2 = oracle.quantize_f32(S, b2, block)
        assert np.array_equal(q2.codes, p2.codes) and np.array_equal(q2.scales, p2.scales)
        assert np.array_equal(y, lib_narrow(oracle.dequantize(q2), dtype))
    if b1 == b2 and b1 != 16:
        y0, _, p20 = oracle.allreduce(xs, dtype, b1, block)
        assert np.array_equal(y, y0) and np.array_equal(p2.codes, p20.codes)


@pytest.mark.parametrize("b1", WIDTHS)
@pytest.mark.parametrize("b2", WIDTHS)
def test_error_bound_per_variant(b1, b2):
    block, P = 128, 4
    xs = list(synth.partials(P, 32, 1024, oracle.FP16, 0.01, 20.0, seed=3))
    y, p1, p2 = oracle.allreduce_ex(xs, oracle.FP16, b1, b2, block)
    v = np.stack([oracle.widen(x, oracle.FP16).astype(np.float64) for x in xs])
    exact = v.sum(0)
    yv = oracle.widen(y, oracle.FP16).astype(np.float64)
    bound = np.zeros_like(exact)
    if b1 != 16:
        step = 0.5 + ((1 << b1) - 1) * 2.0 ** -21
        bound += step * np.stack([np.repeat(p.scales.astype(np.float64), block) for p in p1]).sum(0)
    if b2 != 16:
        step = 0.5 + ((1 << b2) - 1) * 2.0 ** -21
        bound += step * np.repeat(p2.scales.astype(np.float64), block)
    bound += P * 2.0 ** -24 * (np.abs(v).sum(0) + bound) + 2.0 ** -11 * np.abs(yv) + 2.0 ** -24
    assert np.all(np.abs(yv - exact) <= bound)


def test_mse_ordering():
    """More quantized steps or fewer bits -> larger error against the fp32 sum."""
    w = synth.PREFILL_70B_INT8
    xs = list(synth.workload_partials(w, rows=64))
    S = seq_sum([oracle.widen(x, w.dtype) for x in xs]).astype(np.float64)

    def mse(b1, b2):
        y, _, _ = oracle.allreduce_ex(xs, w.dtype, b1, b2, 128)
        return float(np.mean((oracle.widen(y, w.dtype).astype(np.float64) - S) ** 2))

    m = {(b1, b2): mse(b1, b2) for b1 in WIDTHS for b2 in WIDTHS}
    assert m[16, 16] < m[16, 8] < m[8, 8] < m[8, 4] < m[4, 4]
    assert m[16, 16] < m[8, 16] < m[8, 8] < m[4, 8] < m[4, 4]
    assert m[8, 16] < m[4, 16] and m[16, 8] < m[16, 4]


def test_bad_widths():
    xs = case(oracle.FP16)
    for b1, b2 in [(2, 8), (8, 12), (16, 3)]:
        with pytest.raises(oracle.OracleError):
            oracle.allreduce_ex(xs, oracle.FP16, b1, b2, 64)

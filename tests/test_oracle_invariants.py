"""Oracle invariants and closed forms (no re-evaluation of its formulas).

* exact round trip of representable grids (s = 2^-k, codes 0 and qmax present);
* P = 1 reduces to quantize -> dequantize -> requantize -> dequantize;
* P ranks whose blocks are grid values and whose sums are exact give the
  exact sum, whatever the rank order;
* scaling every input by 2^j scales every scale and output by 2^j and leaves
  codes and zero-points alone;
* permuting the elements of each block permutes codes and outputs;
* each block's results depend on that block only;
* all-zero input gives s = 1, z = 0, q = 0, y = 0;
* the all-reduce error is within the sum of the per-step bounds.
"""
import numpy as np
import pytest
import torch

import oracle
from bit_quantized_all_block_b200 import synth
from tests.exact import unpack_codes


def bits_of(x32, dtype):
    x32 = np.ascontiguousarray(x32, dtype=np.float32)
    if dtype == oracle.FP16:
        h = x32.astype(np.float16)
        assert np.array_equal(h.astype(np.float32), x32)
        return h.view(np.uint16)
    t = torch.from_numpy(x32).to(torch.bfloat16)
    assert np.array_equal(t.to(torch.float32).numpy(), x32)
    return t.view(torch.int16).numpy().view(np.uint16)


def grid_block(rng, B, bits, k):
    """Codes with 0 and qmax present, random z; values (q - z) 2^-k."""
    qmax = (1 << bits) - 1
    q = rng.integers(0, qmax + 1, size=B)
    q[rng.permutation(B)[:2]] = [0, qmax]
    z = int(rng.integers(0, qmax + 1))
    return q, z, ((q - z) * 2.0 ** -k).astype(np.float32)


@pytest.mark.parametrize("dtype", [oracle.FP16, oracle.BF16])
@pytest.mark.parametrize("bits", [8, 4])
def test_grid_round_trip(dtype, bits):
    rng = np.random.default_rng(1 + bits)
    B, nb = 32, 16
    qs, zs, ks, xs = [], [], [], []
    for _ in range(nb):
        k = int(rng.integers(2, 9))
        q, z, x = grid_block(rng, B, bits, k)   # |q - z| <= 255 fits fp16 and bf16
        qs.append(q); zs.append(z); ks.append(k); xs.append(x)
    x = np.concatenate(xs)
    xb = bits_of(x, dtype)
    p = oracle.quantize(xb, dtype, bits, B)
    assert np.array_equal(unpack_codes(p.codes, x.size, bits), np.concatenate(qs))
    assert p.zps.tolist() == zs
    assert np.array_equal(p.scales, np.array([2.0 ** -k for k in ks], np.float32))
    assert np.array_equal(oracle.dequantize(p), x)
    # P ranks: rank 0 holds the grid, the others hold zeros -> y == x exactly
    P = 4
    xs_r = [xb] + [np.zeros_like(xb) for _ in range(P - 1)]
    y, p1, p2 = oracle.allreduce(xs_r, dtype, bits, B)
    assert np.array_equal(y, xb)
    assert np.array_equal(p2.codes, p.codes) and np.array_equal(p2.zps, p.zps)


@pytest.mark.parametrize("dtype", [oracle.FP16, oracle.BF16])
@pytest.mark.parametrize("bits", [8, 4])
def test_p1_is_two_quantizations(dtype, bits):
    x = synth.uniform_partials(1, 64 * 32, dtype, seed=3)[0]
    y, p1, p2 = oracle.allreduce([x], dtype, bits, 64)
    xh = oracle.dequantize(oracle.quantize(x, dtype, bits, 64))
    q2 = oracle.quantize_f32(xh, bits, 64)
    assert np.array_equal(q2.codes, p2.codes)
    assert np.array_equal(y, oracle.narrow(oracle.dequantize(q2), dtype))


@pytest.mark.parametrize("bits", [8, 4])
def test_exact_sums_are_rank_order_free(bits):
    """Grid-valued partials whose fp32 sums are exact: y is the exact sum for any rank order."""
    rng = np.random.default_rng(11)
    P, B, nb = 4, 16, 8
    # every rank: block values (q - z) * 2^-4 with codes 0 and qmax present
    ranks = []
    for r in range(P):
        ranks.append(np.concatenate([grid_block(rng, B, bits, 4)[2] for _ in range(nb)]))
    xb = [bits_of(x, oracle.FP16) for x in ranks]
    y, _, p2 = oracle.allreduce(xb, oracle.FP16, bits, B)
    for perm in ([3, 2, 1, 0], [1, 3, 0, 2]):
        y2, _, _ = oracle.allreduce([xb[i] for i in perm], oracle.FP16, bits, B)
        assert np.array_equal(y, y2)


@pytest.mark.parametrize("dtype", [oracle.FP16, oracle.BF16])
@pytest.mark.parametrize("bits", [8, 4])
@pytest.mark.parametrize("j", [-3, 2])
def test_power_of_two_scaling(dtype, bits, j):
    P, B = 3, 32
    xs = synth.uniform_partials(P, B * 12, dtype, seed=5, lo=-4.0, hi=4.0)
    # keep magnitudes away from the subnormal range so the scaling is exact
    xs = [oracle.widen(x, dtype) for x in xs]
    xs = [oracle.narrow(np.where(np.abs(x) < 2.0 ** -6, np.float32(0), x), dtype) for x in xs]
    y, p1, p2 = oracle.allreduce(xs, dtype, bits, B)
    xs_s = [bits_of(oracle.widen(x, dtype) * np.float32(2.0 ** j), dtype) for x in xs]
    y_s, p1_s, p2_s = oracle.allreduce(xs_s, dtype, bits, B)
    for a, b in zip(p1 + [p2], p1_s + [p2_s]):
        assert np.array_equal(a.codes, b.codes) and np.array_equal(a.zps, b.zps)
        assert np.array_equal(a.scales * np.float32(2.0 ** j), b.scales)
    assert np.array_equal(oracle.widen(y, dtype) * np.float32(2.0 ** j), oracle.widen(y_s, dtype))


@pytest.mark.parametrize("bits", [8, 4])
def test_permutation_within_blocks(bits):
    P, B, nb = 2, 32, 6
    xs = synth.uniform_partials(P, B * nb, oracle.FP16, seed=9)
    perm = np.random.default_rng(2).permutation(B)
    idx = np.concatenate([k * B + perm for k in range(nb)])
    y, p1, p2 = oracle.allreduce(xs, oracle.FP16, bits, B)
    y_p, p1_p, p2_p = oracle.allreduce([x[idx] for x in xs], oracle.FP16, bits, B)
    assert np.array_equal(y[idx], y_p)
    for a, b in zip(p1 + [p2], p1_p + [p2_p]):
        assert np.array_equal(unpack_codes(a.codes, a.n, bits)[idx], unpack_codes(b.codes, b.n, bits))
        assert np.array_equal(a.scales, b.scales) and np.array_equal(a.zps, b.zps)


def test_blocks_are_independent():
    P, B, nb = 4, 64, 8
    xs = synth.uniform_partials(P, B * nb, oracle.FP16, seed=13)
    y, _, p2 = oracle.allreduce(xs, oracle.FP16, 8, B)
    xs2 = [x.copy() for x in xs]
    xs2[2][3 * B:4 * B] = synth.uniform_partials(1, B, oracle.FP16, seed=14)[0]
    y2, _, p22 = oracle.allreduce(xs2, oracle.FP16, 8, B)
    keep = np.ones(P * 0 + B * nb, bool)
    keep[3 * B:4 * B] = False
    assert np.array_equal(y[keep], y2[keep])
    assert not np.array_equal(y[~keep], y2[~keep])
    assert np.array_equal(np.delete(p2.scales, 3), np.delete(p22.scales, 3))


@pytest.mark.parametrize("bits", [8, 4])
def test_all_zero(bits):
    xs = [np.zeros(256, np.uint16) for _ in range(2)]
    y, p1, p2 = oracle.allreduce(xs, oracle.FP16, bits, 128)
    assert not y.any()
    for p in p1 + [p2]:
        assert not p.codes.any() and not p.zps.any()
        assert np.array_equal(p.scales, np.ones_like(p.scales))


@pytest.mark.parametrize("dtype", [oracle.FP16, oracle.BF16])
@pytest.mark.parametrize("bits", [8, 4])
def test_allreduce_error_bound(dtype, bits):
    """|y - sum_r x_r| <= sum_r s_r/2 + s2/2 + fp32 summation + output rounding."""
    qmax = (1 << bits) - 1
    P, B, nb = 4, 128, 16
    xs = synth.partials(P, nb, B, dtype, 0.05, 20.0, seed=21)
    y, p1, p2 = oracle.allreduce(xs, dtype, bits, B)
    v = np.stack([oracle.widen(x, dtype).astype(np.float64) for x in xs])
    exact = v.sum(0)
    yv = oracle.widen(y, dtype).astype(np.float64)
    s1 = np.stack([np.repeat(p.scales.astype(np.float64), B) for p in p1])
    s2 = np.repeat(p2.scales.astype(np.float64), B)
    step = 0.5 + qmax * 2.0 ** -21
    bound = step * s1.sum(0) + step * s2
    bound += P * 2.0 ** -24 * (np.abs(v).sum(0) + s1.sum(0) * qmax)   # fp32 sum rounding
    ulp_out = 2.0 ** -11 if dtype == oracle.FP16 else 2.0 ** -8
    bound += ulp_out * np.abs(yv) + 2.0 ** -24
    assert np.all(np.abs(yv - exact) <= bound)


def test_codes_monotone_and_min_code_zero():
    x = synth.uniform_partials(1, 128 * 16, oracle.FP16, seed=17)[0]
    p = oracle.quantize(x, oracle.FP16, 8, 128)
    v = oracle.widen(x, oracle.FP16)
    q = unpack_codes(p.codes, x.size, 8)
    for k in range(16):
        sl = slice(k * 128, (k + 1) * 128)
        o = np.argsort(v[sl], kind="stable")
        assert np.all(np.diff(q[sl][o]) >= 0)
        if v[sl].min() < 0:
            assert q[sl][o[0]] == 0

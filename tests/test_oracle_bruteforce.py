"""Oracle vs brute force on tiny blocks, in exact rational arithmetic.

For each block the checks characterise the result instead of re-evaluating
the oracle's expressions:
  * mn/mx are the extremes of the block together with 0 (Python min/max);
  * the scale is the fp32 value nearest to (range rounded to fp32)/qmax, its
    reciprocal the fp32 value nearest to 1/s (nearest found by comparing
    neighbours exactly);
  * the zero-point is within 1/2 of -mn/s;
  * every code is a nearest grid point: no other code in [0, qmax] lies
    closer to the value;
  * the dequantized value is the fp32 value nearest to (q - z) s, and lies
    within s/2 of the input (the closed-form bound);
Each inequality carries the slack that the fp32 roundings of d, s, 1/s, -mn/s
and v/s allow: every one is a relative error of at most 2^-24 on a quantity
of at most qmax (in units of s), so qmax * 2^-21 (in units of s) covers their
sum with room to spare.  Without the roundings the slack would be zero.
  * the reduce-scatter sum is the fp32 sequential sum over ranks 0..P-1 of the
    dequantized values, and its requantization satisfies all of the above;
  * the output is the library (numpy/torch) rounding of the dequantized sum.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from tests.exact import frac, nearest_f32, seq_sum_f32, unpack_codes

F32 = np.float32


def check_block(v, codes, s, z, bits, xhat):
    qmax = (1 << bits) - 1
    fv = [frac(a) for a in v]
    mn = min([Fraction(0)] + fv)
    mx = max([Fraction(0)] + fv)
    d32 = nearest_f32(mx - mn)
    if d32 == 0:
        assert s == F32(1.0)
    else:
        assert s == nearest_f32(frac(d32) / qmax)
    inv = nearest_f32(1 / frac(s))
    assert np.isfinite(inv)
    fs = frac(s)
    slack = Fraction(qmax, 2**21)
    assert 0 <= z <= qmax
    assert abs(Fraction(z) - (-mn) / fs) <= Fraction(1, 2) + slack
    tol = fs * slack
    for a, q, xh in zip(fv, codes, xhat):
        assert 0 <= q <= qmax
        err = abs(a - (q - z) * fs)
        for q2 in range(qmax + 1):
            assert err <= abs(a - (q2 - z) * fs) + tol, (a, q, q2, z, s)
        assert xh == nearest_f32(Fraction(int(q) - z) * fs)
        assert abs(a - frac(xh)) <= fs * (Fraction(1, 2) + slack)


def tiny_values(rng, n, dtype):
    """Mix of random values with varied magnitudes and grid values with ties."""
    kind = rng.integers(0, 3)
    if kind == 0:
        x = rng.standard_normal(n) * 2.0 ** rng.integers(-6, 6)
    elif kind == 1:      # grid points and midpoints of a power-of-two grid
        k = int(rng.integers(-8, 4))
        x = rng.integers(-40, 40, size=n) * 2.0 ** (k - 1)
    else:                # values with exact zeros and a single sign
        x = np.abs(rng.standard_normal(n)) * (1 if rng.random() < 0.5 else -1)
        x[rng.random(n) < 0.3] = 0.0
    x = x.astype(np.float32)
    if dtype == oracle.FP16:
        return x.astype(np.float16).view(np.uint16)
    return torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("dtype", [oracle.FP16, oracle.BF16])
@pytest.mark.parametrize("bits", [8, 4])
def test_quantize_bruteforce(dtype, bits):
    rng = np.random.default_rng(100 + bits + 10 * dtype)
    for trial in range(60):
        B = int(rng.choice([2, 4, 8]))
        nb = int(rng.integers(1, 4))
        x = tiny_values(rng, B * nb, dtype)
        p = oracle.quantize(x, dtype, bits, B)
        v = oracle.widen(x, dtype)
        q = unpack_codes(p.codes, x.size, bits)
        xh = oracle.dequantize(p)
        for k in range(nb):
            sl = slice(k * B, (k + 1) * B)
            check_block(v[sl], q[sl], p.scales[k], int(p.zps[k]), bits, xh[sl])


@pytest.mark.parametrize("dtype", [oracle.FP16, oracle.BF16])
@pytest.mark.parametrize("bits", [8, 4])
def test_allreduce_bruteforce(dtype, bits):
    rng = np.random.default_rng(200 + bits + 10 * dtype)
    for trial in range(25):
        P = int(rng.integers(1, 4))
        B = int(rng.choice([2, 4, 8]))
        n = P * B * int(rng.integers(1, 3))
        xs = [tiny_values(rng, n, dtype) for _ in range(P)]
        y, p1, p2 = oracle.allreduce(xs, dtype, bits, B)
        xh1 = [oracle.dequantize(p) for p in p1]
        acc = np.array([seq_sum_f32([xh1[r][i] for r in range(P)]) for i in range(n)], dtype=np.float32)
        q2 = unpack_codes(p2.codes, n, bits)
        xh2 = oracle.dequantize(p2)
        for k in range(n // B):
            sl = slice(k * B, (k + 1) * B)
            check_block(acc[sl], q2[sl], p2.scales[k], int(p2.zps[k]), bits, xh2[sl])
        if dtype == oracle.FP16:
            ref = xh2.astype(np.float16).view(np.uint16)
        else:
            ref = torch.from_numpy(xh2).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        assert np.array_equal(y, ref)

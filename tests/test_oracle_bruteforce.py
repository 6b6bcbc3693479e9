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
  * beside those method-level checks, the pinned reading of the integer
    rounding, with zero slack: the zero-point is the nearest integer (ties to
    even) of the exact rational -mn*inv, clamped, and every code is the nearest
    integer of the exact rational v*inv plus z, clamped -- the product is
    rounded once, never first to fp32 (`test_codes_round_the_exact_product`
    builds blocks where the two readings give different codes);
  * the reduce-scatter sum is the fp32 sequential sum over ranks 0..P-1 of the
    dequantized values, and its requantization satisfies all of the above;
  * the output is the library (numpy/torch) rounding of the dequantized sum.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from tests.exact import frac, nearest_f32, rne_fraction, seq_sum_f32, unpack_codes

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
    finv = frac(inv)
    slack = Fraction(qmax, 2**21)
    assert 0 <= z <= qmax
    assert abs(Fraction(z) - (-mn) / fs) <= Fraction(1, 2) + slack
    # the pinned reading, zero slack: one rounding of the exact product
    assert z == min(max(rne_fraction(-mn * finv), 0), qmax), (z, mn, s)
    tol = fs * slack
    for a, q, xh in zip(fv, codes, xhat):
        assert 0 <= q <= qmax
        assert q == min(max(rne_fraction(a * finv) + z, 0), qmax), (a, q, z, s)
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


def format_values(dtype):
    """Every positive finite value of the input format in [2^-12, 2^3)."""
    if dtype == oracle.FP16:
        v = np.arange(0x0C00, 0x4800, dtype=np.uint16).view(np.float16).astype(np.float64)
    else:
        u = np.arange(0x3980, 0x4100, dtype=np.uint32) << 16
        v = u.view(np.float32).astype(np.float64)
    return v[np.isfinite(v) & (v > 0)]


def to_format_bits(x, dtype):
    if dtype == oracle.FP16:
        xb = np.asarray(x, dtype=np.float64).astype(np.float16)
        assert np.array_equal(xb.astype(np.float64), x)
        return xb.view(np.uint16)
    t = torch.tensor(np.asarray(x, dtype=np.float64)).to(torch.bfloat16)
    assert np.array_equal(t.to(torch.float64).numpy(), x)
    return t.view(torch.int16).numpy().view(np.uint16)


def near_tie_blocks(bits, dtype, count, seed):
    """Blocks on which rounding the exact product v*inv once and rounding its
    fp32 value first give different codes or zero-points (an input generator;
    no expected value comes from here).

    Search: draw a block maximum M and minimum mn from the input format, take
    s = RN32((M - mn)/qmax) and inv = RN32(1/s), and look among all format
    values v in [mn, M] for those whose exact product v*inv (formed in double,
    where a 24 x 24-bit product is exact) and fp32 product fall on different
    sides of a half-integer -- the fp32 product lands on the tie, or across it.
    Keep blocks [mn, M, v...] (padded with random in-range values) where at
    least one value, or the zero-point product -mn*inv, is such a case.  The
    caller's checks recompute everything in exact rationals."""
    qmax = (1 << bits) - 1
    rng = np.random.default_rng(seed)
    pos = format_values(dtype)
    vals = np.concatenate([-pos[::-1], [0.0], pos])
    out = []
    for _ in range(20000):
        if len(out) == count:
            break
        M = float(rng.choice(pos[pos >= 0.25]))
        mn = -float(rng.choice(pos[pos <= M])) if rng.random() < 0.7 else 0.0
        s = np.float32(np.float32(M) - np.float32(mn)) / np.float32(qmax)
        inv = np.float32(1.0) / s
        cand = vals[(vals >= mn) & (vals <= M)]
        exact = cand * np.float64(inv)
        r32 = (cand.astype(np.float32) * inv).astype(np.float64)
        hit = cand[np.rint(exact) != np.rint(r32)]
        z_hit = np.rint(-mn * np.float64(inv)) != np.rint(np.float64(np.float32(-mn) * inv))
        if hit.size == 0 and not z_hit:
            continue
        B = int(rng.choice([4, 8]))
        fill = rng.choice(cand, size=B)
        fill[:2] = [mn, M]
        fill[2:2 + min(hit.size, B - 2)] = hit[: B - 2]
        out.append(to_format_bits(rng.permutation(fill), dtype))
    assert len(out) == count, "near-tie search came up short"
    return out


def readings_differ(v, bits):
    """Whether the exact-product and fp32-first readings give a different code or
    zero-point somewhere in the block (exact rationals only)."""
    qmax = (1 << bits) - 1
    fv = [frac(a) for a in v]
    mn, mx = min([Fraction(0)] + fv), max([Fraction(0)] + fv)
    d32 = nearest_f32(mx - mn)
    if d32 == 0:
        return False
    finv = frac(nearest_f32(1 / frac(nearest_f32(frac(d32) / qmax))))
    prods = [-mn * finv] + [a * finv for a in fv]
    return any(rne_fraction(p) != rne_fraction(frac(nearest_f32(p))) for p in prods)


@pytest.mark.parametrize("dtype", [oracle.FP16, oracle.BF16])
@pytest.mark.parametrize("bits", [8, 4])
def test_codes_round_the_exact_product(dtype, bits):
    """Codes and zero-points on near-tie blocks: one rounding of the exact
    product (check_block's zero-slack assertions), where rounding the product to
    fp32 first would give a different code or zero-point."""
    blocks = near_tie_blocks(bits, dtype, 12, 300 + bits + 10 * dtype)
    for x in blocks:
        B = x.size
        assert readings_differ(oracle.widen(x, dtype), bits)
        p = oracle.quantize(x, dtype, bits, B)
        v = oracle.widen(x, dtype)
        q = unpack_codes(p.codes, B, bits)
        check_block(v, q, p.scales[0], int(p.zps[0]), bits, oracle.dequantize(p))

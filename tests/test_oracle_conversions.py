"""Oracle fp16/bf16 conversions vs library conversions (numpy, torch).

Widening is checked on every 16-bit pattern; narrowing on every fp16/bf16
value, every exact midpoint between neighbours (the ties), the fp32 values
one ulp either side of each midpoint, the overflow thresholds and a random
sample of all finite fp32 patterns."""
import numpy as np
import torch

import oracle


def all_u16():
    return np.arange(65536, dtype=np.uint32).astype(np.uint16)


def test_widen_fp16_exhaustive():
    h = all_u16()
    got = oracle.widen(h, oracle.FP16)
    ref = h.view(np.float16).astype(np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_widen_bf16_exhaustive():
    h = all_u16()
    got = oracle.widen(h, oracle.BF16)
    ref = torch.from_numpy(h.view(np.int16)).view(torch.bfloat16).to(torch.float32).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def narrow_cases(dtype):
    h = all_u16()
    vals = oracle.widen(h, dtype)
    fin = np.sort(np.unique(vals[np.isfinite(vals)]).astype(np.float64))
    mids = (fin[:-1] + fin[1:]) / 2.0           # exact in fp64; exact in fp32 too
    mids32 = mids.astype(np.float32)
    assert np.array_equal(mids32.astype(np.float64), mids)
    up = np.nextafter(mids32, np.float32(np.inf))
    dn = np.nextafter(mids32, np.float32(-np.inf))
    rng = np.random.default_rng(7)
    rnd = rng.integers(0, 2**32, size=2_000_000, dtype=np.uint64).astype(np.uint32).view(np.float32)
    rnd = rnd[np.isfinite(rnd)]
    edges = np.array([65504.0, 65519.996, 65520.0, 65536.0, 3.0e38, 3.3895e38, 3.4e38,
                      2.0**-24, 2.0**-25, 2.0**-26, 1.5 * 2.0**-25, 2.0**-133, 2.0**-134,
                      1.5 * 2.0**-134, 1e-45, 0.0], dtype=np.float32)
    c = np.concatenate([fin.astype(np.float32), mids32, up, dn, rnd, edges])
    return np.concatenate([c, -c])


def test_narrow_fp16_vs_numpy():
    c = narrow_cases(oracle.FP16)
    got = oracle.narrow(c, oracle.FP16)
    with np.errstate(over="ignore"):
        ref = c.astype(np.float16).view(np.uint16)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(float(c[i]), hex(got[i]), hex(ref[i])) for i in bad[:5]]


def test_narrow_bf16_vs_torch():
    c = narrow_cases(oracle.BF16)
    got = oracle.narrow(c, oracle.BF16)
    ref = torch.from_numpy(c).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, [(float(c[i]), hex(got[i]), hex(ref[i])) for i in bad[:5]]

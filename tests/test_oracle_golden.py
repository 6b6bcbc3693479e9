"""Oracle vs hand-derived worked examples (tests/golden/*.json).

Each fixture states its derivation; every value in it is a dyadic rational, so
the expected codes, scales, zero-points and outputs follow from the pinned
definitions by exact hand arithmetic."""
import glob
import json
import os

import numpy as np
import pytest

import oracle

GOLDEN = sorted(glob.glob(os.path.join(os.path.dirname(__file__), "golden", "*.json")))
DT = {"fp16": oracle.FP16, "bf16": oracle.BF16}


def to_bits(vals, dtype):
    x = np.asarray(vals, dtype=np.float64)
    if dtype == oracle.FP16:
        b = x.astype(np.float16)
        assert np.array_equal(b.astype(np.float64), x), "fixture value not exact in fp16"
        return b.view(np.uint16)
    import torch
    t = torch.tensor(x, dtype=torch.float64).to(torch.bfloat16)
    assert np.array_equal(t.to(torch.float64).numpy(), x), "fixture value not exact in bf16"
    return t.view(torch.int16).numpy().view(np.uint16)


def f32_bits(a):
    return np.asarray(a, dtype=np.float32).view(np.uint32)


@pytest.mark.parametrize("path", GOLDEN, ids=[os.path.basename(p) for p in GOLDEN])
def test_golden(path):
    fx = json.load(open(path))
    assert fx["cite"] and fx["derivation"]
    bits, block = fx["bits"], fx["block"]
    for dname in fx["dtypes"]:
        dt = DT[dname]
        xs = [to_bits(r, dt) for r in fx["x"]]
        for r, x in enumerate(xs):
            p = oracle.quantize(x, dt, bits, block)
            e = fx["step1"][r]
            assert p.codes.tolist() == e["codes"], (dname, r)
            assert np.array_equal(f32_bits(p.scales), f32_bits(e["scales"])), (dname, r)
            assert p.zps.tolist() == e["zps"], (dname, r)
            if "xhat1" in fx:
                xh = oracle.dequantize(p)
                assert np.array_equal(f32_bits(xh), f32_bits(fx["xhat1"][r])), (dname, r)
        if "step2" in fx:
            y, p1, p2 = oracle.allreduce(xs, dt, bits, block)
            e = fx["step2"]
            assert p2.codes.tolist() == e["codes"], dname
            assert np.array_equal(f32_bits(p2.scales), f32_bits(e["scales"])), dname
            assert p2.zps.tolist() == e["zps"], dname
            assert np.array_equal(y, to_bits(fx["y"], dt)), dname
            # the staged entry points agree with the composed call
            p2s = oracle.rs_dequant_sum_requant(p1)
            assert np.array_equal(p2s.codes, p2.codes)
            assert np.array_equal(oracle.ag_dequant(p2s, dt), y)

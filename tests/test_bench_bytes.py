"""The algorithmic bytes behind every roofline figure of bench.py: per
quantization W2 = n*b/8 + 5*n/B (codes, fp32 scale, uint8 zero-point), fused
with payloads P*n*2 + n*2 + P*W2 + W2, output only P*n*2 + n*2, staged
P*n*2 + 2*P*W2 + 2*W2 + n*2 -- checked against byte counts worked out by
hand for each workload."""
import importlib.util
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    argv = sys.argv
    sys.argv = ["bench.py"]
    try:
        spec.loader.exec_module(mod)
    finally:
        sys.argv = argv
    return mod


# (workload, fused bytes, staged bytes, output-only bytes or None)
TABLE = [
    ("p2_fp16_64x1024_int8_b128", 597_504, 801_792, None),
    ("p4_fp16_8192x8192_int8_b128", 1_019_740_160, 1_368_391_680, 671_088_640),
    ("p4_fp16_8192x8192_int4_b128", 851_968_000, 1_032_847_360, None),
    ("p8_bf16_16384x4096_int4_b4096", 1_510_686_720, 1_813_413_888, None),
    ("p8_bf16_16384x4096_int4_b128", 1_533_542_400, 1_859_125_248, None),
    ("p4_fp16_8x8192_int8_b128", 995_840, 1_336_320, None),
]


@pytest.mark.parametrize("name,fused,staged,out_only", TABLE, ids=[t[0] for t in TABLE])
def test_algorithmic_bytes(bench, name, fused, staged, out_only):
    w = bench.WORKLOADS[name]
    assert bench.algorithmic_bytes(w, "fused") == fused
    assert bench.algorithmic_bytes(w, "staged") == staged
    assert bench.algorithmic_bytes(w, "fused_nopayload") == w.P * w.n * 2 + w.n * 2
    if out_only is not None:
        assert bench.algorithmic_bytes(w, "fused_nopayload") == out_only


def test_job_throughput_is_the_aggregate(bench):
    assert bench.job_throughput(10**9, 1, 1000.0) == pytest.approx(1.0)
    assert bench.job_throughput(10**9, 8, 1000.0) == pytest.approx(8.0)

"""The oracle's pins reject planted mistakes.

Each case copies fco.c, plants one plausible mistake (a dropped term, a wrong
sign, an operand in the wrong place, a different rounding, a different order),
builds the copy on the CPU and runs the pin battery (hand-derived fixtures,
brute force, closed forms, conversions) against it.  At least one pin must
fail for every mutant, and the unmodified file must pass the same battery."""
import os
import subprocess

import pytest

import oracle
from tests import test_oracle_bruteforce as bf
from tests import test_oracle_conversions as cv
from tests import test_oracle_golden as gd
from tests import test_oracle_invariants as inv

SRC = os.path.join(os.path.dirname(oracle.__file__), "fco.c")

MUTANTS = {
    "range_without_zero": ("float mn = 0.0f, mx = 0.0f;", "float mn = v[0], mx = v[0];"),
    "zero_point_sign": ("rne_product(-mn, inv)", "rne_product(mn, inv)"),
    "zero_point_before_rounding": ("return clamp_int(rne_product(v, inv) + z, 0, qmax);",
                                   "return clamp_int((int)nearbyint((double)v * inv + z), 0, qmax);"),
    "no_code_clamp": ("return clamp_int(rne_product(v, inv) + z, 0, qmax);",
                      "return rne_product(v, inv) + z;"),
    "ties_away_from_zero": ("return (int)nearbyint(t);", "return (int)round(t);"),
    "high_nibble_first": ("} else if (i % 2 == 0) {", "} else if (i % 2 == 1) {",
                          "return (i % 2 == 0) ? (codes[i / 2] & 0x0f) : (codes[i / 2] >> 4);",
                          "return (i % 2 == 1) ? (codes[i / 2] & 0x0f) : (codes[i / 2] >> 4);"),
    "rank_order_reversed": ("codes[r], e, bits), scales[r][k], zps[r][k]",
                            "codes[P - r], e, bits), scales[P - r][k], zps[P - r][k]"),
    "sum_in_double": ("float a = fco_dequantize_value(", "double a = fco_dequantize_value("),
    "dequant_sign": ("float qz = (float)(q - z);", "float qz = (float)(z - q);"),
    "scale_over_2_pow_b": ("d / (float)qmax;", "d / (float)(qmax + 1);"),
    "symmetric_range": ("float d = mx - mn;", "float d = 2.0f * fmaxf(mx, -mn);"),
    "output_truncated": ("double kr = nearbyint(k);", "double kr = floor(k);"),
    "zero_block_scale_zero": ("(d == 0.0f) ? 1.0f :", "(d == 0.0f) ? 0.0f :"),
    # the doubly rounded reading: the product rounded to fp32, then to an integer
    "product_rounded_to_fp32_first": ("double t = (double)a * (double)b;", "double t = (double)(float)(a * b);"),
    "reciprocal_from_range": ("float inv = 1.0f / s;", "float inv = (d == 0.0f) ? 1.0f : (float)qmax / d;"),
    "extremes_skip_last_element": ("for (int i = 0; i < B; i++) {\n        if (!isfinite(v[i]))",
                                   "for (int i = 0; i < B - 1; i++) {\n        if (!isfinite(v[i]))"),
    "dequant_divides_by_reciprocal": ("    return qz * s;", "    return qz / (1.0f / s);"),
    "f16_subnormal_read_as_normal": ("        v = ldexp((double)f, -24);", "        v = ldexp((double)(1024 + f), -25);"),
    "f16_subnormal_threshold_one_binade_low": ("    if (r < ldexp(1.0, -14))    /* subnormal",
                                               "    if (r < ldexp(1.0, -15))    /* subnormal"),
    "f16_largest_finite_overflows": ("    if (r > 65504.0)", "    if (r >= 65504.0)"),
    "sum_drops_last_rank": ("for (int r = 1; r < P; r++) {\n                    float xr",
                            "for (int r = 1; r < P - 1; r++) {\n                    float xr"),
}


def battery():
    for path in gd.GOLDEN:
        gd.test_golden(path)
    for dt in (oracle.FP16, oracle.BF16):
        for bits in (8, 4):
            bf.test_quantize_bruteforce(dt, bits)
            bf.test_allreduce_bruteforce(dt, bits)
            bf.test_codes_round_the_exact_product(dt, bits)
            inv.test_grid_round_trip(dt, bits)
            inv.test_allreduce_error_bound(dt, bits)
    cv.test_narrow_fp16_vs_numpy()
    cv.test_narrow_bf16_vs_torch()


def build_variant(tmp_path, name, edits):
    text = open(SRC).read()
    for old, new in zip(edits[0::2], edits[1::2]):
        assert text.count(old) == 1, (name, old)
        text = text.replace(old, new)
    src = tmp_path / f"fco_{name}.c"
    src.write_text(text)
    so = tmp_path / f"libfco_{name}.so"
    subprocess.run(["gcc", *oracle.CFLAGS, "-o", str(so), str(src), "-lm"], check=True)
    return str(so)


def test_unmodified_build_passes_battery(tmp_path):
    so = build_variant(tmp_path, "same", ())
    with oracle.use_library(so):
        battery()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, name):
    so = build_variant(tmp_path, name, MUTANTS[name])
    with oracle.use_library(so):
        with pytest.raises((AssertionError, oracle.OracleError)):
            battery()

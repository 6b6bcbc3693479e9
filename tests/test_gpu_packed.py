"""The kernels' packed fp32 pair operations (two binary32 operations per
instruction, sm_100) equal the scalar round-to-nearest-even operations lane by
lane, and the rank-order accumulation built from them rounds the product and the sum
separately, as the reduce-scatter's definition requires, in both forms the
kernels use: a packed product formed as an FMA with a zero addend followed by
a packed add, and a packed multiply followed by scalar adds.  (A packed add of
a packed multiply's result would not: the compiler may fuse the two into one
packed FMA.)"""
import ctypes
import os
import subprocess

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module")
def checker(tmp_path_factory):
    from bit_quantized_all_block_b200 import build as B
    out = str(tmp_path_factory.mktemp("pk") / "libpackedcheck.so")
    subprocess.run([B.nvcc(), *B.NVCC_FLAGS, "-shared", "-o", out, os.path.join(HERE, "cuda", "packed_check.cu")],
                   check=True)
    lib = ctypes.CDLL(out)
    lib.fc_check_packed.argtypes = [ctypes.c_int, ctypes.c_ulonglong, ctypes.c_uint,
                                    ctypes.POINTER(ctypes.c_ulonglong)]
    return lib


@pytest.mark.parametrize("which", [0, 1], ids=["ops", "accumulate"])
def test_packed_matches_scalar(checker, which):
    bad = ctypes.c_ulonglong()
    for seed in (1, 2):
        assert checker.fc_check_packed(which, 1 << 26, seed, ctypes.byref(bad)) == 0
        assert bad.value == 0, f"{bad.value} of {1 << 26} differ (seed {seed})"
